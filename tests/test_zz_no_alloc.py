"""svg2_sparse_attn_noalloc, the sparse-attention entry point for callers that cannot allocate
device memory at call time: its scratch is a fixed array inside the library instead of a
workspace.  Checked through the C ABI against svg2_sparse_attn on the same inputs, for two calls
in a row with different inputs (the shared array must not carry anything from the first call
into the second).  Both entry points run the same kernel on the same work plan, so their outputs
must be identical bit for bit.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, require_gpu, to_dev

SCALE = float(np.float32(1 / np.sqrt(128)))


def _inputs(seed, H, N, nQ, nK, density):
    rng = np.random.default_rng(seed)
    q_off, k_off, masks = [], [], []
    for h in range(H):
        lq = I.random_labels(N, nQ, seed + 10 * h, 0.1)
        lk = I.random_labels(N, nK, seed + 10 * h + 5, 0.1)
        qo = np.concatenate([[0], np.cumsum(np.bincount(lq, minlength=nQ))]).astype(np.int32)
        ko = np.concatenate([[0], np.cumsum(np.bincount(lk, minlength=nK))]).astype(np.int32)
        m = (rng.random((nQ, nK)) < density).astype(np.uint8)
        ck = np.diff(ko)
        m[:, ck == 0] = 0
        for i in range(nQ):
            if not m[i].any():
                m[i, int(np.argmax(ck))] = 1
        q_off.append(qo)
        k_off.append(ko)
        masks.append(m)
    mask = np.stack(masks)[None]
    sel_count = mask.sum(-1).astype(np.int32)
    sel_idx = np.zeros(mask.shape, np.int32)
    for idx in np.ndindex(*mask.shape[:-1]):
        kept = np.nonzero(mask[idx])[0]
        sel_idx[idx][:kept.size] = kept
    qkv = [bf16_dev(rng.standard_normal((1, H, N, 128), dtype=np.float32)) for _ in range(3)]
    perm = np.stack([rng.permutation(N).astype(np.int32) for _ in range(H)])[None]
    return dict(Qp=qkv[0], Kp=qkv[1], Vp=qkv[2], q_off=to_dev(np.stack(q_off)[None]),
                k_off=to_dev(np.stack(k_off)[None]), sel_count=to_dev(sel_count), sel_idx=to_dev(sel_idx),
                perm_q=to_dev(perm))


@pytest.mark.gpu
def test_noalloc_entry_point_matches_workspace_entry_point():
    svg2 = require_gpu()
    for call, (seed, H, N, nQ, nK, density) in enumerate([(11, 2, 5000, 24, 60, 0.4), (12, 3, 3000, 16, 40, 0.7)]):
        c = _inputs(seed, H, N, nQ, nK, density)
        ref = torch.zeros(1, H, N, 128, dtype=torch.bfloat16, device="cuda")
        ws = svg2.workspace(1, H, N, 128, nQ, nK)
        svg2.svg2_sparse_attn(c["Qp"], c["Kp"], c["Vp"], c["q_off"], c["k_off"], c["sel_count"], c["sel_idx"],
                              SCALE, ref, ws, perm_q=c["perm_q"])
        out = torch.zeros_like(ref)
        status = torch.zeros(4, dtype=torch.int32, device="cuda")
        svg2.svg2_sparse_attn_noalloc(c["Qp"], c["Kp"], c["Vp"], c["q_off"], c["k_off"], c["sel_count"],
                                      c["sel_idx"], SCALE, out, perm_q=c["perm_q"], device_status=status)
        torch.cuda.synchronize()
        svg2.raise_on_device_error(ws)
        assert int(status[0].item()) == 0, f"call {call}: device status {status.tolist()}"
        assert torch.isfinite(out.float()).all()
        diff = int((out != ref).sum().item())
        assert torch.equal(out, ref), f"call {call}: {diff} output elements differ from svg2_sparse_attn"


@pytest.mark.gpu
def test_noalloc_entry_point_rejects_sizes_beyond_its_array():
    svg2 = require_gpu()
    L = svg2.lib()
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    rc = L.svg2_sparse_attn_noalloc(fake, fake, fake, fake, fake, fake, fake, 1, 1024, 1 << 20, 128, 1024, 1024,
                                    ctypes.c_float(SCALE), None, fake, None, None)
    assert rc == 2  # SVG2_ERR_UNSUPPORTED
