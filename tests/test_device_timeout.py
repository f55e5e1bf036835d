"""The give-up path of the bounded device waits (no fault, no hang): a workspace whose wait budget
is a few cycles makes the attention's and the tensor-core assignment's waits run out.  The call
must latch SVG2_ERR_DEVICE_TIMEOUT with the tag of a kernel that waited, the context must stay
usable, and the next call on the same workspace with the default budget must be correct (equal to
a call on a fresh workspace)."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, require_gpu, to_dev
from tests.test_parity_attn import SCALE, _case, _ell

TIMEOUT = 5
ATTN_TAGS = {3, 4, 5}      # key/value producer, MMA issuer, softmax
ASSIGN_TAGS = {2, 7}       # assignment pipeline, its epilogue's tile wait


def _attn(svg2, c, ws):
    B, H, N, d = c["Qp"].shape
    nQ, nK = c["mask"].shape[-2:]
    sel_count, sel_idx = _ell(c["mask"])
    O = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    svg2.svg2_sparse_attn(bf16_dev(c["Qp"]), bf16_dev(c["Kp"]), bf16_dev(c["Vp"]), to_dev(c["q_off"]),
                          to_dev(c["k_off"]), to_dev(sel_count), to_dev(sel_idx), SCALE, O, ws)
    return O


@pytest.mark.gpu
def test_attention_wait_timeout_is_reported_and_recovered():
    svg2 = require_gpu()
    c = _case(3, 12480, 64, 256, 0.5, 2)
    ws = svg2.workspace(1, 2, 12480, 128, 64, 256)
    svg2.svg2_set_wait_budget(ws, 1)
    _attn(svg2, c, ws)
    torch.cuda.synchronize()
    code, where, _ = svg2.svg2_check_status(ws)
    assert code == TIMEOUT and where in ATTN_TAGS, (code, where)
    svg2.svg2_set_wait_budget(ws, 0)
    again = _attn(svg2, c, ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    fresh_ws = svg2.workspace(1, 2, 12480, 128, 64, 256)
    fresh = _attn(svg2, c, fresh_ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(fresh_ws)
    assert torch.equal(again, fresh)


def _assign(svg2, X, C0, ws):
    B, H, N, d = X.shape
    C = to_dev(C0)
    lab = torch.zeros(B, H, N, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, H, C0.shape[2], dtype=torch.int32, device="cuda")
    svg2.svg2_kmeans(bf16_dev(X), C0.shape[2], 1, svg2.SVG2_INIT_GIVEN, C, lab, cnt, ws)
    return C, lab


@pytest.mark.gpu
def test_assignment_wait_timeout_is_reported_and_recovered():
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    data = I.layer_inputs(cfg, 0, [0, 1])
    X = data["k"]
    rng = np.random.default_rng(4)
    C0 = X[:, :, rng.choice(X.shape[2], cfg.nK, replace=False)].astype(np.float32)
    ws = svg2.workspace(1, 2, cfg.N, cfg.d, cfg.nK, cfg.nK)
    svg2.svg2_set_wait_budget(ws, 1)
    _assign(svg2, X, C0, ws)
    torch.cuda.synchronize()
    code, where, _ = svg2.svg2_check_status(ws)
    assert code == TIMEOUT and where in ASSIGN_TAGS, (code, where)
    svg2.svg2_set_wait_budget(ws, 0)
    C, lab = _assign(svg2, X, C0, ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    fresh_ws = svg2.workspace(1, 2, cfg.N, cfg.d, cfg.nK, cfg.nK)
    C2, lab2 = _assign(svg2, X, C0, fresh_ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(fresh_ws)
    assert torch.equal(lab, lab2) and torch.equal(C, C2)
