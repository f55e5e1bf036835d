"""Dense attention (svg2_dense_attn: the one-cluster case of the tcgen05 attention kernel) vs the
oracle's float64 textbook attention over all keys.  Same bar as the sparse kernel: max-abs 2e-2,
mean-abs 2e-3, relative L2 1e-2.  The sizes span several 128-row tiles and 256-row units with a ragged tail, d = 128
and d = 64, and the full Wan-720p length on sampled rows."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, require_gpu

MAX_ABS, MEAN_ABS, REL_L2 = 2e-2, 2e-3, 1e-2


def _rel(got, ref):
    return float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30))


def _rand(rng, shape):
    return I.round_to_bf16(rng.standard_normal(shape, dtype=np.float32))


def _dense_gpu(svg2, Q, K, V, scale):
    B, H, N, d = Q.shape
    O = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    ws = svg2.dense_workspace(B, H, N, d)
    svg2.svg2_dense_attn(bf16_dev(Q), bf16_dev(K), bf16_dev(V), scale, O, ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    return host(O).astype(np.float64)


@pytest.mark.gpu
@pytest.mark.parametrize("H,N,d,rows", [
    (2, 1000, 128, None),      # 8 Q tiles, the last ragged; 4 units
    (3, 4096, 64, None),       # d = 64, whole tiles
    (1, 257, 128, None),       # one row past a unit
    (1, 1, 128, None),         # a single token
    (2, 12480, 128, 200),      # the small shape's length, sampled rows
])
def test_dense_matches_oracle(oracle, H, N, d, rows):
    svg2 = require_gpu()
    rng = np.random.default_rng(N * 7 + d + H)
    Q, K, V = (_rand(rng, (1, H, N, d)) for _ in range(3))
    scale = float(np.float32(1.0 / np.sqrt(d)))
    out = _dense_gpu(svg2, Q, K, V, scale)
    errs = []
    for h in range(H):
        sel = None if rows is None else np.sort(rng.choice(N, rows, replace=False))
        ref = oracle.dense_attention_rows(Q[0, h], K[0, h], V[0, h], scale, sel)
        got = out[0, h] if sel is None else out[0, h][sel]
        errs.append(np.abs(got - ref))
        assert _rel(got, ref) <= REL_L2, (h, _rel(got, ref))
    err = np.concatenate([e.ravel() for e in errs])
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


@pytest.mark.gpu
def test_dense_at_wan_length_sampled_rows(oracle):
    """The Wan-720p length (75600 keys per row) on two heads, 64 sampled rows each."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["wan720p"]
    rng = np.random.default_rng(5)
    H, N, d = 2, cfg.N, cfg.d
    Q, K, V = (_rand(rng, (1, H, N, d)) for _ in range(3))
    scale = float(np.float32(cfg.scale))
    out = _dense_gpu(svg2, Q, K, V, scale)
    for h in range(H):
        sel = np.sort(rng.choice(N, 64, replace=False))
        ref = oracle.dense_attention_rows(Q[0, h], K[0, h], V[0, h], scale, sel)
        err = np.abs(out[0, h][sel] - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (h, err.max(), err.mean())
        assert _rel(out[0, h][sel], ref) <= REL_L2, (h, _rel(out[0, h][sel], ref))


@pytest.mark.gpu
def test_dense_matches_torch_sdpa():
    """The same softmax as torch's scaled_dot_product_attention on the same bf16 tensors, at the small
    shape's length (both bf16 kernels: they agree to rounding)."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    rng = np.random.default_rng(9)
    B, H, N, d = 1, 2, cfg.N, cfg.d
    Q, K, V = (_rand(rng, (B, H, N, d)) for _ in range(3))
    scale = float(np.float32(cfg.scale))
    dense = _dense_gpu(svg2, Q, K, V, scale)
    sdpa = torch.nn.functional.scaled_dot_product_attention(bf16_dev(Q), bf16_dev(K), bf16_dev(V), scale=scale)
    err = np.abs(dense - host(sdpa).astype(np.float64))
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert _rel(dense, host(sdpa).astype(np.float64)) <= REL_L2
