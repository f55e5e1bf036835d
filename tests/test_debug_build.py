"""The debug build of the library (libsvg2_debug.so, compiled with -DSVG2_DEBUG): the same parity
cases pass with no device error, and data-derived indices out of range -- which both builds clamp or
skip, so nothing is read or written out of bounds -- are reported as SVG2_ERR_DEVICE_BOUNDS with the
kernel's tag instead of passing silently."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import build as Bld
from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, pool_layer_inputs, require_gpu, to_dev
from tests.test_parity_attn import SCALE, _case, _compare, _ell

BOUNDS = 6


@pytest.fixture
def debug_svg2():
    svg2 = require_gpu()
    Bld.build(debug=True)
    svg2.use_debug_library(True)
    try:
        yield svg2
    finally:
        svg2.use_debug_library(False)


@pytest.mark.gpu
def test_debug_build_attention_parity(oracle, debug_svg2):
    svg2 = debug_svg2
    c = _case(3, 12480, 64, 256, 0.5, 2)
    sel_count, sel_idx = _ell(c["mask"])
    O = torch.zeros(1, 2, 12480, 128, dtype=torch.bfloat16, device="cuda")
    ws = svg2.workspace(1, 2, 12480, 128, 64, 256)
    svg2.svg2_sparse_attn(bf16_dev(c["Qp"]), bf16_dev(c["Kp"]), bf16_dev(c["Vp"]), to_dev(c["q_off"]),
                          to_dev(c["k_off"]), to_dev(sel_count), to_dev(sel_idx), SCALE, O, ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    _compare(oracle, c, host(O), SCALE)


@pytest.mark.gpu
def test_debug_build_layer_small_heads(oracle, debug_svg2):
    from tests.test_layer import check_head, run_layer
    svg2 = debug_svg2
    cfg = I.CONFIGS["small"]
    data = pool_layer_inputs(cfg, range(2))
    res = run_layer(svg2, cfg, data, 0.9)           # raises on any device status
    for h in range(2):
        check_head(oracle, cfg, data, res, h, 0.9, rows=np.arange(0, cfg.N, 13))


@pytest.mark.gpu
def test_debug_build_reports_out_of_range_indices(debug_svg2):
    svg2 = debug_svg2
    c = _case(4, 700, 3, 5, 0.6, 1)
    sel_count, sel_idx = _ell(c["mask"])
    sel_idx[0, 0, 0, 0] = 5 + 3                      # a kept-cluster index past nK
    O = torch.zeros(1, 1, 700, 128, dtype=torch.bfloat16, device="cuda")
    ws = svg2.workspace(1, 1, 700, 128, 3, 5)
    svg2.svg2_sparse_attn(bf16_dev(c["Qp"]), bf16_dev(c["Kp"]), bf16_dev(c["Vp"]), to_dev(c["q_off"]),
                          to_dev(c["k_off"]), to_dev(sel_count), to_dev(sel_idx), SCALE, O, ws)
    torch.cuda.synchronize()
    code, where, info = svg2.svg2_check_status(ws)
    assert code == BOUNDS and where == 15 and info[1] == 8, (code, where, info)   # plan / range table
    # a permutation entry past N in the fused inverse permutation
    perm = np.random.default_rng(0).permutation(700).astype(np.int32)[None, None]
    perm[0, 0, 17] = 700 + 9
    sel_count, sel_idx = _ell(c["mask"])
    svg2.svg2_sparse_attn(bf16_dev(c["Qp"]), bf16_dev(c["Kp"]), bf16_dev(c["Vp"]), to_dev(c["q_off"]),
                          to_dev(c["k_off"]), to_dev(sel_count), to_dev(sel_idx), SCALE, O, ws,
                          perm_q=to_dev(perm))
    torch.cuda.synchronize()
    code, where, info = svg2.svg2_check_status(ws)
    assert code == BOUNDS and where == 5 and info == (17, 709), (code, where, info)  # attention epilogue
    # the release build clamps the same inputs silently
    svg2.use_debug_library(False)
    svg2.svg2_sparse_attn(bf16_dev(c["Qp"]), bf16_dev(c["Kp"]), bf16_dev(c["Vp"]), to_dev(c["q_off"]),
                          to_dev(c["k_off"]), to_dev(sel_count), to_dev(sel_idx), SCALE, O, ws,
                          perm_q=to_dev(perm))
    torch.cuda.synchronize()
    assert svg2.svg2_check_status(ws)[0] == 0
