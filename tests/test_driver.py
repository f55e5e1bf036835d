"""The denoising-loop driver (svg2_driver_*): its schedule and argument checks on the host, and on
the GPU that every call equals the layer call it stands for (dense, cold, or warm from the same
layer's previous centroids), bit for bit, with the cache holding exactly those centroids."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import build as B
from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, require_gpu, to_dev

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: the calls below stop at validation


@pytest.fixture(scope="module")
def svg2():
    B.build()
    from sparse_attention_video_head_b200 import svg2 as s
    return s


def _cfg(svg2, **kw):
    p = svg2.LayerParams(nQ=kw.pop("nQ", 8), nK=kw.pop("nK", 16), iters=kw.pop("iters", 3))
    c = dict(num_steps=6, num_layers=2, dense_steps=1, warm_iters=2)
    c.update(kw)
    return svg2.SvgDriverConfig(c["num_steps"], c["num_layers"], c["dense_steps"], c["warm_iters"], p.c())


def _create(svg2, cfg, B=1, H=2, N=1000, d=128):
    h = ctypes.c_void_p(None)
    rc = svg2.lib().svg2_driver_create(ctypes.byref(cfg), B, H, N, d, ctypes.byref(h))
    return rc, h


def test_schedule_before_any_call(svg2):
    d = svg2.Driver(1, 2, 1000, 128, num_steps=10, num_layers=3, dense_steps=2, warm_iters=2,
                    params=svg2.LayerParams(nQ=8, nK=16, iters=3), allocate=False)
    for layer in range(3):
        assert [d.plan(s, layer) for s in range(10)] == [svg2.SVG2_STEP_DENSE] * 2 + [svg2.SVG2_STEP_COLD] * 8
    # cache: per layer [B,H,nQ,d] then [B,H,nK,d] float32
    assert d.cache_bytes() == 3 * 1 * 2 * (8 + 16) * 128 * 4
    assert d.workspace_bytes() >= svg2.svg2_workspace_size(1, 2, 1000, 128, 8, 16)
    assert d.workspace_bytes() >= svg2.svg2_dense_attn_workspace_size(1, 2, 1000, 128)
    d.close()


def test_config_validation(svg2):
    assert _create(svg2, _cfg(svg2))[0] == OK
    for bad in (dict(num_steps=0), dict(num_layers=0), dict(dense_steps=-1), dict(dense_steps=7),
                dict(warm_iters=0), dict(iters=0), dict(nQ=0), dict(nK=1001)):
        assert _create(svg2, _cfg(svg2, **bad))[0] == INVALID, bad
    assert _create(svg2, _cfg(svg2), d=96)[0] == UNSUPPORTED
    assert _create(svg2, _cfg(svg2), N=0)[0] == INVALID
    L = svg2.lib()
    assert L.svg2_driver_create(ctypes.byref(_cfg(svg2)), 1, 2, 1000, 128, None) == INVALID
    assert L.svg2_driver_create(None, 1, 2, 1000, 128, ctypes.byref(ctypes.c_void_p())) == INVALID


def test_call_validation(svg2):
    L = svg2.lib()
    rc, h = _create(svg2, _cfg(svg2))
    assert rc == OK
    kind = ctypes.c_int(-1)
    assert L.svg2_driver_plan(h, 6, 0, ctypes.byref(kind)) == INVALID    # step out of range
    assert L.svg2_driver_plan(h, 0, 2, ctypes.byref(kind)) == INVALID    # layer out of range
    assert L.svg2_driver_plan(h, -1, 0, ctypes.byref(kind)) == INVALID
    assert L.svg2_driver_plan(None, 0, 0, ctypes.byref(kind)) == INVALID
    args = lambda step, uq=FAKE: (h, step, 0, FAKE, FAKE, FAKE, uq, FAKE, FAKE, FAKE, 1 << 30, None)
    assert L.svg2_driver_layer(*args(1)) == WORKSPACE                      # sparse step, no cache bound
    need = ctypes.c_size_t(0)
    assert L.svg2_driver_cache_bytes(h, ctypes.byref(need)) == OK
    assert L.svg2_driver_bind_cache(h, FAKE, need.value - 4) == WORKSPACE
    assert L.svg2_driver_bind_cache(h, ctypes.c_void_p(0x10004), need.value) == INVALID  # not 16-byte aligned
    assert L.svg2_driver_bind_cache(h, FAKE, need.value) == OK
    assert L.svg2_driver_layer(*args(1, uq=None)) == INVALID               # cold start needs the uniforms
    assert L.svg2_driver_layer(*args(7)) == INVALID
    assert L.svg2_driver_reset(h) == OK and L.svg2_driver_reset(None) == INVALID
    assert L.svg2_driver_destroy(h) == OK


@pytest.mark.gpu
@pytest.mark.parametrize("attn_fp8", [0, 1])
def test_driver_calls_equal_the_layer_calls_they_stand_for(attn_fp8):
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    H, N, d = 2, cfg.N, cfg.d
    params = svg2.LayerParams(nQ=cfg.nQ, nK=cfg.nK, iters=cfg.iters, top_p=0.9, scale=float(np.float32(cfg.scale)),
                              attn_fp8=attn_fp8)
    steps, layers = 4, 2
    drv = svg2.Driver(1, H, N, d, num_steps=steps, num_layers=layers, dense_steps=1, warm_iters=2, params=params)
    rng = np.random.default_rng(3)
    ws = svg2.workspace(1, H, N, d, cfg.nQ, cfg.nK)
    dws = svg2.dense_workspace(1, H, N, d)
    ref_c = {l: (torch.zeros(1, H, cfg.nQ, d, device="cuda"), torch.zeros(1, H, cfg.nK, d, device="cuda"))
             for l in range(layers)}
    kinds = []
    for step in range(steps):
        for l in range(layers):
            Q, K, V = (bf16_dev(I.round_to_bf16(rng.standard_normal((1, H, N, d), dtype=np.float32))) for _ in range(3))
            uq = to_dev(rng.random((1, H, cfg.nQ)))
            uk = to_dev(rng.random((1, H, cfg.nK)))
            kind = drv.plan(step, l)
            kinds.append(kind)
            O = torch.empty_like(Q)
            drv.layer(step, l, Q, K, V, O, uq, uk)
            R = torch.empty_like(Q)
            if kind == svg2.SVG2_STEP_DENSE:
                svg2.svg2_dense_attn(Q, K, V, params.scale, R, dws)
            else:
                p = svg2.LayerParams(**{**params.__dict__})
                if kind == svg2.SVG2_STEP_COLD:
                    p.init = svg2.SVG2_INIT_KMEANSPP
                else:
                    p.init, p.iters = svg2.SVG2_INIT_GIVEN, 2
                svg2.svg2_layer(Q, K, V, p, ref_c[l][0], ref_c[l][1], R, ws, uq=uq, uk=uk)
            torch.cuda.synchronize()
            svg2.raise_on_device_error(drv.ws)
            assert torch.equal(O, R), (step, l, kind)
            if kind != svg2.SVG2_STEP_DENSE:
                per = H * (cfg.nQ + cfg.nK) * d
                cache = drv.cache[l * per:(l + 1) * per]
                assert torch.equal(cache[:H * cfg.nQ * d], ref_c[l][0].flatten())
                assert torch.equal(cache[H * cfg.nQ * d:], ref_c[l][1].flatten())
    D, C, W = svg2.SVG2_STEP_DENSE, svg2.SVG2_STEP_COLD, svg2.SVG2_STEP_WARM
    assert kinds == [D, D, C, C, W, W, W, W]
    drv.reset()
    assert drv.plan(1, 0) == C
    drv.close()
