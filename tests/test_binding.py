"""The Python binding's argument checks, on the host (no GPU).

The library receives plain pointers, so it cannot see how large a caller's buffer is: a tensor
that is too small, or of the wrong element type, would be read or written past its end on the
device.  The binding therefore checks every tensor against include/svg2.h (dtype and element
count for the sizes of the call) before it takes the pointer.  Here the library and the pointer
step are replaced by recorders, so each wrapper runs on CPU tensors: correct arguments reach the
library with the sizes the header defines, and each undersized or mistyped buffer is refused
before any call.
"""
import ctypes

import pytest
import torch

from sparse_attention_video_head_b200 import svg2

i32, f32, f64, u8, bf16 = torch.int32, torch.float32, torch.float64, torch.uint8, torch.bfloat16


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append((name, args))
            return 0
        return call


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(svg2, "lib", lambda: r)
    monkeypatch.setattr(svg2, "_p", lambda t: None if t is None else ctypes.c_void_p(t.data_ptr() or 16))
    monkeypatch.setattr(svg2, "_stream", lambda stream=None: None)
    return r


def _t(*shape, dtype):
    return torch.zeros(*shape, dtype=dtype)


def _each_bad(args, keys):
    """Variants of `args` with one tensor one element short, then with the wrong dtype."""
    for k in keys:
        t = args[k]
        short = torch.zeros(t.numel() - 1, dtype=t.dtype) if t.numel() > 0 else None
        yield k, "short", {**args, k: short}
        wrong = torch.zeros(t.shape, dtype=torch.int64 if t.dtype != torch.int64 else torch.int32)
        yield k, "dtype", {**args, k: wrong}


def _expect_refused(rec, fn, args, keys):
    for k, how, bad in _each_bad(args, keys):
        n = len(rec.calls)
        with pytest.raises(ValueError):
            fn(**bad)
        assert len(rec.calls) == n, (k, how)


def test_kmeans_and_seeding(rec):
    B, H, N, d, k = 1, 2, 300, 128, 7
    args = dict(X=_t(B, H, N, d, dtype=bf16), k=k, iters=3, init=svg2.SVG2_INIT_KMEANSPP,
                centroids=_t(B, H, k, d, dtype=f32), labels=_t(B, H, N, dtype=i32), counts=_t(B, H, k, dtype=i32),
                ws=_t(1024, dtype=u8), u=_t(B, H, k, dtype=f64), perm=_t(B, H, N, dtype=i32),
                offsets=_t(B, H, k + 1, dtype=i32))
    svg2.svg2_kmeans(**args)
    name, a = rec.calls[-1]
    assert name == "svg2_kmeans" and a[1:9] == (svg2.SVG2_BF16, B, H, N, d, k, 3, svg2.SVG2_INIT_KMEANSPP)
    assert a[17] == 1024                                    # workspace bytes
    _expect_refused(rec, svg2.svg2_kmeans, args, ["centroids", "labels", "counts", "u", "perm", "offsets"])
    # a warm start ignores u; optional outputs may be left out
    svg2.svg2_kmeans(**{**args, "init": svg2.SVG2_INIT_GIVEN, "u": None, "perm": None, "offsets": None})
    with pytest.raises(ValueError):
        svg2.svg2_kmeans(**{**args, "u": None})           # a cold start needs the uniforms
    with pytest.raises(ValueError):
        svg2.svg2_kmeans(**{**args, "X": _t(B, H, N, d, dtype=torch.float16)})
    # a float32 workspace is counted in bytes
    svg2.svg2_kmeans(**{**args, "ws": _t(256, dtype=f32)})
    assert rec.calls[-1][1][17] == 1024
    sargs = dict(X=args["X"], k=k, u=args["u"], centroids=args["centroids"], ws=args["ws"])
    svg2.svg2_kmeanspp(**sargs)
    assert rec.calls[-1][0] == "svg2_kmeanspp"
    _expect_refused(rec, svg2.svg2_kmeanspp, sargs, ["u", "centroids"])


def test_select_calls(rec):
    B, H, nQ, nK, d = 1, 3, 5, 9, 128
    args = dict(cq=_t(B, H, nQ, d, dtype=f32), ck=_t(B, H, nK, d, dtype=f32), count_k=_t(B, H, nK, dtype=i32),
                top_p=0.9, scale=0.1, mask=_t(B, H, nQ, nK, dtype=u8), sel_count=_t(B, H, nQ, dtype=i32),
                sel_idx=_t(B, H, nQ, nK, dtype=i32), ws=_t(256, dtype=u8), weights=_t(B, H, nQ, nK, dtype=f32),
                stream_len=_t(B, H, nQ, dtype=i32))
    svg2.svg2_select(**args)
    name, a = rec.calls[-1]
    assert name == "svg2_select" and a[3:8] == (B, H, nQ, nK, d)
    _expect_refused(rec, svg2.svg2_select, args, ["count_k", "mask", "sel_count", "sel_idx", "weights", "stream_len"])
    svg2.svg2_select(**{**args, "weights": None, "stream_len": None})
    wargs = dict(weights=args["weights"], count_k=args["count_k"], top_p=0.5, mask=args["mask"],
                 sel_count=args["sel_count"], sel_idx=args["sel_idx"], ws=args["ws"], stream_len=args["stream_len"])
    svg2.svg2_select_from_weights(**wargs)
    assert rec.calls[-1][1][2:6] == (B, H, nQ, nK)
    _expect_refused(rec, svg2.svg2_select_from_weights, wargs, ["count_k", "mask", "sel_count", "sel_idx",
                                                                 "stream_len"])


def test_permutation_calls(rec):
    B, H, N, d, k = 2, 2, 100, 128, 6
    sargs = dict(labels=_t(B, H, N, dtype=i32), k=k, perm=_t(B, H, N, dtype=i32), offsets=_t(B, H, k + 1, dtype=i32),
                 counts=_t(B, H, k, dtype=i32), ws=_t(256, dtype=u8))
    svg2.svg2_sort(**sargs)
    assert rec.calls[-1][1][1:5] == (B, H, N, k)
    _expect_refused(rec, svg2.svg2_sort, sargs, ["perm", "offsets", "counts"])
    gargs = dict(X=_t(B, H, N, d, dtype=f32), perm=_t(B, H, N, dtype=i32), Xp=_t(B, H, N, d, dtype=bf16))
    svg2.svg2_gather(**gargs)
    assert rec.calls[-1][1][1] == svg2.SVG2_F32
    _expect_refused(rec, svg2.svg2_gather, gargs, ["perm", "Xp"])
    pargs = dict(X=gargs["X"], labels=sargs["labels"], k=k, Xp=gargs["Xp"], perm=sargs["perm"],
                 offsets=sargs["offsets"], counts=None, ws=sargs["ws"])
    svg2.svg2_permute(**pargs)
    _expect_refused(rec, svg2.svg2_permute, pargs, ["labels", "Xp", "perm", "offsets"])
    uargs = dict(Op=gargs["Xp"], perm=sargs["perm"], O=_t(B, H, N, d, dtype=bf16))
    svg2.svg2_unpermute(**uargs)
    _expect_refused(rec, svg2.svg2_unpermute, uargs, ["perm", "O"])


def test_attention_calls(rec):
    B, H, N, d, nQ, nK = 1, 2, 500, 128, 4, 6
    args = dict(Qp=_t(B, H, N, d, dtype=bf16), Kp=_t(B, H, N, d, dtype=bf16), Vp=_t(B, H, N, d, dtype=bf16),
                q_off=_t(B, H, nQ + 1, dtype=i32), k_off=_t(B, H, nK + 1, dtype=i32), sel_count=_t(B, H, nQ, dtype=i32),
                sel_idx=_t(B, H, nQ, nK, dtype=i32), scale=0.1, O=_t(B, H, N, d, dtype=bf16),
                ws=_t(512, dtype=u8), perm_q=_t(B, H, N, dtype=i32))
    svg2.svg2_sparse_attn(**args)
    name, a = rec.calls[-1]
    assert name == "svg2_sparse_attn" and a[7:13] == (B, H, N, d, nQ, nK)
    # perm_q then O follow the scale, as the header orders them
    assert a[14].value == args["perm_q"].data_ptr() and a[15].value == args["O"].data_ptr() and a[17] == 512
    _expect_refused(rec, svg2.svg2_sparse_attn, args, ["Kp", "Vp", "sel_count", "sel_idx", "O", "perm_q"])
    nargs = {key: v for key, v in args.items() if key != "ws"}
    status = _t(4, dtype=i32)
    svg2.svg2_sparse_attn_noalloc(**nargs, device_status=status)
    a = rec.calls[-1][1]
    assert a[14].value == args["perm_q"].data_ptr() and a[15].value == args["O"].data_ptr()
    assert a[16].value == status.data_ptr()
    with pytest.raises(ValueError):
        svg2.svg2_sparse_attn_noalloc(**nargs, device_status=_t(3, dtype=i32))
    _expect_refused(rec, svg2.svg2_sparse_attn_noalloc, nargs, ["Kp", "Vp", "sel_count", "sel_idx", "O"])
    dargs = dict(Q=args["Qp"], K=args["Kp"], V=args["Vp"], scale=0.1, O=args["O"], ws=args["ws"])
    svg2.svg2_dense_attn(**dargs)
    assert rec.calls[-1][1][3:7] == (B, H, N, d)
    _expect_refused(rec, svg2.svg2_dense_attn, dargs, ["K", "V", "O"])


def test_layer_calls(rec):
    B, H, N, d, nQ, nK = 1, 2, 400, 128, 5, 11
    prm = svg2.LayerParams(nQ, nK, 2)
    args = dict(Q=_t(B, H, N, d, dtype=bf16), K=_t(B, H, N, d, dtype=bf16), V=_t(B, H, N, d, dtype=bf16), params=prm,
                cq=_t(B, H, nQ, d, dtype=f32), ck=_t(B, H, nK, d, dtype=f32), O=_t(B, H, N, d, dtype=bf16),
                ws=_t(2048, dtype=u8), uq=_t(B, H, nQ, dtype=f64), uk=_t(B, H, nK, dtype=f64))
    outs = svg2.layer_output_buffers(B, H, N, nQ, nK, device="cpu")
    svg2.svg2_layer(**args, outs=outs)
    name, a = rec.calls[-1]
    assert name == "svg2_layer" and a[3:8] == (svg2.SVG2_BF16, B, H, N, d) and a[16] == 2048
    assert a[13].value == args["O"].data_ptr()
    c_outs = a[14]._obj
    assert c_outs.sel_idx == outs["sel_idx"].data_ptr() and c_outs.mask == outs["mask"].data_ptr()
    _expect_refused(rec, svg2.svg2_layer, args, ["K", "V", "cq", "ck", "O", "uq", "uk"])
    for key in outs:
        bad = dict(outs)
        bad[key] = torch.zeros(outs[key].numel() - 1, dtype=outs[key].dtype)
        with pytest.raises(ValueError):
            svg2.svg2_layer(**args, outs=bad)
    # a warm start needs no uniforms; K and V must match Q's dtype
    svg2.svg2_layer(**{**args, "params": svg2.LayerParams(nQ, nK, 2, svg2.SVG2_INIT_GIVEN), "uq": None, "uk": None})
    with pytest.raises(ValueError):
        svg2.svg2_layer(**{**args, "K": _t(B, H, N, d, dtype=f32)})
    hargs = dict(Qh=args["Q"], Kh=args["K"], Vh=args["V"], Oh=_t(B, H, N, d, dtype=bf16),
                 Q=_t(B, H, N, d, dtype=bf16), K=_t(B, H, N, d, dtype=bf16), V=_t(B, H, N, d, dtype=bf16),
                 O=_t(B, H, N, d, dtype=bf16), params=prm, cq=args["cq"], ck=args["ck"], ws=args["ws"],
                 uq=args["uq"], uk=args["uk"])
    svg2.svg2_layer_host(**hargs, heads_per_group=1)
    name, a = rec.calls[-1]
    assert name == "svg2_layer_host" and a[8:13] == (svg2.SVG2_BF16, B, H, N, d) and a[18] == 1
    _expect_refused(rec, svg2.svg2_layer_host, hargs, ["Kh", "Vh", "Oh", "Q", "K", "V", "O", "cq", "ck", "uq", "uk"])


def test_layer_output_sizes_cover_every_field():
    names = [n for n, _ in svg2.SvgLayerOutputs._fields_]
    sizes = svg2._layer_out_sizes(100, 3, 5)
    assert sorted(sizes) == sorted(names)
    bufs = svg2.layer_output_buffers(1, 1, 100, 3, 5, device="cpu")
    for n in names:
        assert bufs[n].dtype in sizes[n][0] and bufs[n].numel() == sizes[n][1], n


def test_driver_layer_and_selftest(rec):
    B, H, N, d, nQ, nK = 1, 2, 300, 128, 4, 8
    drv = svg2.Driver(B, H, N, d, num_steps=3, num_layers=1, dense_steps=1, warm_iters=2,
                      params=svg2.LayerParams(nQ, nK, 2), allocate=False)
    args = dict(step=1, layer=0, Q=_t(B, H, N, d, dtype=bf16), K=_t(B, H, N, d, dtype=bf16),
                V=_t(B, H, N, d, dtype=bf16), O=_t(B, H, N, d, dtype=bf16), uq=_t(B, H, nQ, dtype=f64),
                uk=_t(B, H, nK, dtype=f64))
    with pytest.raises(ValueError):
        drv.layer(**args)                                   # no workspace was allocated
    drv.ws = _t(4096, dtype=u8)
    drv.layer(**args)
    name, a = rec.calls[-1]
    assert name == "svg2_driver_layer" and a[1:3] == (1, 0) and a[10] == 4096
    drv.layer(**{**args, "uq": None, "uk": None})          # a dense or warm step needs no uniforms
    _expect_refused(rec, drv.layer, args, ["Q", "K", "V", "O", "uq", "uk"])
    A, V = _t(128, 128, dtype=bf16), _t(128, 128, dtype=bf16)
    svg2.svg2_selftest_mma(A, _t(64, 128, dtype=bf16), V, _t(256, dtype=u8))
    assert rec.calls[-1][1][2] == 64
    with pytest.raises(ValueError):
        svg2.svg2_selftest_mma(A, _t(64, 127, dtype=bf16), V, _t(256, dtype=u8))
