"""The C-ABI boundary on the host (no GPU): the library loads, exports every entry point that
include/svg2.h declares, and rejects bad arguments with the documented status codes before it
touches the GPU."""
import ctypes
import os
import re

import pytest

from sparse_attention_video_head_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svg2.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module")
def L():
    B.build()
    from sparse_attention_video_head_b200 import svg2
    return svg2.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SVG2_API\s+(?:const\s+)?\w+\*?\s+\**(svg2_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("svg2_kmeans", "svg2_select", "svg2_select_from_weights", "svg2_sort", "svg2_gather", "svg2_permute",
              "svg2_sparse_attn", "svg2_unpermute", "svg2_layer", "svg2_workspace_size", "svg2_check_status"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_library_has_no_driver_or_torch_link_dependency():
    B.build()
    import subprocess
    out = subprocess.run(["ldd", B.LIB], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out and "not found" not in out


def test_status_strings(L):
    from sparse_attention_video_head_b200 import svg2
    assert svg2.status_string(0) == "SVG2_OK"
    for c in range(1, 7):
        assert svg2.status_string(c).startswith("SVG2_ERR")


def test_workspace_size_is_monotone_and_validates(L):
    from sparse_attention_video_head_b200 import svg2
    small = svg2.svg2_workspace_size(1, 8, 12480, 128, 64, 256)
    big = svg2.svg2_workspace_size(1, 40, 75600, 128, 100, 500)
    assert 0 < small < big
    # Wan-720p: Q, K, V permuted copies plus the un-fused output copy dominate (4 x 774 MB)
    assert big > 4 * 40 * 75600 * 128 * 2
    out = ctypes.c_size_t(0)
    assert L.svg2_workspace_size(1, 1, 100, 96, 4, 4, ctypes.byref(out)) == UNSUPPORTED
    assert L.svg2_workspace_size(1, 1, 100, 128, 0, 4, ctypes.byref(out)) == INVALID
    assert L.svg2_workspace_size(1, 1, 100, 128, 101, 4, ctypes.byref(out)) == INVALID
    assert L.svg2_workspace_size(1, 1, 5000, 128, 2000, 4, ctypes.byref(out)) == UNSUPPORTED
    assert L.svg2_workspace_size(0, 1, 100, 128, 4, 4, ctypes.byref(out)) == INVALID
    assert L.svg2_workspace_size(1, 1, 100, 128, 4, 4, None) == INVALID
    # B*H*N must stay below 2^31 rows; B*H at most 65535 (a grid dimension in several kernels)
    assert L.svg2_workspace_size(1, 256, 1 << 23, 128, 4, 4, ctypes.byref(out)) == UNSUPPORTED
    assert L.svg2_workspace_size(2, 128, (1 << 23) - 1, 128, 4, 4, ctypes.byref(out)) == OK
    assert L.svg2_workspace_size(1, (1 << 20) + 1, 4, 128, 4, 4, ctypes.byref(out)) == UNSUPPORTED
    assert L.svg2_workspace_size(1, 65536, 4, 128, 4, 4, ctypes.byref(out)) == UNSUPPORTED
    assert L.svg2_workspace_size(3, 21845, 4, 128, 4, 4, ctypes.byref(out)) == OK


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation first


def test_kmeans_rejects_bad_arguments(L):
    P = None
    args = lambda **kw: dict(dict(X=FAKE, dt=0, B=1, H=1, N=100, d=128, k=4, it=1, init=0, u=P, st=0, C=FAKE,
                                  lab=FAKE, cnt=FAKE, perm=P, off=P, ws=FAKE, wsb=1 << 30), **kw)
    def call(**kw):
        a = args(**kw)
        return L.svg2_kmeans(a["X"], a["dt"], a["B"], a["H"], a["N"], a["d"], a["k"], a["it"], a["init"], a["u"],
                             a["st"], a["C"], a["lab"], a["cnt"], a["perm"], a["off"], a["ws"], a["wsb"], None)
    assert call(X=None) == INVALID
    assert call(dt=7) == INVALID
    assert call(k=0) == INVALID
    assert call(k=101) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(it=0) == INVALID
    assert call(init=5) == INVALID
    assert call(init=1, u=None) == INVALID           # k-means++ needs its uniforms
    assert call(st=-1) == INVALID
    assert call(init=1, u=FAKE, N=100, k=40, st=30) == INVALID   # 34 candidates for 40 seeds
    assert call(ws=None) == WORKSPACE
    assert call(wsb=16) == WORKSPACE
    assert call(ws=ctypes.c_void_p(0x10010)) == WORKSPACE   # not 256-byte aligned


def test_kmeanspp_rejects_bad_arguments(L):
    def call(X=FAKE, dt=0, B=1, H=1, N=100, d=128, k=4, u=FAKE, st=0, C=FAKE, ws=FAKE, wsb=1 << 30):
        return L.svg2_kmeanspp(X, dt, B, H, N, d, k, u, st, C, ws, wsb, None)
    assert call(X=None) == INVALID
    assert call(u=None) == INVALID
    assert call(C=None) == INVALID
    assert call(dt=7) == INVALID
    assert call(k=0) == INVALID
    assert call(k=101) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(st=-1) == INVALID
    assert call(N=100, k=40, st=30) == INVALID   # 34 candidates for 40 seeds
    assert call(ws=None) == WORKSPACE
    assert call(wsb=16) == WORKSPACE


def test_layer_host_rejects_bad_arguments(L):
    from sparse_attention_video_head_b200 import svg2
    prm = svg2.SvgParams(4, 8, 2, 1, 0.9, 0.1, 0, 1)
    def call(Qh=FAKE, Oh=FAKE, Qd=FAKE, B=1, H=2, N=100, d=128, hpg=1, p=ctypes.byref(prm), cq=FAKE, u=FAKE, ws=FAKE,
             wsb=1 << 30):
        return L.svg2_layer_host(Qh, FAKE, FAKE, Oh, Qd, FAKE, FAKE, FAKE, 0, B, H, N, d, p, u, u, cq, FAKE, hpg, ws,
                                 wsb, None, None)
    assert call(Qh=None) == INVALID
    assert call(Oh=None) == INVALID
    assert call(Qd=None) == INVALID
    assert call(hpg=-1) == INVALID
    assert call(p=None) == INVALID
    assert call(cq=None) == INVALID
    assert call(u=None) == INVALID          # k-means++ needs its uniforms
    assert call(d=96) == UNSUPPORTED
    assert call(wsb=16) == WORKSPACE        # checked for every head group before any copy


def test_select_and_topp_reject_bad_arguments(L):
    F = ctypes.c_float
    assert L.svg2_select(FAKE, FAKE, FAKE, 1, 1, 4, 8, 128, F(0.0), F(0.1), None, FAKE, FAKE, FAKE, None, FAKE,
                         1 << 20, None) == INVALID
    assert L.svg2_select(FAKE, FAKE, FAKE, 1, 1, 4, 2000, 128, F(0.9), F(0.1), None, FAKE, FAKE, FAKE, None, FAKE,
                         1 << 20, None) == UNSUPPORTED
    assert L.svg2_select(FAKE, FAKE, None, 1, 1, 4, 8, 128, F(0.9), F(0.1), None, FAKE, FAKE, FAKE, None, FAKE,
                         1 << 20, None) == INVALID
    assert L.svg2_select_from_weights(None, FAKE, 1, 1, 4, 8, F(0.9), FAKE, FAKE, FAKE, None, FAKE, 1 << 20,
                                      None) == INVALID
    assert L.svg2_select_from_weights(FAKE, FAKE, 1, 1, 4, 8, F(float("nan")), FAKE, FAKE, FAKE, None, FAKE, 1 << 20,
                                      None) == INVALID
    assert L.svg2_select_from_weights(FAKE, FAKE, 1, 1, 4, 8, F(0.9), FAKE, FAKE, FAKE, None, None, 0,
                                      None) == WORKSPACE


def test_permutation_calls_reject_bad_arguments(L):
    assert L.svg2_sort(None, 1, 1, 10, 4, FAKE, FAKE, None, FAKE, 1 << 20, None) == INVALID
    assert L.svg2_sort(FAKE, 1, 1, 10, 0, FAKE, FAKE, None, FAKE, 1 << 20, None) == INVALID
    assert L.svg2_sort(FAKE, 1, 1, 10, 4096, FAKE, FAKE, None, FAKE, 1 << 20, None) == UNSUPPORTED
    assert L.svg2_sort(FAKE, 1, 1, 10, 4, FAKE, FAKE, None, FAKE, 8, None) == WORKSPACE
    assert L.svg2_gather(FAKE, 3, FAKE, 1, 1, 10, 128, FAKE, None) == INVALID
    assert L.svg2_gather(FAKE, 0, FAKE, 1, 1, 10, 32, FAKE, None) == UNSUPPORTED
    assert L.svg2_gather(ctypes.c_void_p(0x10002), 0, FAKE, 1, 1, 10, 128, FAKE, None) == INVALID
    assert L.svg2_unpermute(FAKE, None, 1, 1, 10, 128, FAKE, None) == INVALID


def test_attention_and_layer_reject_bad_arguments(L):
    from sparse_attention_video_head_b200.svg2 import SvgParams
    F = ctypes.c_float
    assert L.svg2_sparse_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1000, 96, 4, 4, F(0.1), None, FAKE,
                              FAKE, 1 << 30, None) == UNSUPPORTED   # the attention kernel is built for d = 64, 128
    assert L.svg2_sparse_attn(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1, 1, 1000, 128, 4, 4, F(0.1), None, FAKE,
                              FAKE, 1 << 30, None) == INVALID
    assert L.svg2_sparse_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1000, 128, 4, 4, F(0.1), None, FAKE,
                              FAKE, 64, None) == WORKSPACE
    p = SvgParams(4, 8, 2, 1, 0.9, 0.1, 0, 1)
    args = [FAKE, FAKE, FAKE, 0, 1, 1, 1000, 128, ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 34,
            None]
    bad = SvgParams(4, 8, 2, 1, 0.9, 0.1, 0, 1)
    bad.top_p = -1.0
    assert L.svg2_layer(*args[:8], ctypes.byref(bad), *args[9:]) == INVALID
    bad = SvgParams(4, 8, 0, 1, 0.9, 0.1, 0, 1)
    assert L.svg2_layer(*args[:8], ctypes.byref(bad), *args[9:]) == INVALID
    assert L.svg2_layer(*args[:9], None, *args[10:]) == INVALID          # k-means++ without uniforms
    assert L.svg2_layer(*args[:16], 1024, None) == WORKSPACE
    assert L.svg2_layer(*args[:8], None, *args[9:]) == INVALID


def test_dense_attn_rejects_bad_arguments(L):
    from sparse_attention_video_head_b200 import svg2
    out = ctypes.c_size_t(0)
    assert L.svg2_dense_attn_workspace_size(1, 2, 1000, 128, ctypes.byref(out)) == OK and out.value > 0
    assert L.svg2_dense_attn_workspace_size(1, 2, 1000, 96, ctypes.byref(out)) == UNSUPPORTED
    assert L.svg2_dense_attn_workspace_size(1, 2, 1000, 128, None) == INVALID
    # much smaller than the layer's workspace: no permuted copies, one cluster
    assert svg2.svg2_dense_attn_workspace_size(1, 40, 75600, 128) < svg2.svg2_workspace_size(1, 40, 75600, 128, 1, 1) // 100
    ws_ok = 1 << 30
    call = lambda **kw: L.svg2_dense_attn(*[dict(dict(Q=FAKE, K=FAKE, V=FAKE, B=1, H=2, N=1000, d=128, s=0.08, O=FAKE,
                                                      ws=FAKE, wsb=ws_ok, st=None), **kw)[n]
                                            for n in ("Q", "K", "V", "B", "H", "N", "d", "s", "O", "ws", "wsb", "st")])
    assert call(Q=None) == INVALID
    assert call(O=None) == INVALID
    assert call(V=ctypes.c_void_p(0x10008)) == INVALID            # not 16-byte aligned
    assert call(s=float("nan")) == INVALID
    assert call(s=float("inf")) == INVALID
    assert call(d=96) == UNSUPPORTED
    assert call(N=0) == INVALID
    assert call(ws=None) == WORKSPACE
    assert call(ws=ctypes.c_void_p(0x10010)) == WORKSPACE        # not 256-byte aligned
    assert call(wsb=16) == WORKSPACE


def test_set_wait_budget_rejects_a_missing_or_misaligned_workspace(L):
    assert L.svg2_set_wait_budget(None, 100, None) == INVALID
    assert L.svg2_set_wait_budget(ctypes.c_void_p(0x10010), 100, None) == INVALID  # not 256-byte aligned


def test_fp8_calls_reject_bad_arguments(L):
    from sparse_attention_video_head_b200.svg2 import SvgParams
    F = ctypes.c_float
    q = lambda X=FAKE, dt=0, perm=None, d=128, X8=FAKE, sc=FAKE: L.svg2_quantize_e4m3(X, dt, perm, 1, 2, 100, d, X8, sc, None)
    assert q(X=None) == INVALID
    assert q(X8=None) == INVALID
    assert q(sc=None) == INVALID
    assert q(dt=7) == INVALID
    assert q(d=96) == UNSUPPORTED
    assert q(X8=ctypes.c_void_p(0x10008)) == INVALID          # not 16-byte aligned

    def a(d=128, sq=FAKE, V8=FAKE, s=0.1, wsb=1 << 30):
        return L.svg2_sparse_attn_fp8(FAKE, FAKE, V8, sq, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1000, d, 4, 4,
                                      F(s), None, FAKE, FAKE, wsb, None)
    assert a(d=64) == UNSUPPORTED                              # the FP8 kernel is built for d = 128
    assert a(d=96) == UNSUPPORTED
    assert a(sq=None) == INVALID
    assert a(V8=None) == INVALID
    assert a(s=float("nan")) == INVALID
    assert a(wsb=64) == WORKSPACE

    args = [FAKE, FAKE, FAKE, 0, 1, 1, 1000, 128, None, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 34, None]
    bad = SvgParams(4, 8, 2, 1, 0.9, 0.1, 0, 1, 2)           # attn_fp8 is 0 or 1
    assert L.svg2_layer(*args[:8], ctypes.byref(bad), *args[9:]) == INVALID
    fp8 = SvgParams(4, 8, 2, 1, 0.9, 0.1, 0, 1, 1)
    assert L.svg2_layer(*args[:7], 64, ctypes.byref(fp8), *args[9:]) == UNSUPPORTED



def test_noalloc_checks_sizes_before_any_cuda_call(L):
    F = ctypes.c_float

    def call(B=1, H=1, N=1000, d=128, nQ=4, nK=4, Q=FAKE):
        return L.svg2_sparse_attn_noalloc(Q, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, B, H, N, d, nQ, nK, F(0.1), None,
                                          FAKE, None, None)
    assert call(H=65536) == UNSUPPORTED        # the (b,h) planes are a grid dimension of their own
    assert call(B=2, H=32768) == UNSUPPORTED
    assert call(d=96) == UNSUPPORTED
    assert call(nQ=2000, N=5000) == UNSUPPORTED
    assert call(B=0) == INVALID
    assert call(nQ=1001) == INVALID            # more clusters than tokens
    assert call(Q=None) == INVALID
    assert call(Q=ctypes.c_void_p(0x10008)) == INVALID
