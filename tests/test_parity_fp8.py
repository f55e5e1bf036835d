"""The FP8 (E4M3) attention variant and its per-head quantiser against the oracle (the project's roadmap
item "Support FP8 attention", GitHub README, Open-source Plan).  The oracle defines the variant as
attention over the dequantised values E4M3(code) * scale of each (b,h) plane.

Tolerances:
* quantiser: codes and scales bit-exact (integer work from the same float32 steps);
* exact-P case: integer logits, so every P the kernel rounds to E4M3 is a power of two inside E4M3's
  range and stays exact; what is left is float32 accumulation, the cubic 2^x's 7.5e-5 on the row sum
  and the bf16 output: every element within one bf16 step (2^-8 relative) of the oracle, relative
  L2 at most 2e-3.  A transposed byte of the packed P, a wrong V step or a dropped tile fails it;
* random inputs: relative L2 per head at most 5e-2.  Rounding P to E4M3 alone gives 2.4-3.0 % on
  N(0,1) data in a float64 simulation (key streams of 300 to 30000 keys, running maxima up to 2^8
  stale), since P's 3 mantissa bits carry a relative error of up to 2^-4 per key.
"""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, pool_layer_inputs, require_gpu, to_dev
from tests.test_parity_attn import SCALE, _case, _ell, _growth_case, _late_growth_rows, rel_l2

EXACT_REL_L2, REL_L2 = 2e-3, 5e-2


def _quantize_oracle(oracle, X):
    """Per-plane codes and scales of X [1, H, N, d] float32."""
    B, H, N, d = X.shape
    codes, scale = oracle.quantize_e4m3(X.reshape(B * H, N * d))
    return codes.reshape(X.shape), scale.reshape(B, H)


def _run_fp8(svg2, c, scale, perm_q=None):
    """c: Q8, K8, V8 uint8 [1,H,N,d]; sq, sk, sv float32 [1,H]; q_off, k_off, mask as _case."""
    B, H, N, d = c["Q8"].shape
    nQ, nK = c["mask"].shape[-2:]
    sel_count, sel_idx = _ell(c["mask"])
    O = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    ws = svg2.workspace(B, H, N, d, nQ, nK)
    svg2.svg2_sparse_attn_fp8(to_dev(c["Q8"]), to_dev(c["K8"]), to_dev(c["V8"]), to_dev(c["sq"]), to_dev(c["sk"]),
                              to_dev(c["sv"]), to_dev(c["q_off"]), to_dev(c["k_off"]), to_dev(sel_count),
                              to_dev(sel_idx), scale, O, ws, perm_q=None if perm_q is None else to_dev(perm_q))
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    return host(O)


def _reference(oracle, c, scale, h, rows=None):
    return oracle.sparse_attention_fp8_rows(c["Q8"][0, h], c["K8"][0, h], c["V8"][0, h], c["sq"][0, h], c["sk"][0, h],
                                            c["sv"][0, h], c["q_off"][0, h], c["k_off"][0, h], c["mask"][0, h],
                                            scale, rows)


def _quantized_case(svg2, oracle, c):
    """Quantise _case's bf16 Qp, Kp, Vp on the GPU; the codes and scales must equal the oracle's."""
    out = dict(c)
    for name, key in (("Qp", "Q"), ("Kp", "K"), ("Vp", "V")):
        X = c[name]
        codes = torch.empty(X.shape, dtype=torch.uint8, device="cuda")
        scale = torch.empty(X.shape[:2], dtype=torch.float32, device="cuda")
        svg2.svg2_quantize_e4m3(bf16_dev(X), codes, scale)
        torch.cuda.synchronize()
        ref_codes, ref_scale = _quantize_oracle(oracle, X)
        assert np.array_equal(host(codes), ref_codes), name
        assert np.array_equal(host(scale), ref_scale), name
        out[key + "8"], out["s" + key.lower()] = ref_codes, ref_scale
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("with_perm", [False, True])
def test_quantize_is_bit_exact(oracle, dtype, with_perm):
    svg2 = require_gpu()
    rng = np.random.default_rng(50)
    H, N, d = 4, 1000, 128
    X = (rng.standard_normal((1, H, N, d)) * np.array([0.01, 1.0, 700.0, 0.0])[None, :, None, None]).astype(np.float32)
    if dtype == "bf16":
        X = I.round_to_bf16(X)
    X[0, 1, 5, 7] = np.nan                    # ignored by the maximum, quantised to the NaN code
    X[0, 0, 9, :] = -0.0                       # negative zeros keep their sign
    Xd = bf16_dev(X) if dtype == "bf16" else to_dev(X)
    perm = np.stack([rng.permutation(N) for _ in range(H)]).astype(np.int32)[None] if with_perm else None
    codes = torch.empty(X.shape, dtype=torch.uint8, device="cuda")
    scale = torch.empty((1, H), dtype=torch.float32, device="cuda")
    svg2.svg2_quantize_e4m3(Xd, codes, scale, perm=None if perm is None else to_dev(perm))
    torch.cuda.synchronize()
    ref_codes, ref_scale = _quantize_oracle(oracle, X)
    if perm is not None:
        ref_codes = np.stack([ref_codes[0, h][perm[0, h]] for h in range(H)])[None]
    np.testing.assert_array_equal(host(scale), ref_scale)
    got = host(codes)
    assert np.array_equal(got, ref_codes), int((got != ref_codes).sum())
    assert ref_scale[0, 3] == 1.0 and not (ref_codes[0, 3] & 0x7F).any()   # an all-zero plane: +-0 codes, scale 1


def _exact_p_case(seed, N, nQ, nK, density, H):
    """Integer logits in [-4, 4]: Q rows hold four entries of +-1, K rows six, the rest 0 (exact E4M3
    codes 0x38, 0xB8, 0x00), scales 1, and softmax scale ln 2, so p = 2^(s - m) with s - m an integer
    in [-8, 8]: every P is a power of two that E4M3 holds exactly.  V is any E4M3 plane."""
    rng = np.random.default_rng(seed)
    c = _case(seed, N, nQ, nK, density, H)
    d = 128

    def pm1(n_nonzero):
        codes = np.zeros((1, H, N, d), np.uint8)
        for h in range(H):
            for r in range(N):
                cols = rng.choice(d, n_nonzero, replace=False)
                codes[0, h, r, cols] = np.where(rng.random(n_nonzero) < 0.5, 0x38, 0xB8)
        return codes

    c["Q8"], c["K8"] = pm1(4), pm1(6)
    c["V8"] = rng.integers(0, 0x7F, (1, H, N, d)).astype(np.uint8) | (rng.integers(0, 2, (1, H, N, d)) << 7).astype(np.uint8)
    c["V8"][(c["V8"] & 0x7F) >= 0x78] = 0x30   # keep |v| <= 240 (no 0x7F NaN codes)
    c["sq"] = np.ones((1, H), np.float32)
    c["sk"] = np.ones((1, H), np.float32)
    c["sv"] = np.full((1, H), 0.5, np.float32)
    return c


@pytest.mark.gpu
@pytest.mark.parametrize("seed,N,nQ,nK,density,H", [(60, 3000, 20, 40, 0.4, 2), (61, 2000, 25, 8, 1.0, 1)])
def test_fp8_attention_exact_p(oracle, seed, N, nQ, nK, density, H):
    svg2 = require_gpu()
    c = _exact_p_case(seed, N, nQ, nK, density, H)
    scale = float(np.float32(np.log(2.0)))
    O = _run_fp8(svg2, c, scale)
    for h in range(H):
        ref = _reference(oracle, c, scale, h)
        err = np.abs(O[0, h] - ref)
        # half a bf16 step is up to 2^-8 of the value; 2e-4 more covers the row sum's cubic 2^x values
        # (7.5e-5) and float32 accumulation
        bound = (2.0 ** -8 + 2e-4) * np.abs(ref) + 1e-6 * np.abs(ref).max()
        rel = rel_l2(O[0, h], ref)
        print(f"head {h}: relative L2 {rel:.3e}, worst error / bound {float((err / bound).max()):.3f}")
        assert np.all(err <= bound), int((err > bound).sum())
        assert rel <= EXACT_REL_L2, rel


@pytest.mark.gpu
@pytest.mark.parametrize("seed,N,nQ,nK,density,H", [(1, 3000, 20, 50, 0.3, 2), (3, 12480, 64, 256, 0.5, 2)])
def test_fp8_attention_random_inputs(oracle, seed, N, nQ, nK, density, H):
    svg2 = require_gpu()
    c = _quantized_case(svg2, oracle, _case(seed, N, nQ, nK, density, H))
    O = _run_fp8(svg2, c, SCALE)
    rels = [rel_l2(O[0, h], _reference(oracle, c, SCALE, h)) for h in range(H)]
    print("relative L2 per head", rels)
    assert max(rels) <= REL_L2, rels


@pytest.mark.gpu
def test_fp8_attention_ragged_edges_and_single_tile_units(oracle):
    """Ragged clusters (1 ... 257 rows, 1 ... 129 keys) and, separately, every Q cluster of at most
    128 rows over a stream of all N keys (the kernel's one-Q-tile ring schedule), sampled rows."""
    svg2 = require_gpu()
    q_sizes = [1, 127, 128, 129, 255, 256, 257, 0, 300]
    k_sizes = [1, 2, 127, 128, 129, 0, 560, 506]
    c = _quantized_case(svg2, oracle, _case(5, sum(q_sizes), len(q_sizes), len(k_sizes), 0.5, 1, q_sizes, k_sizes))
    O = _run_fp8(svg2, c, SCALE)
    rel = rel_l2(O[0, 0], _reference(oracle, c, SCALE, 0))
    assert rel <= REL_L2, rel
    c = _quantized_case(svg2, oracle, _case(7, 9000, 90, 9, 1.0, 1, empty=0.0))
    O = _run_fp8(svg2, c, SCALE)
    rows = np.random.default_rng(0).choice(9000, 600, replace=False)
    rel = rel_l2(O[0, 0][rows], _reference(oracle, c, SCALE, 0, rows))
    assert rel <= REL_L2, rel


@pytest.mark.gpu
def test_fp8_attention_running_max_growth(oracle):
    """Rows whose maximum grows by more than 2^8 after the first key tile: the O rescale runs on the
    FP8 path too (and P stays within E4M3's range, below 2^8 by the lazy threshold)."""
    svg2 = require_gpu()
    q_sizes = [200, 100, 256, 300, 1, 143]
    k_sizes = [90, 70, 130, 1, 64, 200, 37, 150, 58, 200]
    plants = {0: [(7, 1.0)], 1: [(5, 0.6), (9, 1.2)], 2: [(8, 1.0)], 3: [(6, 0.5), (9, 1.0)], 5: [(2, 1.0)]}
    c = _growth_case(31, q_sizes, k_sizes, plants, H=2)
    assert sum(_late_growth_rows(c, h, SCALE, 128) for h in range(2)) >= 300
    c = _quantized_case(svg2, oracle, c)
    O = _run_fp8(svg2, c, SCALE)
    rels = [rel_l2(O[0, h], _reference(oracle, c, SCALE, h)) for h in range(2)]
    print("relative L2 per head", rels)
    assert max(rels) <= REL_L2, rels


@pytest.mark.gpu
def test_fp8_layer_matches_oracle_and_the_host_buffer_layer(oracle):
    """svg2_layer with attn_fp8 = 1: the clustering stages are the bf16 layer's (same labels,
    offsets, mask), the output equals the oracle's FP8 attention on the layer's own permutation,
    offsets and mask, and svg2_layer_host (head groups) gives the same bits."""
    from tests.test_layer import run_layer
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    data = pool_layer_inputs(cfg, range(cfg.H))
    ref16 = run_layer(svg2, cfg, data, 0.9)
    res = run_layer(svg2, cfg, data, 0.9, attn_fp8=1)
    for key in ("labels_q", "labels_k", "perm_q", "perm_k", "q_off", "k_off", "mask", "sel_count"):
        np.testing.assert_array_equal(res[key], ref16[key], err_msg=key)
    valid = np.arange(cfg.nK)[None, None, None, :] < res["sel_count"][..., None]   # entries past sel_count are undefined
    np.testing.assert_array_equal(np.where(valid, res["sel_idx"], -1), np.where(valid, ref16["sel_idx"], -1))
    scale = float(np.float32(cfg.scale))
    rels = []
    for h in range(cfg.H):
        q, k, v = (data[x][0, h][None, None] for x in ("q", "k", "v"))
        (Q8, sq), (K8, sk), (V8, sv) = (_quantize_oracle(oracle, x) for x in (q, k, v))
        pq, pk = res["perm_q"][0, h], res["perm_k"][0, h]
        inv = np.empty_like(pq)
        inv[pq] = np.arange(pq.size, dtype=np.int32)
        ref = oracle.sparse_attention_fp8_rows(Q8[0, 0][pq], K8[0, 0][pk], V8[0, 0][pk], sq[0, 0], sk[0, 0],
                                               sv[0, 0], res["q_off"][0, h], res["k_off"][0, h], res["mask"][0, h],
                                               scale, inv)
        rels.append(rel_l2(res["o"][0, h], ref))
    print("relative L2 per head", rels)
    assert max(rels) <= REL_L2, rels

    B, H, N, d = data["q"].shape
    pin = lambda x: torch.from_numpy(x).to(torch.bfloat16).pin_memory()
    hq, hk, hv = pin(data["q"]), pin(data["k"]), pin(data["v"])
    ho = torch.empty(B, H, N, d, dtype=torch.bfloat16).pin_memory()
    Q, K, V = (torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    O = torch.empty_like(Q)
    cq = torch.zeros(B, H, cfg.nQ, d, device="cuda")
    ck = torch.zeros(B, H, cfg.nK, d, device="cuda")
    ws = svg2.workspace(B, H, N, d, cfg.nQ, cfg.nK)
    prm = svg2.LayerParams(cfg.nQ, cfg.nK, cfg.iters, svg2.SVG2_INIT_KMEANSPP, 0.9, scale, 1, svg2.DEFAULT_SEED_TOKENS,
                           attn_fp8=1)
    svg2.svg2_layer_host(hq, hk, hv, ho, Q, K, V, O, prm, cq, ck, ws, to_dev(data["uq"]), to_dev(data["uk"]),
                         heads_per_group=3, copy_stream=torch.cuda.Stream())
    torch.cuda.current_stream().synchronize()
    svg2.raise_on_device_error(ws)
    assert torch.equal(ho.view(torch.int16), torch.from_numpy(res["o"]).to(torch.bfloat16).view(torch.int16))


@pytest.mark.gpu
def test_fp8_rejects_other_head_dims():
    svg2 = require_gpu()
    x = torch.zeros(1, 1, 256, 64, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, 1, device="cuda")
    off = torch.tensor([[[0, 256]]], dtype=torch.int32, device="cuda")
    cnt = torch.ones(1, 1, 1, dtype=torch.int32, device="cuda")
    idx = torch.zeros(1, 1, 1, 1, dtype=torch.int32, device="cuda")
    O = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16, device="cuda")
    ws = svg2.workspace(1, 1, 256, 64, 1, 1)
    with pytest.raises(svg2.Svg2Error) as e:
        svg2.svg2_sparse_attn_fp8(x, x, x, s, s, s, off, off, cnt, idx, 0.125, O, ws)
    assert e.value.code == 2  # SVG2_ERR_UNSUPPORTED


@pytest.mark.gpu
def test_fp8_layer_from_float32_inputs(oracle):
    """The FP8 layer on float32 inputs: the quantiser reads the float32 values themselves (not a bf16
    rounding of them), so the oracle quantises the float32 planes."""
    from types import SimpleNamespace
    from tests.test_layer import run_layer
    svg2 = require_gpu()
    rng = np.random.default_rng(90)
    H, N, d, nQ, nK = 2, 1500, 128, 10, 30

    def mixture(comps=6, sigma=0.3):
        out = np.empty((1, H, N, d), np.float32)
        for h in range(H):
            centres = rng.standard_normal((comps, d), dtype=np.float32)
            out[0, h] = centres[rng.integers(0, comps, N)] + sigma * rng.standard_normal((N, d), dtype=np.float32)
        return out

    data = {"q": mixture(), "k": mixture(), "v": rng.standard_normal((1, H, N, d), dtype=np.float32),
            "uq": rng.random((1, H, nQ)), "uk": rng.random((1, H, nK))}
    assert not np.array_equal(data["q"], I.round_to_bf16(data["q"]))
    cfg = SimpleNamespace(nQ=nQ, nK=nK, iters=3, scale=float(np.float32(1 / np.sqrt(d))), dtype="f32")
    res = run_layer(svg2, cfg, data, 0.9, seed_tokens=0, attn_fp8=1)
    rels = []
    for h in range(H):
        (Q8, sq), (K8, sk), (V8, sv) = (_quantize_oracle(oracle, data[x][:, h:h + 1]) for x in ("q", "k", "v"))
        pq, pk = res["perm_q"][0, h], res["perm_k"][0, h]
        inv = np.empty_like(pq)
        inv[pq] = np.arange(pq.size, dtype=np.int32)
        ref = oracle.sparse_attention_fp8_rows(Q8[0, 0][pq], K8[0, 0][pk], V8[0, 0][pk], sq[0, 0], sk[0, 0],
                                               sv[0, 0], res["q_off"][0, h], res["k_off"][0, h], res["mask"][0, h],
                                               cfg.scale, inv)
        rels.append(rel_l2(res["o"][0, h], ref))
    print("relative L2 per head", rels)
    assert max(rels) <= REL_L2, rels


def test_exact_p_bound_catches_misordered_keys(oracle):
    """On the CPU: the exact-P bound has the power the GPU test relies on.  A wrong byte order in the
    packed P (keys of a 4-key group multiplied by each other's V rows) is planted in the oracle's inputs
    as V rows swapped pairwise inside every group of 4; the output then leaves the bound almost
    everywhere, while the unplanted reference stays inside it."""
    c = _exact_p_case(60, 1500, 10, 20, 0.5, 1)
    scale = float(np.float32(np.log(2.0)))
    ref = _reference(oracle, c, scale, 0)
    planted = dict(c)
    v = c["V8"].copy()
    n4 = v.shape[2] // 4 * 4
    g = v[0, 0, :n4].reshape(-1, 4, v.shape[3])
    v[0, 0, :n4] = g[:, [2, 3, 0, 1]].reshape(n4, v.shape[3])
    planted["V8"] = v
    wrong = _reference(oracle, planted, scale, 0)
    bound = (2.0 ** -8 + 2e-4) * np.abs(ref) + 1e-6 * np.abs(ref).max()
    outside = float((np.abs(wrong - ref) > bound).mean())
    assert outside > 0.9, outside
    assert rel_l2(wrong, ref) > 100 * EXACT_REL_L2
