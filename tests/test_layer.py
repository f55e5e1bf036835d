"""The whole layer through the C ABI (svg2_layer) vs the oracle, on the configured workloads.

Per head, each stage is checked against the oracle given the GPU's own upstream results (so a
near-tie label difference in k-means does not leak into the attention check):
  permutation/offsets from the GPU labels: bit-exact; selection from the GPU centroids: mask equal
  except where a float32 weight rounds differently (counted); attention on the GPU's permuted
  inputs and mask: max-abs 2e-2, mean-abs 2e-3 and relative L2 1e-2 (sampled rows at full size).  The independent
  end-to-end agreement (labels, density, output error vs the oracle's own layer) is reported.
"""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, pool_layer_inputs, require_gpu, to_dev

MAX_ABS, MEAN_ABS, REL_L2 = 2e-2, 2e-3, 1e-2


def run_layer(svg2, cfg, data, top_p, init=None, cq=None, ck=None, fuse=1, seed_tokens=None, attn_fp8=0):
    B, H, N, d = data["q"].shape
    conv = to_dev if cfg.dtype == "f32" else bf16_dev
    Q, K, V = conv(data["q"]), conv(data["k"]), conv(data["v"])
    cq = torch.zeros(B, H, cfg.nQ, d, device="cuda") if cq is None else cq
    ck = torch.zeros(B, H, cfg.nK, d, device="cuda") if ck is None else ck
    O = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    outs = svg2.layer_output_buffers(B, H, N, cfg.nQ, cfg.nK)
    ws = svg2.workspace(B, H, N, d, cfg.nQ, cfg.nK)
    prm = svg2.LayerParams(cfg.nQ, cfg.nK, cfg.iters, svg2.SVG2_INIT_KMEANSPP if init is None else init, top_p,
                           float(np.float32(cfg.scale)), fuse,
                           svg2.DEFAULT_SEED_TOKENS if seed_tokens is None else seed_tokens, attn_fp8)
    svg2.svg2_layer(Q, K, V, prm, cq, ck, O, ws, to_dev(data["uq"]), to_dev(data["uk"]), outs)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    res = {k: host(v) for k, v in outs.items()}
    res.update(o=host(O), cq=host(cq), ck=host(ck))
    return res


def check_head(oracle, cfg, data, res, h, top_p, rows=None):
    scale = float(np.float32(cfg.scale))
    q, k, v = data["q"][0, h], data["k"][0, h], data["v"][0, h]
    g = {key: val[0, h] for key, val in res.items()}
    # permutation of the GPU labels: bit-exact
    pq, qo = oracle.permute(g["labels_q"], cfg.nQ)
    pk, ko = oracle.permute(g["labels_k"], cfg.nK)
    assert np.array_equal(g["perm_q"], pq) and np.array_equal(g["q_off"], qo)
    assert np.array_equal(g["perm_k"], pk) and np.array_equal(g["k_off"], ko)
    assert np.array_equal(g["count_q"], np.diff(qo)) and np.array_equal(g["count_k"], np.diff(ko))
    # centroids are the means of the GPU's final labels (float64 sums rounded to float32)
    for C, X, lab, kk in ((g["cq"], q, g["labels_q"], cfg.nQ), (g["ck"], k, g["labels_k"], cfg.nK)):
        Cref, cnt = oracle.update(X, lab, C.astype(np.float64))
        np.testing.assert_array_equal(C, Cref.astype(np.float32))
    # selection from the GPU centroids
    w_ref = oracle.select_weights(g["cq"], g["ck"], g["count_k"], scale)
    np.testing.assert_allclose(g["weights"], w_ref, rtol=1e-6)
    mask_ref = oracle.topp(w_ref, g["count_k"], top_p)
    mism = int((g["mask"] != mask_ref).sum())
    assert mism <= 2, mism
    # attention on the GPU's permuted inputs and mask, compared in token order
    Qp, Kp, Vp = oracle.gather_rows(q, pq), oracle.gather_rows(k, pk), oracle.gather_rows(v, pk)
    if cfg.dtype == "f32":   # the kernels compute in bf16: the permuted copies are rounded
        Qp, Kp, Vp = I.round_to_bf16(Qp), I.round_to_bf16(Kp), I.round_to_bf16(Vp)
    inv = np.empty_like(pq)
    inv[pq] = np.arange(pq.size, dtype=np.int32)
    tok = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    ref = oracle.sparse_attention_rows(Qp, Kp, Vp, qo, ko, g["mask"], scale, inv[tok])
    err = np.abs(g["o"][tok] - ref)
    rel = float(np.linalg.norm((g["o"][tok] - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30))
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert rel <= REL_L2, rel
    dens = oracle.density(g["mask"], g["count_q"], g["count_k"])
    return dict(mask_mismatch=mism, max_abs=float(err.max()), mean_abs=float(err.mean()), rel_l2=rel, density=dens)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name", ["tiny", "small"])
def test_layer_small_configs_every_head(oracle, cfg_name):
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    data = pool_layer_inputs(cfg, range(cfg.H))
    top_p = cfg.top_p[0]
    res = run_layer(svg2, cfg, data, top_p)
    for h in range(cfg.H):
        st = check_head(oracle, cfg, data, res, h, top_p)
        e2e = oracle.layer_head(data["q"][0, h], data["k"][0, h], data["v"][0, h], cfg.nQ, cfg.nK, cfg.iters, top_p,
                                float(np.float32(cfg.scale)), data["uq"][0, h], data["uk"][0, h],
                                seed_tokens=svg2.DEFAULT_SEED_TOKENS)
        agree_q = float((res["labels_q"][0, h] == e2e["labels_q"]).mean())
        agree_k = float((res["labels_k"][0, h] == e2e["labels_k"]).mean())
        o_rel = float(np.linalg.norm(res["o"][0, h] - e2e["o"]) / np.linalg.norm(e2e["o"]))
        print(f"{cfg_name} head {h}: {st}; e2e label agreement q {agree_q:.5f} k {agree_k:.5f}, O rel-L2 {o_rel:.2e}")
        assert agree_q >= 0.99 and agree_k >= 0.99


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name", ["wan720p", "hunyuan720p"])
def test_layer_full_size_sampled_heads(oracle, cfg_name):
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    data = pool_layer_inputs(cfg, range(cfg.H))
    top_p = 0.9
    res = run_layer(svg2, cfg, data, top_p)
    rng = np.random.default_rng(cfg.cfg_id)
    for h in (0, cfg.H // 2, cfg.H - 1):
        rows = np.sort(rng.choice(cfg.N, 384, replace=False))
        st = check_head(oracle, cfg, data, res, h, top_p, rows)
        print(f"{cfg_name} head {h}: {st}")


@pytest.mark.gpu
def test_top_p_one_equals_dense_attention():
    """With every pair kept the permutation cancels (section 4.1): the layer equals dense attention."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    data = pool_layer_inputs(cfg, range(2))
    res = run_layer(svg2, cfg, data, 1.0)
    q, k, v = (torch.from_numpy(data[n]).cuda() for n in ("q", "k", "v"))
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=float(np.float32(cfg.scale)))
    err = np.abs(res["o"] - dense.cpu().numpy())
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


@pytest.mark.gpu
def test_unfused_and_fused_inverse_permutation_agree():
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    data = pool_layer_inputs(cfg, range(2))
    a = run_layer(svg2, cfg, data, 0.9, fuse=1)
    b = run_layer(svg2, cfg, data, 0.9, fuse=0)
    np.testing.assert_array_equal(a["o"], b["o"])


@pytest.mark.gpu
def test_warm_start_sequence_tracks_cold_start(oracle):
    """Centroid cache across denoising steps (section 4.3, Fig. 7(a)): warm start from the previous
    step's centroids with 2 iterations stays as close to dense attention (the oracle's, float64) as
    a cold start does."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    heads = range(2)
    d0 = pool_layer_inputs(cfg, heads, 0)
    r0 = run_layer(svg2, cfg, d0, 0.9)
    cq, ck = torch.from_numpy(r0["cq"]).cuda(), torch.from_numpy(r0["ck"]).cuda()
    warm_cfg = I.LayerConfig(**{**cfg.__dict__, "iters": 2, "drift": 0.05})
    for step in range(1, 5):
        ds = {key: val.copy() for key, val in d0.items()}
        eps = np.random.default_rng(step).standard_normal(ds["q"].shape, dtype=np.float32)
        ds["q"] = I.round_to_bf16(ds["q"] + 0.05 * step * eps)
        ds["k"] = I.round_to_bf16(ds["k"] + 0.05 * step * eps[:, :, ::-1])
        warm = run_layer(svg2, warm_cfg, ds, 0.9, init=svg2.SVG2_INIT_GIVEN, cq=cq.clone(), ck=ck.clone())
        cold = run_layer(svg2, cfg, ds, 0.9)
        for h in heads:
            check_head(oracle, warm_cfg, ds, warm, h, 0.9, rows=np.arange(0, cfg.N, 97))
        # both outputs against the oracle's float64 dense attention of this step (64 sampled rows
        # per head): the sparsity's error, which warm start must not make worse than a cold start
        rows = np.sort(np.random.default_rng(100 + step).choice(cfg.N, 64, replace=False))
        scale = float(np.float32(cfg.scale))
        dense = np.stack([oracle.dense_attention_rows(ds["q"][0, h], ds["k"][0, h], ds["v"][0, h], scale, rows)
                          for h in heads])
        e_w = np.linalg.norm(warm["o"][0][:, rows] - dense) / np.linalg.norm(dense)
        e_c = np.linalg.norm(cold["o"][0][:, rows] - dense) / np.linalg.norm(dense)
        drift_q = np.linalg.norm(warm["cq"] - host(cq)) / np.linalg.norm(host(cq))
        print(f"step {step}: rel-L2 vs float64 dense attention: warm {e_w:.4f} cold {e_c:.4f}; Q centroid drift {drift_q:.4f}")
        assert e_w <= 1.5 * e_c + 0.02
        cq, ck = torch.from_numpy(warm["cq"]).cuda(), torch.from_numpy(warm["ck"]).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("heads_per_group,separate_copy_stream", [(3, True), (0, True), (8, False)])
def test_host_buffer_layer_matches_device_layer(heads_per_group, separate_copy_stream):
    """svg2_layer_host (pinned host in/out, head groups, copies on their own stream) gives the same
    bits as svg2_layer on device buffers: the heads are independent and every kernel is the same."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    data = pool_layer_inputs(cfg, range(cfg.H))
    ref = run_layer(svg2, cfg, data, 0.9)
    B, H, N, d = data["q"].shape
    pin = lambda x: torch.from_numpy(x).to(torch.bfloat16).pin_memory()
    hq, hk, hv = pin(data["q"]), pin(data["k"]), pin(data["v"])
    ho = torch.empty(B, H, N, d, dtype=torch.bfloat16).pin_memory()
    Q, K, V = (torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    O = torch.empty_like(Q)
    cq = torch.zeros(B, H, cfg.nQ, d, device="cuda")
    ck = torch.zeros(B, H, cfg.nK, d, device="cuda")
    ws = svg2.workspace(B, H, N, d, cfg.nQ, cfg.nK)
    prm = svg2.LayerParams(cfg.nQ, cfg.nK, cfg.iters, svg2.SVG2_INIT_KMEANSPP, 0.9, float(np.float32(cfg.scale)), 1,
                           svg2.DEFAULT_SEED_TOKENS)
    cs = torch.cuda.Stream() if separate_copy_stream else None
    svg2.svg2_layer_host(hq, hk, hv, ho, Q, K, V, O, prm, cq, ck, ws, to_dev(data["uq"]), to_dev(data["uk"]),
                         heads_per_group=heads_per_group, copy_stream=cs)
    torch.cuda.current_stream().synchronize()
    svg2.raise_on_device_error(ws)
    assert torch.equal(ho.view(torch.int16), torch.from_numpy(ref["o"]).to(torch.bfloat16).view(torch.int16))
    np.testing.assert_array_equal(host(cq), ref["cq"])
    np.testing.assert_array_equal(host(ck), ref["ck"])


def _mixture(rng, B, H, N, d, comps=8, sigma=0.3):
    out = np.empty((B, H, N, d), np.float32)
    for b in range(B):
        for h in range(H):
            centres = rng.standard_normal((comps, d), dtype=np.float32)
            out[b, h] = centres[rng.integers(0, comps, N)] + sigma * rng.standard_normal((N, d), dtype=np.float32)
    return I.round_to_bf16(out)


def _run_and_check(oracle, B, H, N, nQ, nK, iters, top_p, seed_tokens, seed):
    """svg2_layer on a (B, H) batch of mixtures, every (b, h) plane checked stage by stage."""
    from types import SimpleNamespace
    svg2 = require_gpu()
    rng = np.random.default_rng(seed)
    d = 128
    data = {"q": _mixture(rng, B, H, N, d), "k": _mixture(rng, B, H, N, d),
            "v": I.round_to_bf16(rng.standard_normal((B, H, N, d), dtype=np.float32)),
            "uq": rng.random((B, H, nQ)), "uk": rng.random((B, H, nK))}
    cfg = SimpleNamespace(nQ=nQ, nK=nK, iters=iters, scale=float(np.float32(1 / np.sqrt(d))), dtype="bf16")
    res = run_layer(svg2, cfg, data, top_p, seed_tokens=seed_tokens)
    stats = []
    for b in range(B):
        db = {key: val[b:b + 1] for key, val in data.items()}
        rb = {key: val[b:b + 1] for key, val in res.items()}
        for h in range(H):
            stats.append(check_head(oracle, cfg, db, rb, h, top_p))
    return stats


@pytest.mark.gpu
def test_layer_batch_of_two_ragged_length(oracle):
    """B = 2 (every kernel indexes (b, h) planes), N = 1000 (ragged 128-row tiles and 256-row units),
    k-means++ over strided candidates."""
    stats = _run_and_check(oracle, B=2, H=3, N=1000, nQ=12, nK=40, iters=3, top_p=0.9, seed_tokens=400, seed=21)
    print(stats)


@pytest.mark.gpu
def test_layer_degenerate_cluster_counts(oracle):
    """One Q cluster holding every token, and as many K clusters as tokens (k-means++ then runs out of
    positive D^2 and picks repeated seeds, so some K clusters stay empty)."""
    stats = _run_and_check(oracle, B=1, H=2, N=300, nQ=1, nK=300, iters=2, top_p=0.5, seed_tokens=0, seed=22)
    print(stats)
