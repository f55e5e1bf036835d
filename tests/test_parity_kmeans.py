"""k-means kernels vs the oracle (Method (1)).

Assignments are checked lockstep (one iteration from the oracle's centroids, at every iteration):
a token may differ from the oracle only at a near-tie (oracle top-2 distance gap < 1e-4 relative),
and such tokens must be <= 0.1%.  Centroids: relative error <= 1e-3 per non-empty cluster.  The
k-means++ seeds are exact (same fixed-point D^2 sampling), which the first iteration checks.
"""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, near_tie, pool_layer_inputs, require_gpu, to_dev


def _xdev(cfg, x):
    return to_dev(x) if cfg.dtype == "f32" else bf16_dev(x)


def _run(svg2, cfg, X, k, iters, init, C0=None, u=None, seed_tokens=0):
    B, H, N, d = X.shape
    Xd = _xdev(cfg, X)
    C = to_dev(C0.astype(np.float32)) if C0 is not None else torch.zeros(B, H, k, d, device="cuda")
    lab = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, H, k, dtype=torch.int32, device="cuda")
    ws = svg2.workspace(B, H, N, d, k, k)
    svg2.svg2_kmeans(Xd, k, iters, init, C, lab, cnt, ws, u=None if u is None else to_dev(u), seed_tokens=seed_tokens)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    return host(C), host(lab), host(cnt)


def _rel_centroid_err(C, Cref, counts):
    nz = counts > 0
    num = np.linalg.norm(C[nz].astype(np.float64) - Cref[nz], axis=1)
    den = np.maximum(np.linalg.norm(Cref[nz], axis=1), 1e-30)
    return float((num / den).max()) if nz.any() else 0.0


def _check_assign(labels, ref_labels, d1, d2, what):
    diff = labels != ref_labels
    tie = near_tie(d1, d2)
    assert not (diff & ~tie).any(), f"{what}: {(diff & ~tie).sum()} mismatches away from near-ties"
    assert diff.sum() <= 0.001 * labels.size, f"{what}: {diff.sum()} near-tie mismatches"
    return int(diff.sum()), int(tie.sum())


def _seeds(svg2, X, k, u, seed_tokens, dev_x):
    B, H, N, d = X.shape
    C = torch.zeros(B, H, k, d, device="cuda")
    ws = svg2.workspace(B, H, N, d, k, k)
    svg2.svg2_kmeanspp(dev_x, k, to_dev(u), C, ws, seed_tokens=seed_tokens)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    return host(C)


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name,heads,role,seed_tokens", [
    ("tiny", [0], "k", 0),                     # float32, d = 64 (CUDA-core seeding)
    ("small", [0, 3], "k", 0),                 # 12480 candidates, k = 256, clusters of several CTAs
    ("small", [1], "q", 5000),                 # 5000 candidates, ragged last tile
    ("small", [2], "k", 300),                  # 300 candidates for 256 seeds, one CTA
    ("wan720p", [4], "q", 16384), ("wan720p", [9], "k", 16384),
    ("wan720p", [1], "k", 0),                  # all 75600 tokens: 13+ CTAs per head
    ("hunyuan720p", [6], "k", 16384)])         # k = 1000
def test_kmeanspp_seeds_bit_exact(oracle, cfg_name, heads, role, seed_tokens):
    """The seeds are the oracle's: same fixed-point D^2 sampling, float64 D^2 in the same order."""
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    data = pool_layer_inputs(cfg, heads)
    X, u = data[role], data["u" + role]
    k = cfg.nQ if role == "q" else cfg.nK
    C = _seeds(svg2, X, k, u, seed_tokens, _xdev(cfg, X))
    idx = oracle.seed_candidates(X.shape[2], seed_tokens)
    for h in range(len(heads)):
        _, Cref = oracle.kmeanspp(np.ascontiguousarray(X[0, h][idx]), k, u[0, h])
        bad = np.nonzero((C[0, h] != Cref.astype(np.float32)).any(axis=1))[0]
        assert bad.size == 0, f"{cfg_name} head {heads[h]}: first differing seed {bad[:1]} of {k}"


@pytest.mark.gpu
def test_kmeanspp_seeds_with_duplicate_tokens(oracle):
    """Three distinct rows repeated: after three seeds every D^2 is 0, so the rest are uniform picks."""
    svg2 = require_gpu()
    rng = np.random.default_rng(11)
    base = I.round_to_bf16(rng.standard_normal((3, 128)).astype(np.float32))
    X = base[rng.integers(0, 3, size=4096)][None, None].copy()
    u = rng.random((1, 1, 8))
    C = _seeds(svg2, X, 8, u, 0, bf16_dev(X))
    _, Cref = oracle.kmeanspp(X[0, 0], 8, u[0, 0])
    np.testing.assert_array_equal(C[0, 0], Cref.astype(np.float32))


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name,heads,role,seed_tokens", [
    ("tiny", [0], "q", 0), ("tiny", [0], "k", 0), ("small", [0, 5], "q", 0), ("small", [0, 5], "k", 0),
    ("wan720p", [7], "k", 0), ("wan720p", [7], "q", 16384), ("wan720p", [2], "k", 16384),
    ("hunyuan720p", [3], "k", 0), ("hunyuan720p", [5], "k", 16384)])
def test_kmeanspp_then_lockstep_lloyd(oracle, cfg_name, heads, role, seed_tokens):
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    data = pool_layer_inputs(cfg, heads)
    X = data[role]
    u = data["u" + role]
    k = cfg.nQ if role == "q" else cfg.nK
    iters = cfg.iters
    # iteration 1 from k-means++ seeds (the seeds themselves are checked through it)
    C1, lab1, cnt1 = _run(svg2, cfg, X, k, 1, svg2.SVG2_INIT_KMEANSPP, u=u, seed_tokens=seed_tokens)
    idx = oracle.seed_candidates(X.shape[2], seed_tokens)
    seeds0 = lambda h: oracle.kmeanspp(np.ascontiguousarray(X[0, h][idx]), k, u[0, h])[1]
    stats = []
    for h in range(len(heads)):
        C0 = seeds0(h)
        ref_lab, d1, d2 = oracle.assign(X[0, h], C0)
        stats.append(_check_assign(lab1[0, h], ref_lab, d1, d2, f"{cfg_name} head {heads[h]} iter 1"))
        Cref, cref = oracle.update(X[0, h], lab1[0, h], C0)          # same labels: exact up to fp32 rounding
        np.testing.assert_allclose(C1[0, h], Cref.astype(np.float32), rtol=0, atol=0)
        assert np.array_equal(cnt1[0, h], cref)
    # lockstep: every further iteration starts from the oracle's own centroids
    Cor = np.stack([oracle.lloyd(X[0, h], seeds0(h), 1)[0] for h in range(len(heads))])
    flipped_clusters = 0
    for it in range(2, iters + 1):
        Cin = Cor.astype(np.float32).astype(np.float64)
        C, lab, cnt = _run(svg2, cfg, X, k, 1, svg2.SVG2_INIT_GIVEN, C0=Cin[None])
        nxt = []
        for h in range(len(heads)):
            ref_lab, d1, d2 = oracle.assign(X[0, h], Cin[h])
            stats.append(_check_assign(lab[0, h], ref_lab, d1, d2, f"{cfg_name} head {heads[h]} iter {it}"))
            # the update given the GPU's own labels is exact (float64 sums in the oracle's order)
            Cg, cg = oracle.update(X[0, h], lab[0, h], Cin[h])
            np.testing.assert_array_equal(C[0, h], Cg.astype(np.float32))
            assert np.array_equal(cnt[0, h], cg)
            # against the oracle's labels: every cluster no near-tie flip touched is within 1e-3
            Cref, cref = oracle.update(X[0, h], ref_lab, Cin[h])
            moved = lab[0, h] != ref_lab
            touched = np.zeros(k, bool)
            touched[lab[0, h][moved]] = True
            touched[ref_lab[moved]] = True
            flipped_clusters += int(touched.sum())
            keep = ~touched
            assert _rel_centroid_err(C[0, h][keep], Cref[keep], cref[keep]) <= 1e-3
            nxt.append(oracle.update(X[0, h], oracle.assign(X[0, h], Cor[h])[0], Cor[h])[0])
        Cor = np.stack(nxt)
    print(f"{cfg_name}/{role}: clusters touched by near-tie flips over the lockstep run: {flipped_clusters}")
    print(f"{cfg_name}/{role} seed_tokens={seed_tokens}: (near-tie mismatches, near-ties) per head/iteration: {stats}")


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name,role", [("tiny", "k"), ("small", "k")])
def test_full_run_matches_oracle(oracle, cfg_name, role):
    """All iterations on the GPU from k-means++ (reported; mismatches may cascade from near-ties)."""
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    heads = [0, 1] if cfg.H > 1 else [0]
    data = pool_layer_inputs(cfg, heads)
    X, u = data[role], data["u" + role]
    k = cfg.nQ if role == "q" else cfg.nK
    C, lab, cnt = _run(svg2, cfg, X, k, cfg.iters, svg2.SVG2_INIT_KMEANSPP, u=u)
    for h in range(len(heads)):
        Cref, lref, cref = oracle.kmeans(X[0, h], k, cfg.iters, u[0, h])
        agree = float((lab[0, h] == lref).mean())
        err = _rel_centroid_err(C[0, h], Cref, cref)
        print(f"{cfg_name}/{role} head {heads[h]}: label agreement {agree:.6f}, centroid rel err {err:.2e}")
        assert agree >= 0.99
        assert cnt[0, h].sum() == X.shape[2]


def overflow_case(seed=21, H=4, groups=40, per_group=12, N=4096, gap=3e-4, offset=8.0):
    """Tokens with more than four centroids inside the assignment's tolerance band.

    Per head, `groups` base points x_g with coordinates near +-offset (so ||x||^2 ~ 128 offset^2 and
    float32 scores ||c||^2 - 2 x.c carry rounding errors far larger than the spacing below), and
    per base point `per_group` float32 centroids at squared distance (1 + gap*i) from it, i = 0..,
    in shuffled index order.  Every token is a copy of one base point.  Its nearest centroid is then
    ahead of the next by a relative gap of `gap` (not a near-tie), while all `per_group` centroids lie
    within 2^-11 (||x||^2 + d_min) of the nearest, so a short candidate list kept by approximate
    score can miss the nearest one.
    """
    rng = np.random.default_rng(seed)
    d, k = 128, groups * per_group
    X = np.empty((1, H, N, d), np.float32)
    C = np.empty((1, H, k, d), np.float32)
    for h in range(H):
        base = offset * rng.choice([-1.0, 1.0], size=(groups, d)) + 0.5 * rng.standard_normal((groups, d))
        base = I.round_to_bf16(base.astype(np.float32)).astype(np.float64)
        for g in range(groups):
            u = rng.standard_normal((per_group, d))
            u /= np.linalg.norm(u, axis=1, keepdims=True)
            r = np.sqrt(1.0 + gap * np.arange(per_group))
            idx = g * per_group + rng.permutation(per_group)
            C[0, h, idx] = (base[g] + r[:, None] * u).astype(np.float32)
        X[0, h] = base[rng.integers(0, groups, size=N)].astype(np.float32)
    return X, C


def test_overflow_case_has_crowded_candidates_and_no_near_ties(oracle):
    """The construction itself (CPU): nearest centroid unique by >= 1e-4 relative, and at least
    eight centroids within 2^-11 (||x||^2 + d_min) of the nearest for every token."""
    X, C = overflow_case(H=1, N=256)
    x, c = X[0, 0].astype(np.float64), C[0, 0].astype(np.float64)
    lab, d1, d2 = oracle.assign(X[0, 0], c)
    assert not near_tie(d1, d2).any()
    dist = ((x[:, None, :] - c[None, :, :]) ** 2).sum(-1)
    band = 2.0 ** -11 * ((x * x).sum(1) + d1)
    crowd = (dist <= (d1 + band)[:, None]).sum(1)
    assert crowd.min() >= 8, crowd.min()
    np.testing.assert_array_equal(lab, dist.argmin(1))


@pytest.mark.gpu
def test_assign_candidate_list_overflow(oracle):
    """A token whose tolerance band holds more centroids than the epilogue's candidate list must
    still get its exact nearest centroid: 0 mismatches away from near-ties (there are none here)."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]          # bf16, d = 128: the tensor-core assignment and its re-rank
    X, C0 = overflow_case()
    k = C0.shape[2]
    _, lab, _ = _run(svg2, cfg, X, k, 1, svg2.SVG2_INIT_GIVEN, C0=C0.astype(np.float64))
    for h in range(X.shape[1]):
        ref_lab, d1, d2 = oracle.assign(X[0, h], C0[0, h].astype(np.float64))
        assert not near_tie(d1, d2).any()
        bad = int((lab[0, h] != ref_lab).sum())
        assert bad == 0, f"head {h}: {bad} of {X.shape[2]} tokens not at their nearest centroid"


def _pruned_iteration_check(oracle, svg2, cfg, X, C_in, what):
    """Iteration 2 of a k-means run from C_in (the pruned search for k >= 500) against the oracle's
    assignment to the centroids iteration 1 produced (exact given the GPU's own iteration-1 labels)."""
    k = C_in.shape[2]
    _, lab1, _ = _run(svg2, cfg, X, k, 1, svg2.SVG2_INIT_GIVEN, C0=C_in)
    C2, lab2, _ = _run(svg2, cfg, X, k, 2, svg2.SVG2_INIT_GIVEN, C0=C_in)
    stats = []
    for h in range(X.shape[1]):
        C1, _ = oracle.update(X[0, h], lab1[0, h], C_in[0, h])
        ref, d1, d2 = oracle.assign(X[0, h], C1)
        stats.append(_check_assign(lab2[0, h], ref, d1, d2, f"{what} head {h} iteration 2"))
        Cref, _ = oracle.update(X[0, h], lab2[0, h], C1)
        np.testing.assert_array_equal(C2[0, h], Cref.astype(np.float32))
    return stats


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name,heads,stage,k", [("small", [0, 3], 0, 512), ("wan720p", [2], 0, 500),
                                                   ("wan720p", [5], 2, 500), ("hunyuan720p", [1], 0, 1000)])
def test_pruned_assignment_lockstep(oracle, cfg_name, heads, stage, k):
    """The Lloyd iterations after the first use the pruned search when k >= 500 (the K side of the
    Wan and Hunyuan layers): from the k-means++ seeds (stage 0) or from centroids two oracle
    iterations later (stage 2); the small shape with k = 512 gives tiles of few tokens per cluster."""
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    data = pool_layer_inputs(cfg, heads)
    X = data["k"]
    u = np.random.default_rng(cfg.cfg_id + 77).random((1, len(heads), k))
    idx = oracle.seed_candidates(X.shape[2], svg2.DEFAULT_SEED_TOKENS)
    C_in = []
    for h in range(len(heads)):
        C0 = oracle.kmeanspp(np.ascontiguousarray(X[0, h][idx]), k, u[0, h])[1]
        if stage:
            C0 = oracle.lloyd(X[0, h], C0, stage)[0]
        C_in.append(C0.astype(np.float32).astype(np.float64))
    stats = _pruned_iteration_check(oracle, svg2, cfg, X, np.stack(C_in)[None], cfg_name)
    print(f"{cfg_name} stage {stage}: (near-tie mismatches, near-ties) {stats}")


@pytest.mark.gpu
def test_pruned_assignment_duplicate_centroids_and_far_tokens(oracle):
    """Centroids given twice (distance 0 between them: neither may prune the other, and the first
    iteration's ties go to the lower index), and a few tokens far from every centroid (a large
    radius that keeps most clusters as candidates: the search then runs over several chunks of 64)."""
    svg2 = require_gpu()
    cfg = I.CONFIGS["small"]
    rng = np.random.default_rng(33)
    k, N = 600, 9000
    centres = rng.standard_normal((k, 128))
    centres[300:] = centres[:300]                       # clusters 300..599 duplicate 0..299
    lab = rng.integers(0, 300, size=N)
    X = centres[lab] + 0.3 * rng.standard_normal((N, 128))
    X[:40] = 6.0 * rng.standard_normal((40, 128))       # far tokens
    X = I.round_to_bf16(X.astype(np.float32))[None, None]
    C_in = centres.astype(np.float32).astype(np.float64)[None, None]
    _, lab1, _ = _run(svg2, cfg, X, k, 1, svg2.SVG2_INIT_GIVEN, C0=C_in)
    assert (lab1[0, 0] < 300).all()                     # a duplicate never beats the lower index
    stats = _pruned_iteration_check(oracle, svg2, cfg, X, C_in, "duplicates")
    print(stats)
