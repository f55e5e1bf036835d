"""Variable-block-size sparse attention kernel vs the oracle on oracle-supplied permuted inputs,
cluster offsets and masks (Method (4); section 4.3).  Tolerance: max-abs 2e-2, mean-abs 2e-3
(bf16 kernel vs float64 oracle)."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, require_gpu, to_dev

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _case(seed, N, nQ, nK, density, H=1, q_sizes=None, k_sizes=None, empty=0.1):
    rng = np.random.default_rng(seed)
    d = 128
    out = {k: [] for k in ("Qp", "Kp", "Vp", "q_off", "k_off", "mask")}
    for h in range(H):
        if q_sizes is None:
            lq = I.random_labels(N, nQ, seed * 7 + h, empty)
            qo = np.concatenate([[0], np.cumsum(np.bincount(lq, minlength=nQ))])
        else:
            qo = np.concatenate([[0], np.cumsum(q_sizes)])
        if k_sizes is None:
            lk = I.random_labels(N, nK, seed * 11 + h, empty)
            ko = np.concatenate([[0], np.cumsum(np.bincount(lk, minlength=nK))])
        else:
            ko = np.concatenate([[0], np.cumsum(k_sizes)])
        mask = (rng.random((nQ, nK)) < density).astype(np.uint8)
        ck = np.diff(ko)
        for i in range(nQ):
            if not (mask[i] & (ck > 0)).any():
                mask[i, int(np.argmax(ck))] = 1
        mask[:, ck == 0] = 0
        out["q_off"].append(qo.astype(np.int32))
        out["k_off"].append(ko.astype(np.int32))
        out["mask"].append(mask)
        for key in ("Qp", "Kp", "Vp"):
            out[key].append(I.round_to_bf16(rng.standard_normal((N, d), dtype=np.float32)))
    return {k: np.stack(v)[None] for k, v in out.items()}


def _ell(mask):
    nK = mask.shape[-1]
    sel_count = mask.sum(-1).astype(np.int32)
    sel_idx = np.zeros(mask.shape, np.int32)
    it = np.ndindex(*mask.shape[:-1])
    for idx in it:
        kept = np.nonzero(mask[idx])[0]
        sel_idx[idx][:kept.size] = kept
    return sel_count, sel_idx


def _run_gpu(svg2, c, scale, perm_q=None):
    B, H, N, d = c["Qp"].shape
    nQ, nK = c["mask"].shape[-2:]
    sel_count, sel_idx = _ell(c["mask"])
    O = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    ws = svg2.workspace(B, H, N, d, nQ, nK)
    svg2.svg2_sparse_attn(bf16_dev(c["Qp"]), bf16_dev(c["Kp"]), bf16_dev(c["Vp"]), to_dev(c["q_off"]),
                          to_dev(c["k_off"]), to_dev(sel_count), to_dev(sel_idx), scale, O, ws,
                          perm_q=None if perm_q is None else to_dev(perm_q))
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    return host(O)


def _compare(oracle, c, O, scale, heads=None, rows=None):
    H = c["Qp"].shape[1]
    worst, means = 0.0, []
    for h in (range(H) if heads is None else heads):
        ref = oracle.sparse_attention_rows(c["Qp"][0, h], c["Kp"][0, h], c["Vp"][0, h], c["q_off"][0, h],
                                           c["k_off"][0, h], c["mask"][0, h], scale, rows)
        got = O[0, h] if rows is None else O[0, h][rows]
        err = np.abs(got - ref)
        worst = max(worst, float(err.max()))
        means.append(float(err.mean()))
    assert worst <= MAX_ABS, worst
    assert max(means) <= MEAN_ABS, means
    return worst, max(means)


SCALE = float(np.float32(1 / np.sqrt(128)))


@pytest.mark.gpu
@pytest.mark.parametrize("seed,N,nQ,nK,density,H", [
    (1, 3000, 20, 50, 0.3, 2),
    (2, 4096, 16, 32, 1.0, 1),
    (3, 12480, 64, 256, 0.5, 2),
    (4, 700, 3, 5, 0.6, 1),
])
def test_sparse_attention_matches_oracle(oracle, seed, N, nQ, nK, density, H):
    svg2 = require_gpu()
    c = _case(seed, N, nQ, nK, density, H)
    O = _run_gpu(svg2, c, SCALE)
    print("max/mean abs err", _compare(oracle, c, O, SCALE))


@pytest.mark.gpu
def test_ragged_cluster_edges(oracle):
    """Q clusters of 1, 127, 128, 129, 255, 256, 257 rows; K clusters of 1, 2, 127, 128, 129 keys."""
    svg2 = require_gpu()
    q_sizes = [1, 127, 128, 129, 255, 256, 257, 0, 300]
    k_sizes = [1, 2, 127, 128, 129, 0, 560, 506]
    N = sum(q_sizes)
    assert sum(k_sizes) == N
    c = _case(5, N, len(q_sizes), len(k_sizes), 0.5, 1, q_sizes, k_sizes)
    c["mask"][0, 0, 1, :] = 0
    c["mask"][0, 0, 1, 0] = 1            # a Q cluster that sees a single key: output = that V row
    O = _run_gpu(svg2, c, SCALE)
    _compare(oracle, c, O, SCALE)
    r = q_sizes[0]
    np.testing.assert_array_equal(O[0, 0, r:r + 127], np.broadcast_to(c["Vp"][0, 0, 0], (127, 128)))


@pytest.mark.gpu
def test_fused_inverse_permutation(oracle):
    svg2 = require_gpu()
    c = _case(6, 2500, 12, 40, 0.4, 2)
    perm = np.stack([np.random.default_rng(h).permutation(2500).astype(np.int32) for h in range(2)])[None]
    Op = _run_gpu(svg2, c, SCALE)
    O = _run_gpu(svg2, c, SCALE, perm_q=perm)
    for h in range(2):
        np.testing.assert_array_equal(O[0, h][perm[0, h]], Op[0, h])


@pytest.mark.gpu
def test_single_tile_units_and_long_streams(oracle):
    """Every Q cluster <= 128 rows (single-tile units) and all keys kept (stream of N keys)."""
    svg2 = require_gpu()
    c = _case(7, 9000, 90, 9, 1.0, 1, empty=0.0)
    O = _run_gpu(svg2, c, SCALE)
    rows = np.random.default_rng(0).choice(9000, 600, replace=False)
    _compare(oracle, c, O, SCALE, rows=rows)
