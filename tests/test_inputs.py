"""The seeded input generator holds to its stated recipe (no GPU needed).

The generator stands in for the Wan 2.1 / HunyuanVideo activations the pages measure on
("Sparse VideoGen2" wiki summary, Results, Table 1): Gaussian mixtures whose component is
piecewise constant over voxels of the (t, h, w) token grid, optionally with a fraction of tokens
given a random component, bf16-rounded for the bf16 shapes.  These tests check that recipe
against things outside the generator: torch's own float32 -> bfloat16 conversion, the voxel
geometry, and reproducibility of every seeded stream.
"""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I


def test_round_to_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0,
        rng.standard_normal(2000).astype(np.float32) * 1e-30,         # subnormal range of float32
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38], np.float32),
    ])
    # exact ties: bf16 value + half an ulp, both parities of the kept bit
    base = rng.standard_normal(1000).astype(np.float32)
    base = (base.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties])
    ours = I.round_to_bf16(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), theirs.view(np.uint32))
    # already-bf16 values are fixed points and bf16_bits keeps their top half
    np.testing.assert_array_equal(I.round_to_bf16(ours).view(np.uint32), ours.view(np.uint32))
    np.testing.assert_array_equal(I.bf16_bits(ours), (ours.view(np.uint32) >> 16).astype(np.uint16))


def test_round_to_bf16_rejects_non_finite():
    with pytest.raises(ValueError):
        I.round_to_bf16(np.array([1.0, np.inf], np.float32))


@pytest.mark.parametrize("name", ["tiny", "small", "wan720p"])
def test_component_map_is_piecewise_constant_over_voxels(name):
    cfg = I.CONFIGS[name]
    comp = I.component_map(cfg, 0, 3 % cfg.H)
    T, Hg, Wg = cfg.grid
    vt, vh, vw = cfg.voxel
    assert comp.shape == (cfg.N,) and comp.min() >= 0 and comp.max() < cfg.components
    grid = comp.reshape(T, Hg, Wg)
    # voxel id of every token under the flatten order n = (t * Hg + h) * Wg + w
    t, h, w = np.meshgrid(np.arange(T) // vt, np.arange(Hg) // vh, np.arange(Wg) // vw, indexing="ij")
    nvh, nvw = -(-Hg // vh), -(-Wg // vw)
    vox = ((t * nvh + h) * nvw + w).reshape(-1)
    # the most common component of each voxel, and how many tokens differ from it
    off = 0
    for v in np.unique(vox):
        members = grid.reshape(-1)[vox == v]
        off += members.size - np.bincount(members).max()
    # without random tokens every voxel is constant; with them, about rand_frac of the tokens
    # (minus the ~1/components that draw the voxel's own component) differ
    if cfg.rand_frac == 0:
        assert off == 0
    else:
        expect = cfg.rand_frac * (1 - 1 / cfg.components) * cfg.N
        assert abs(off - expect) < 0.1 * expect


def test_head_inputs_are_seeded_bf16_exact_and_independent_per_head():
    cfg = I.CONFIGS["small"]
    a = I.head_inputs(cfg, 0, 1)
    b = I.head_inputs(cfg, 0, 1)
    c = I.head_inputs(cfg, 0, 2)
    for key in ("q", "k", "v", "uq", "uk"):
        np.testing.assert_array_equal(a[key], b[key])
        assert not np.array_equal(a[key], c[key])
    for key in ("q", "k", "v"):
        assert a[key].dtype == np.float32 and a[key].shape == (cfg.N, cfg.d)
        np.testing.assert_array_equal(I.round_to_bf16(a[key]), a[key])
    assert a["uq"].shape == (cfg.nQ,) and a["uk"].shape == (cfg.nK,)
    assert (a["uq"] >= 0).all() and (a["uq"] < 1).all()
    # V is standard normal, Q and K sit on mixture centres with noise sigma
    assert abs(a["v"].mean()) < 0.01 and abs(a["v"].std() - 1) < 0.01
    tiny = I.head_inputs(I.CONFIGS["tiny"], 0, 0)
    assert not np.array_equal(I.round_to_bf16(tiny["q"]), tiny["q"])    # the float32 shape stays float32


def test_warm_sequence_drift_follows_its_recipe():
    cfg = I.CONFIGS["wan720p_warm"]
    small = I.LayerConfig(**{**cfg.__dict__, "grid": (3, 10, 16)})
    s0 = I.head_inputs(small, 0, 0, 0)
    s3 = I.head_inputs(small, 0, 0, 3)
    # Q_s - Q_0 = drift * s * eps with eps ~ N(0, 1), up to bf16 rounding of both ends
    dq = (s3["q"] - s0["q"]) / (small.drift * 3)
    assert abs(dq.std() - 1) < 0.05 and abs(dq.mean()) < 0.02
    assert not np.array_equal(s0["v"], s3["v"])                          # V redrawn each step
    assert not np.array_equal(s0["uq"], s3["uq"])


def test_random_labels_and_weights_edge_case_generators():
    lab = I.random_labels(5000, 40, 7, empty_fraction=0.5)
    assert lab.dtype == np.int32 and lab.min() >= 0 and lab.max() < 40
    assert np.unique(lab).size == 20
    np.testing.assert_array_equal(lab, I.random_labels(5000, 40, 7, empty_fraction=0.5))
    w = I.random_weights(16, 64, 3)
    assert w.dtype == np.float32 and (w > 0).all()
    assert (w == np.float32(0.25)).mean() > 0.1                            # many exact ties
