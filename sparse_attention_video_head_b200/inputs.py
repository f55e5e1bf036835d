"""Seeded synthetic inputs shaped like the DiT attention layers that Sparse VideoGen2 accelerates.

This module is shared by the tests, the benchmark and the oracle checks.  It only draws
numbers; it contains none of the method's arithmetic (no clustering, scoring, selection,
permutation or attention).

The pages measure SVG2 on real Wan 2.1 / HunyuanVideo activations ("Sparse VideoGen2" wiki
summary, Results; Table 1).  Those models and prompts are not available, so per (batch, head)
Q and K are drawn from a Gaussian mixture whose component is chosen per token by a seeded
piecewise-constant map over 3D voxels of the (t, h, w) token grid, which gives clusters that are
semantically tight but spatially scattered, the situation the pages' semantic-aware permutation
targets ("Sparse VideoGen2" wiki summary, Key claims, section 4.1).  V ~ N(0, 1).

Token flatten order: n = (t * Hgrid + h) * Wgrid + w.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import numpy as np

# Role codes that enter the seed; one independent stream per (config, batch, head, role, step).
ROLE_MAP, ROLE_Q, ROLE_K, ROLE_V, ROLE_UQ, ROLE_UK, ROLE_EPS_Q, ROLE_EPS_K, ROLE_RANDTOK = range(9)


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    cfg_id: int
    B: int
    H: int
    grid: Tuple[int, int, int]      # (T, Hgrid, Wgrid)
    d: int
    dtype: str                      # "bf16" or "f32"
    components: int
    sigma: float
    voxel: Tuple[int, int, int]     # voxel edge in tokens along (t, h, w)
    rand_frac: float                # fraction of tokens given a uniformly random component
    nQ: int
    nK: int
    iters: int
    top_p: Tuple[float, ...]
    # denoising-sequence settings (warm-start config only)
    steps: int = 1
    warm_iters: int = 0
    drift: float = 0.0

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


CONFIGS: Dict[str, LayerConfig] = {
    # 1 head, 4x32x32 tokens, d=64, fp32; 24 components over 4x4x4 voxels; 16/32 clusters, 10 iterations.
    "tiny": LayerConfig("tiny", 0, 1, 1, (4, 32, 32), 64, "f32", 24, 0.3, (4, 4, 4), 0.0,
                        16, 32, 10, (0.9,)),
    # 8 heads, 8x30x52 tokens, d=128, bf16; 64 components; 64/256 clusters, 8 iterations.
    "small": LayerConfig("small", 1, 1, 8, (8, 30, 52), 128, "bf16", 64, 0.25, (4, 4, 4), 0.0,
                         64, 256, 8, (0.9,)),
    # Wan-2.1-14B 720p layer: 40 heads, 21x45x80 tokens; 200 components, 3x5x5 voxels + 10% random tokens.
    "wan720p": LayerConfig("wan720p", 2, 1, 40, (21, 45, 80), 128, "bf16", 200, 0.2, (3, 5, 5), 0.1,
                           100, 500, 5, (0.8, 0.9, 0.95)),
    # HunyuanVideo-13B 720p layer: 24 heads, 33x45x80 tokens; 400 components.
    "hunyuan720p": LayerConfig("hunyuan720p", 3, 1, 24, (33, 45, 80), 128, "bf16", 400, 0.2, (3, 5, 5), 0.1,
                               400, 1000, 5, (0.8, 0.9, 0.95)),
    # Warm-start denoising sequence on the Wan-720p shapes: 10 steps, 2 warm iterations per step.
    "wan720p_warm": LayerConfig("wan720p_warm", 4, 1, 40, (21, 45, 80), 128, "bf16", 200, 0.2, (3, 5, 5), 0.1,
                                100, 500, 5, (0.9,), steps=10, warm_iters=2, drift=0.05),
}


def _rng(cfg: LayerConfig, b: int, h: int, role: int, step: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.cfg_id, b, h, role, step])))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even) and return them as float32."""
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    if not np.isfinite(x).all():
        raise ValueError("round_to_bf16 expects finite values")
    bits = x.view(np.uint32)
    lsb = bits >> np.uint32(16)
    lsb &= np.uint32(1)
    lsb += np.uint32(0x7FFF)
    bits += lsb
    bits &= np.uint32(0xFFFF0000)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-exact (uint16 view for upload)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def component_map(cfg: LayerConfig, b: int, h: int) -> np.ndarray:
    """Per-token component index, piecewise constant over voxels, plus optional random tokens."""
    T, Hg, Wg = cfg.grid
    vt, vh, vw = cfg.voxel
    nvt, nvh, nvw = -(-T // vt), -(-Hg // vh), -(-Wg // vw)
    rng = _rng(cfg, b, h, ROLE_MAP)
    vox = rng.integers(0, cfg.components, size=(nvt, nvh, nvw))
    ti = np.arange(T) // vt
    hi = np.arange(Hg) // vh
    wi = np.arange(Wg) // vw
    comp = vox[ti[:, None, None], hi[None, :, None], wi[None, None, :]].reshape(-1)
    if cfg.rand_frac > 0:
        r2 = _rng(cfg, b, h, ROLE_RANDTOK)
        n_rand = int(round(cfg.rand_frac * comp.size))
        idx = r2.choice(comp.size, size=n_rand, replace=False)
        comp = comp.copy()
        comp[idx] = r2.integers(0, cfg.components, size=n_rand)
    return comp.astype(np.int64)


def _mixture(cfg: LayerConfig, b: int, h: int, role: int, comp: np.ndarray) -> np.ndarray:
    rng = _rng(cfg, b, h, role)
    centres = rng.standard_normal((cfg.components, cfg.d), dtype=np.float32)
    noise = rng.standard_normal((comp.size, cfg.d), dtype=np.float32)
    return centres[comp] + np.float32(cfg.sigma) * noise


def head_inputs(cfg: LayerConfig, b: int, h: int, step: int = 0) -> Dict[str, np.ndarray]:
    """Q, K, V [N, d] float32 (bf16-exact for bf16 configs) and the k-means++ uniforms for one head.

    For the warm-start sequence, step s uses Q_s = Q_0 + drift * s * eps_s (fresh eps_s), likewise
    K_s, and a freshly drawn V_s.
    """
    comp = component_map(cfg, b, h)
    q = _mixture(cfg, b, h, ROLE_Q, comp)
    k = _mixture(cfg, b, h, ROLE_K, comp)
    if step > 0:
        eq = _rng(cfg, b, h, ROLE_EPS_Q, step).standard_normal(q.shape, dtype=np.float32)
        ek = _rng(cfg, b, h, ROLE_EPS_K, step).standard_normal(k.shape, dtype=np.float32)
        q = q + np.float32(cfg.drift * step) * eq
        k = k + np.float32(cfg.drift * step) * ek
    v = _rng(cfg, b, h, ROLE_V, step).standard_normal((cfg.N, cfg.d), dtype=np.float32)
    if cfg.dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
    uq = _rng(cfg, b, h, ROLE_UQ, step).random(cfg.nQ)
    uk = _rng(cfg, b, h, ROLE_UK, step).random(cfg.nK)
    return {"q": q, "k": k, "v": v, "uq": uq, "uk": uk}


def layer_inputs(cfg: LayerConfig, step: int = 0, heads=None) -> Dict[str, np.ndarray]:
    """Stack head_inputs over (b, h) into [B, H, N, d] / [B, H, k] arrays (heads: optional subset)."""
    hs = list(range(cfg.H)) if heads is None else list(heads)
    out = {key: [] for key in ("q", "k", "v", "uq", "uk")}
    for b in range(cfg.B):
        per = {key: [] for key in out}
        for h in hs:
            hi = head_inputs(cfg, b, h, step)
            for key in out:
                per[key].append(hi[key])
        for key in out:
            out[key].append(np.stack(per[key]))
    return {key: np.stack(v) for key, v in out.items()}


def random_labels(n: int, k: int, seed: int, empty_fraction: float = 0.0) -> np.ndarray:
    """Seeded labels in [0, k) with a chosen fraction of clusters left empty (edge-case inputs)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    keep = np.arange(k)
    if empty_fraction > 0:
        keep = np.sort(rng.choice(k, size=max(1, int(round(k * (1 - empty_fraction)))), replace=False))
    return keep[rng.integers(0, keep.size, size=n)].astype(np.int32)


def random_weights(rows: int, cols: int, seed: int) -> np.ndarray:
    """Seeded positive float32 weights with many exact ties (edge-case inputs for selection)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    w = rng.gamma(0.5, 1.0, size=(rows, cols)).astype(np.float32)
    tie = rng.random((rows, cols)) < 0.2
    w[tie] = np.float32(0.25)
    return w
