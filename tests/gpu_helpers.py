"""Shared helpers of the GPU parity tests: device checks and numpy <-> torch moves."""
import os

import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import build as B


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if major != 10:
        pytest.skip("needs an sm_100 device")
    B.build()
    from sparse_attention_video_head_b200 import svg2
    svg2.lib()
    return svg2


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    """float32 values (bf16-exact or not) -> device bf16, rounded to nearest even."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def near_tie(d1: np.ndarray, d2: np.ndarray, rel: float = 1e-4) -> np.ndarray:
    """Tokens whose two smallest oracle distances are within `rel` of the smallest."""
    return (d2 - d1) < rel * np.maximum(d1, 1e-30)


def pool_layer_inputs(cfg, heads, step=0, procs=None):
    """Generate [1, len(heads), N, d] inputs in parallel processes (spawned, so safe after CUDA init)."""
    import multiprocessing as mp
    from sparse_attention_video_head_b200 import inputs as I
    heads = list(heads)
    procs = procs or max(1, min(len(heads), len(os.sched_getaffinity(0))))
    if procs == 1 or len(heads) == 1:
        return I.layer_inputs(cfg, step, heads)
    ctx = mp.get_context("spawn")
    with ctx.Pool(procs) as pool:
        parts = pool.starmap(I.head_inputs, [(cfg, 0, h, step) for h in heads])
    return {k: np.stack([p[k] for p in parts])[None] for k in parts[0]}
