"""Head-sharded layer through the library (the multi-GPU partition, run here as separate calls on
one GPU): svg2_layer on each rank's contiguous block of heads, shard.head_range(H, 2, r), must give
exactly the bits of the unsharded layer for those heads.  Every (b, h) plane is an independent
problem (Method (1)-(4) act per head), so no exchange is needed and the partition is exact."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from sparse_attention_video_head_b200.shard import head_range
from tests.gpu_helpers import pool_layer_inputs, require_gpu
from tests.test_layer import run_layer


def _slice(data, h0, h1):
    return {key: np.ascontiguousarray(val[:, h0:h1]) for key, val in data.items()}


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name,heads,world", [("small", range(8), 2), ("small", range(7), 3),
                                                  ("wan720p", range(4), 2)])
def test_head_sharded_layer_equals_unsharded(cfg_name, heads, world):
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    data = pool_layer_inputs(cfg, heads)
    full = run_layer(svg2, cfg, data, 0.9)
    H = len(heads)
    for r in range(world):
        h0, h1 = head_range(H, world, r)
        part = run_layer(svg2, cfg, _slice(data, h0, h1), 0.9)
        for key in ("o", "cq", "ck", "labels_q", "labels_k", "mask", "perm_q", "perm_k"):
            np.testing.assert_array_equal(part[key], full[key][:, h0:h1], err_msg=f"rank {r} {key}")
