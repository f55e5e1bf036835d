"""The warm-start denoising sequence at the Wan-2.1-720p shape, in the launch configuration the
benchmark times (all 40 heads in one layer call).  The centroid cache is described in the paper's
section 4.3 (Fig. 7(a)).  Step 0 is a cold layer: k-means++ seeding, then 5 Lloyd iterations.  Step 1
(Q_1 = Q_0 + 0.05*eps, likewise K, V redrawn) starts both k-means from step 0's centroids and runs
2 iterations.  On three sampled heads and 384 sampled rows, every stage of the warm layer is checked
against the oracle, given the GPU's own upstream results.  The warm k-means is also checked against
the oracle's warm k-means from the same centroids: the labels must agree except at near-ties."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import pool_layer_inputs, require_gpu
from tests.test_layer import check_head, run_layer


@pytest.mark.gpu
def test_warm_step_at_wan_shape(oracle):
    svg2 = require_gpu()
    cfg = I.CONFIGS["wan720p_warm"]
    warm_cfg = I.LayerConfig(**{**cfg.__dict__, "iters": cfg.warm_iters})
    top_p = cfg.top_p[0]
    d0 = pool_layer_inputs(cfg, range(cfg.H), 0)
    r0 = run_layer(svg2, cfg, d0, top_p)
    del d0
    d1 = pool_layer_inputs(cfg, range(cfg.H), 1)
    cq, ck = torch.from_numpy(r0["cq"]).cuda(), torch.from_numpy(r0["ck"]).cuda()
    r1 = run_layer(svg2, warm_cfg, d1, top_p, init=svg2.SVG2_INIT_GIVEN, cq=cq, ck=ck)
    rng = np.random.default_rng(cfg.cfg_id)
    for h in (0, cfg.H // 2, cfg.H - 1):
        rows = np.sort(rng.choice(cfg.N, 384, replace=False))
        st = check_head(oracle, warm_cfg, d1, r1, h, top_p, rows)
        agree = {}
        for role, k in (("q", cfg.nQ), ("k", cfg.nK)):
            C0 = r0["c" + role][0, h].astype(np.float64)
            _, lab, _ = oracle.lloyd(d1[role][0, h], C0, warm_cfg.iters)
            agree[role] = float((r1["labels_" + role][0, h] == lab).mean())
            assert agree[role] >= 0.99, (h, role, agree[role])
        print(f"wan720p warm step 1, head {h}: {st}; label agreement with the oracle's warm k-means {agree}")
