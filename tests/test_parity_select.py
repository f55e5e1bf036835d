"""Selection kernels vs the oracle (section 4.2, Eq. 1-2): top-p masks bit-exact from identical
weights; weights from identical centroids within 1e-6 relative."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import host, require_gpu, to_dev


def _check_ell(mask, sel_count, sel_idx, stream_len, count_k):
    for i in range(mask.shape[0]):
        kept = np.nonzero(mask[i])[0]
        assert sel_count[i] == kept.size
        assert np.array_equal(sel_idx[i, :kept.size], kept)
        assert stream_len[i] == count_k[kept].sum()


@pytest.mark.gpu
@pytest.mark.parametrize("nK", [1, 7, 500, 1000, 1024])
def test_topp_from_weights_is_bit_exact(oracle, nK):
    svg2 = require_gpu()
    B, H, nQ = 1, 3, 17
    rng = np.random.default_rng(nK)
    w = np.stack([I.random_weights(nQ, nK, 10 * nK + h) for h in range(H)])[None]
    count_k = rng.integers(0, 40, (B, H, nK)).astype(np.int32)
    count_k[..., 0] = 5
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for p in [1e-6, 0.3, 0.5, 0.8, 0.9, 0.95, 0.999, 1.0]:
        mask = torch.empty(B, H, nQ, nK, dtype=torch.uint8, device="cuda")
        sc = torch.empty(B, H, nQ, dtype=torch.int32, device="cuda")
        si = torch.empty(B, H, nQ, nK, dtype=torch.int32, device="cuda")
        sl = torch.empty(B, H, nQ, dtype=torch.int32, device="cuda")
        svg2.svg2_select_from_weights(to_dev(w), to_dev(count_k), p, mask, sc, si, ws, sl)
        torch.cuda.synchronize()
        for h in range(H):
            ref = oracle.topp(w[0, h], count_k[0, h], p)
            assert np.array_equal(host(mask)[0, h], ref), (p, h)
            _check_ell(ref, host(sc)[0, h], host(si)[0, h], host(sl)[0, h], count_k[0, h])


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_name", ["small", "wan720p", "hunyuan720p"])
def test_weights_match_oracle_and_masks_agree(oracle, cfg_name):
    svg2 = require_gpu()
    cfg = I.CONFIGS[cfg_name]
    B, H, d = 1, 2, cfg.d
    rng = np.random.default_rng(cfg.cfg_id)
    cq = rng.standard_normal((B, H, cfg.nQ, d), dtype=np.float32)
    ck = rng.standard_normal((B, H, cfg.nK, d), dtype=np.float32)
    count_k = rng.integers(0, 300, (B, H, cfg.nK)).astype(np.int32)
    count_k[..., ::17] = 0
    scale = float(np.float32(cfg.scale))
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    W = torch.empty(B, H, cfg.nQ, cfg.nK, dtype=torch.float32, device="cuda")
    mask = torch.empty(B, H, cfg.nQ, cfg.nK, dtype=torch.uint8, device="cuda")
    sc = torch.empty(B, H, cfg.nQ, dtype=torch.int32, device="cuda")
    si = torch.empty(B, H, cfg.nQ, cfg.nK, dtype=torch.int32, device="cuda")
    sl = torch.empty(B, H, cfg.nQ, dtype=torch.int32, device="cuda")
    svg2.svg2_select(to_dev(cq), to_dev(ck), to_dev(count_k), 0.9, scale, mask, sc, si, ws, W, sl)
    torch.cuda.synchronize()
    mismatches = 0
    for h in range(H):
        w_ref = oracle.select_weights(cq[0, h], ck[0, h], count_k[0, h], scale)
        w = host(W)[0, h]
        nz = w_ref > 0
        assert np.array_equal(w == 0, ~nz)
        np.testing.assert_allclose(w[nz], w_ref[nz], rtol=1e-6)
        # the mask from the GPU's own weights is bit-exact; from the oracle's it may differ only
        # where a float32 weight rounded differently
        assert np.array_equal(host(mask)[0, h], oracle.topp(w, count_k[0, h], 0.9))
        mismatches += int((host(mask)[0, h] != oracle.topp(w_ref, count_k[0, h], 0.9)).sum())
        _check_ell(host(mask)[0, h], host(sc)[0, h], host(si)[0, h], host(sl)[0, h], count_k[0, h])
    print(f"{cfg_name}: end-to-end mask mismatches {mismatches} of {H * cfg.nQ * cfg.nK}")
    assert mismatches <= 2
