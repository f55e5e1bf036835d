"""Permutation kernels vs the oracle, bit-exact (Method (2): stable counting sort, row gathers and
the inverse permutation)."""
import numpy as np
import pytest
import torch

from sparse_attention_video_head_b200 import inputs as I
from tests.gpu_helpers import bf16_dev, host, require_gpu, to_dev

CASES = [  # (B, H, N, k, empty fraction)
    (1, 1, 1, 1, 0.0),
    (1, 2, 1000, 37, 0.3),
    (1, 8, 12480, 256, 0.2),
    (1, 3, 4096, 1024, 0.5),
    (2, 2, 5000, 3, 0.0),
    (1, 2, 75600, 500, 0.0),
]


def _labels(B, H, N, k, empty, seed=0):
    return np.stack([np.stack([I.random_labels(N, k, seed + 97 * b + h, empty) for h in range(H)])
                     for b in range(B)])


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,k,empty", CASES)
def test_sort_is_bit_exact(oracle, B, H, N, k, empty):
    svg2 = require_gpu()
    lab = _labels(B, H, N, k, empty)
    perm = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
    off = torch.empty(B, H, k + 1, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, H, k, dtype=torch.int32, device="cuda")
    ws = svg2.workspace(B, H, max(N, k), 128, min(k, max(N, k)), min(k, max(N, k)))
    svg2.svg2_sort(to_dev(lab), k, perm, off, cnt, ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    for b in range(B):
        for h in range(H):
            p_ref, o_ref = oracle.permute(lab[b, h], k)
            assert np.array_equal(host(perm)[b, h], p_ref)
            assert np.array_equal(host(off)[b, h], o_ref)
            assert np.array_equal(host(cnt)[b, h], np.diff(o_ref))


@pytest.mark.gpu
@pytest.mark.parametrize("f32", [False, True])
def test_gather_and_unpermute_are_bit_exact(oracle, f32):
    svg2 = require_gpu()
    B, H, N, d, k = 1, 3, 3001, 128, 40
    rng = np.random.default_rng(3)
    X = rng.standard_normal((B, H, N, d), dtype=np.float32)
    lab = _labels(B, H, N, k, 0.1, 5)
    Xd = to_dev(X) if f32 else bf16_dev(X)
    Xp = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    perm = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
    off = torch.empty(B, H, k + 1, dtype=torch.int32, device="cuda")
    ws = svg2.workspace(B, H, N, d, k, k)
    svg2.svg2_permute(Xd, to_dev(lab), k, Xp, perm, off, None, ws)
    back = torch.empty_like(Xp)
    svg2.svg2_unpermute(Xp, perm, back)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    Xb = Xd.to(torch.bfloat16)   # torch rounds float32 to bf16 to nearest even, as the kernel must
    for h in range(H):
        p_ref, _ = oracle.permute(lab[0, h], k)
        assert torch.equal(Xp[0, h].cpu(), Xb[0, h].cpu()[torch.from_numpy(p_ref).long()])
    assert torch.equal(back, Xb)


@pytest.mark.gpu
def test_out_of_range_label_is_reported_not_faulted():
    svg2 = require_gpu()
    lab = np.zeros((1, 1, 100), np.int32)
    lab[0, 0, 17] = 9   # k = 4: invalid
    perm = torch.empty(1, 1, 100, dtype=torch.int32, device="cuda")
    off = torch.empty(1, 1, 5, dtype=torch.int32, device="cuda")
    ws = svg2.workspace(1, 1, 100, 128, 4, 4)
    svg2.svg2_sort(to_dev(lab), 4, perm, off, None, ws)
    code, where, info = svg2.svg2_check_status(ws)
    assert code == 6 and info[1] == 17
    assert svg2.svg2_check_status(ws)[0] == 0   # reading clears it
