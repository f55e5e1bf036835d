"""tcgen05 building blocks on the B200: TMA 128B-swizzled tiles, SS and TS forms of tcgen05.mma,
TMEM loads and stores (the pieces the k-means assignment and the attention are built from)."""
import numpy as np
import pytest
import torch

from tests.gpu_helpers import require_gpu


@pytest.mark.gpu
@pytest.mark.parametrize("n", [64, 128, 256])
def test_tcgen05_gemm_and_tmem_operand(n):
    svg2 = require_gpu()
    rng = np.random.default_rng(n)
    A = torch.from_numpy(rng.standard_normal((128, 128), dtype=np.float32)).to(torch.bfloat16).cuda()
    Bm = torch.from_numpy(rng.standard_normal((n, 128), dtype=np.float32)).to(torch.bfloat16).cuda()
    V = torch.from_numpy(rng.standard_normal((128, 128), dtype=np.float32)).to(torch.bfloat16).cuda()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    C, O = svg2.svg2_selftest_mma(A, Bm, V, ws)
    torch.cuda.synchronize()
    svg2.raise_on_device_error(ws)
    C_ref = A.double().cpu() @ Bm.double().cpu().T
    np.testing.assert_allclose(C.cpu().numpy(), C_ref.numpy(), rtol=1e-5, atol=2e-4)
    P = torch.zeros(128, 128, dtype=torch.float64)
    P[:, :min(n, 128)] = C.cpu()[:, :min(n, 128)].to(torch.bfloat16).double()
    O_ref = P @ V.double().cpu()
    np.testing.assert_allclose(O.cpu().numpy(), O_ref.numpy(), rtol=1e-5, atol=1e-3)
