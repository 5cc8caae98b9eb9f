"""MXFP8 quantisation on the GPU (moe_mxfp8_quantize) against the oracle's definition
(oracle/mxfp8.py, after the OCP Microscaling v1.0 MXFP8 (E4M3) format): the E4M3 bytes and
the E8M0 scale bytes must be the oracle's, bit for bit."""
import numpy as np
import pytest
import torch

import expert_dispatch_fp32_b200 as M
from oracle import mxfp8

pytestmark = pytest.mark.gpu


def _rows(rows, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((rows, K), generator=g)
    # blocks over many binades, exact zeros, ties between E4M3 values, the clamp range
    x[0, :32] = 0.0
    x[1, :32] = torch.linspace(-3, 3, 32)
    x[2] *= 1e-30
    x[3] *= 1e30
    x[4, :32] = torch.tensor([448.0, 464.0, 480.0, 496.0] * 8)         # [448, 512): clamp and ties
    x[5, :32] = torch.tensor([1.0, 1.0625, 1.125, 1.1875] * 8) * 256   # halfway cases after scaling
    x[6] = torch.exp2(torch.randint(-40, 40, (K,), generator=g).float()) * torch.sign(x[6])
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,K", [(7, 64), (300, 2048), (129, 7168)])
def test_quantize_matches_the_oracle_bit_for_bit(rows, K):
    x = _rows(rows, K, seed=rows + K)
    xd = x.cuda()
    q = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, K // 32), dtype=torch.uint8, device="cuda")
    M.moe_mxfp8_quantize(xd, rows, K, q, s)
    torch.cuda.synchronize()
    qv_ref, s_ref = mxfp8.quantize_mxfp8(x.to(torch.float64).numpy(), axis=-1)
    assert np.array_equal(s.cpu().numpy().astype(np.int64) - 127, s_ref)
    qv = q.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(qv, qv_ref)
