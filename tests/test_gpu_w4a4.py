"""W4A4 (MX_A_E2M1_E8M0_1X32 = 3 with MX_B_E2M1_E8M0_1X32, kind::mxf4)
against the fp64 oracle (a_fmt 3 = the packed e2m1 activation operand), within
|y_gpu - y| <= 2^-8 |y| + 1e-5 T; and mx_quant_act's e2m1 activation codes
bit-exact against oracle.quant_act_e2m1.  Tile widths 240 / 256, 128- and
256-row tiles, ragged M / N, K a multiple of 128 but not of 256 (a last stage
with one scale chunk), several tiles per CTA."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import Case

pytestmark = pytest.mark.gpu
A_E2M1, B_E2M1 = 3, 1
NONE, BIAS, GELU, SWIGLU = 0, 1, 2, 3


def test_quant_act_e2m1_bit_exact(mx):
    x = synth.bf16_matrix(16000, 37, 1024, 1.0)
    x[3, 64:96] = 0
    codes = torch.empty(37, 512, dtype=torch.uint8, device="cuda")
    scales = torch.empty(37, 32, dtype=torch.uint8, device="cuda")
    mx.mx_quant_act(x.cuda(), codes, scales, fmt=A_E2M1)
    torch.cuda.synchronize()
    c_ref, s_ref = oracle.quant_act_e2m1(x)
    assert np.array_equal(codes.cpu().numpy(), c_ref) and np.array_equal(scales.cpu().numpy(), s_ref)


@pytest.mark.parametrize("epi", [NONE, BIAS, GELU, SWIGLU])
@pytest.mark.parametrize("M,N,K", [(200, 544, 640), (300, 1024, 1024), (65, 640, 384), (600, 480, 256)])
@pytest.mark.parametrize("block_n,block_m,ctas", [(0, 0, 0), (256, 128, 3), (240, 256, 2)])
def test_w4a4_gemm(mx, epi, M, N, K, block_n, block_m, ctas):
    if epi == SWIGLU and N % 64:
        pytest.skip("SwiGLU needs N % 64 == 0")
    c = Case(M, N, K, A_E2M1, B_E2M1, epi, seed=16100 + M + K + epi)
    y = c.run_gpu(mx, block_n=block_n, splits=1, max_ctas=ctas, block_m=block_m)
    assert c.last_plan["kernel"] == "tile"
    c.check(y, f"w4a4 M={M} N={N} K={K} epi={epi}")


def test_w4a4_decode_sized_m_uses_the_tile_kernel(mx):
    c = Case(16, 1024, 2048, A_E2M1, B_E2M1, SWIGLU, seed=16200)
    y = c.run_gpu(mx)
    assert c.last_plan["kernel"] == "tile"
    c.check(y, "w4a4 M=16")
