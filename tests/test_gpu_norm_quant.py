"""mx_add_rms_quant (residual add + RMSNorm + 1 x 32 E8M0 quantisation, the
sly README's fused add_rms_quant producer) against the oracle's unfused chain.
The residual written back is bit-exact; y is within one bf16 rounding of the
oracle's (the sum of squares is fp32 on the GPU and fp64 in the oracle, so a
rounding may fall on the other side of a bf16 midpoint); the codes and scales
are bit-exact against the oracle's quantisation of the kernel's own y (both
sides take the integer decisions on the same bf16 values)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("M,K", [(1, 7168), (7, 5120), (64, 2048), (300, 4096), (3, 32), (5, 96), (2, 16384)])
@pytest.mark.parametrize("eps", [1e-6, 0.0])
def test_add_rms_quant(mx, M, K, eps):
    x = synth.bf16_matrix(14000 + K, M, K, 1.0)
    r = synth.bf16_matrix(14001 + K, M, K, 1.0)
    w = synth.bf16_matrix(14002 + K, 1, K, 0.2)[0] + 1.0
    res = r.cuda().clone()
    y = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    codes = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    scales = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
    mx.mx_add_rms_quant(x.cuda(), res, w.cuda(), eps, y, codes, scales)
    torch.cuda.synchronize()
    res_ref, y_ref, _, _ = oracle.add_rms_quant(x, r, w, eps)
    assert np.array_equal(bits(res), res_ref)
    yg = oracle.bf16_bits_to_f64(bits(y))
    yr = oracle.bf16_bits_to_f64(y_ref)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(yr), 2.0 ** -126))) - 7)
    assert (np.abs(yg - yr) <= ulp).all()
    c_ref, s_ref = oracle.quant_act_e8m0(bits(y))
    assert np.array_equal(codes.cpu().numpy(), c_ref) and np.array_equal(scales.cpu().numpy(), s_ref)


def test_add_rms_quant_without_y(mx):
    M, K = 4, 1024
    x = synth.bf16_matrix(14100, M, K, 1.0)
    r = synth.bf16_matrix(14101, M, K, 1.0)
    w = synth.bf16_matrix(14102, 1, K, 0.2)[0] + 1.0
    res, codes = r.cuda().clone(), torch.empty(M, K, dtype=torch.uint8, device="cuda")
    scales = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
    y = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    mx.mx_add_rms_quant(x.cuda(), res, w.cuda(), 1e-6, y, codes, scales)
    res2, codes2 = r.cuda().clone(), torch.empty_like(codes)
    scales2 = torch.empty_like(scales)
    mx.mx_add_rms_quant(x.cuda(), res2, w.cuda(), 1e-6, None, codes2, scales2)
    torch.cuda.synchronize()
    assert torch.equal(codes, codes2) and torch.equal(scales, scales2) and torch.equal(res, res2)
