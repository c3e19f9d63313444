"""MX_EPI_SWIGLU_MXQ: the SwiGLU GEMM whose bf16 result is handed on as e4m3
codes + 1 x 32 E8M0 scales (out = codes [M, N/2], then scales [M, N/64]), the
sly README's fused silu_mul_quant producer.

Parity, in the precision that decides (the codes are integers decided on the
kernel's own bf16 SwiGLU value):
  * deterministic plans (decode cluster split, whole tiles; tile kernel): the
    codes and scales equal, bit for bit, the oracle's 1 x 32 quantisation of
    the bf16 output of the same plan run with MX_EPI_SWIGLU, and the oracle's
    own producer (gemm_swiglu_mxq) wherever its bf16 block equals the kernel's;
  * every plan (stream-K too, whose fp32 atomics make y depend on arrival
    order): dequantised codes x scales within the GEMM tolerance of the fp64
    oracle plus one bf16 rounding and half an e4m3 step at the block scale.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import Case, to_dev

pytestmark = pytest.mark.gpu
SWIGLU, MXQ = 3, 5
E8, E2 = 0, 1


def run(mx, c, epi, ws="full", **tune):
    a, sa = to_dev(c.a_codes), to_dev(c.a_scales)
    b, sb = to_dev(c.b_codes), to_dev(c.b_scales)
    M, N, K = c.M, c.N, c.K
    if epi == MXQ:
        out = torch.full((M * N // 2 + M * N // 64 + 64,), 0xEE, dtype=torch.uint8, device="cuda")
    else:
        out = torch.empty((M, N // 2), dtype=torch.bfloat16, device="cuda")
    mx.mx_set_tuning(tune.get("block_n", 0), tune.get("splits", 0), 0, tune.get("block_m", 0))
    mx.mx_set_decode_tuning(tune.get("decode", 0), 0, 0, 0, tune.get("split", 0), tune.get("cluster", 0))
    try:
        wsb = mx.workspace(M, N, K, c.a_fmt, c.b_fmt, epi) if ws == "full" else mx.workspace()
        plan = mx.mx_gemm_plan_info(M, N, K, c.a_fmt, c.b_fmt, epi, wsb.numel())
        mx.mx_gemm(a, sa, c.a_fmt, b, sb, c.b_fmt, None if c.bias is None else c.bias.cuda(), epi, out, M, N, K, wsb)
    finally:
        mx.mx_set_tuning(0, 0)
        mx.mx_set_decode_tuning(0, 0, 0, 0, 0, 0)
    torch.cuda.synchronize()
    assert mx.mx_workspace_status(wsb) == 0
    if epi == MXQ:
        o = out.cpu().numpy()
        codes = o[:M * N // 2].reshape(M, N // 2)
        scales = o[M * N // 2:M * N // 2 + M * N // 64].reshape(M, N // 64)
        assert (o[M * N // 2 + M * N // 64:] == 0xEE).all(), "write past the scales"
        return codes, scales, plan
    return out.cpu().contiguous().view(torch.int16).numpy().view(np.uint16), plan


DETERMINISTIC = [
    ("decode-cluster", dict(decode=1, split=1, cluster=4), "min"),
    ("decode-cluster8", dict(decode=1, split=1, cluster=8), "min"),
    ("decode-whole", dict(decode=1, split=3), "min"),
    ("tile", dict(decode=-1, block_n=256, splits=1), "full"),
]


@pytest.mark.parametrize("name,tune,ws", DETERMINISTIC)
@pytest.mark.parametrize("M", [1, 16, 33, 64])
@pytest.mark.parametrize("b_fmt", [E8, E2])
def test_mxq_equals_quantised_swiglu_output(mx, name, tune, ws, M, b_fmt):
    N, K = 640, 1024
    c = Case(M, N, K, 0, b_fmt, SWIGLU, seed=15000 + M + b_fmt)
    y_bits, plan_s = run(mx, c, SWIGLU, ws=ws, **tune)
    codes, scales, plan_q = run(mx, c, MXQ, ws=ws, **tune)
    c_ref, s_ref = oracle.quant_act_e8m0(y_bits)
    assert np.array_equal(codes, c_ref) and np.array_equal(scales, s_ref), (name, plan_q)
    # the oracle's producer, on every block whose bf16 values the kernel matched
    yb, c_or, s_or, _, _ = oracle.gemm_swiglu_mxq(c.a_codes, c.a_scales, 0, c.b_codes, c.b_scales, b_fmt, c.bias,
                                                  M, N, K)
    same = (yb.reshape(M, N // 64, 32) == y_bits.reshape(M, N // 64, 32)).all(-1)
    assert same.mean() > 0.9, "bf16 SwiGLU output differs from the oracle's in too many blocks"
    assert np.array_equal(scales[same], s_or[same])
    assert np.array_equal(codes.reshape(M, N // 64, 32)[same], c_or.reshape(M, N // 64, 32)[same])


@pytest.mark.parametrize("name,tune,ws", DETERMINISTIC + [("decode-streamk", dict(decode=1, split=2), "full")])
@pytest.mark.parametrize("M", [1, 40, 64, 300])
def test_mxq_against_oracle(mx, name, tune, ws, M):
    if name.startswith("decode") and M > 64:
        pytest.skip("decode kernels take M <= 64")
    N, K = 640, 1024
    c = Case(M, N, K, 0, E2, SWIGLU, seed=15100 + M)
    codes, scales, plan = run(mx, c, MXQ, ws=ws, **tune)
    y, t = c.ref()
    scale = np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=1)
    deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy() * scale
    # GEMM tolerance, one bf16 rounding, half an e4m3 step (2^-4 relative for
    # normal codes, 2^-10 of the block scale for subnormal ones)
    bound = (2.0 ** -8 + 2.0 ** -9 + 2.0 ** -4) * np.abs(y) + 1e-5 * t + 2.0 ** -10 * scale
    assert (np.abs(deq - y) <= bound).all(), (name, plan)
