"""The in-place residual epilogue (MX_EPI_RESIDUAL: out = out + (acc + bias),
the ViT page's `vt_add` update x += y + b fused into the GEMM) against the
oracle's gemm_residual, element by element within
|y_gpu - y| <= 2^-8 |y| + 1e-5 T, on every kernel and plan: the decode kernel
(cluster, whole tiles, stream-K), the tile
kernel with 128- and 256-row tiles, K split through the workspace or over a
cluster, and the CTA-pair kernel; with and without a bias; ragged M and N."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import Case, guarded, guards_intact, to_dev

pytestmark = pytest.mark.gpu
RESIDUAL = 4  # MX_EPI_RESIDUAL


def run_residual(mx, c, res, bias, ws="full", **tune):
    a, sa = to_dev(c.a_codes), to_dev(c.a_scales)
    b, sb = to_dev(c.b_codes), to_dev(c.b_scales)
    full, out = guarded(c.M * c.N)
    out.copy_(res.reshape(-1).cuda())
    mx.mx_set_tuning(tune.get("block_n", 0), tune.get("splits", 0), tune.get("max_ctas", 0), tune.get("block_m", 0))
    mx.mx_set_decode_tuning(tune.get("decode", 0), tune.get("decode_ctas", 0), 0, 0, tune.get("split", 0),
                            tune.get("cluster", 0))
    try:
        wsb = mx.workspace(c.M, c.N, c.K, c.a_fmt, c.b_fmt, RESIDUAL) if ws == "full" else mx.workspace()
        plan = mx.mx_gemm_plan_info(c.M, c.N, c.K, c.a_fmt, c.b_fmt, RESIDUAL, wsb.numel())
        mx.mx_gemm(a, sa, c.a_fmt, b, sb, c.b_fmt, None if bias is None else bias.cuda(), RESIDUAL, out,
                   c.M, c.N, c.K, wsb)
    finally:
        mx.mx_set_tuning(0, 0)
        mx.mx_set_decode_tuning(0, 0, 0, 0, 0, 0)
    torch.cuda.synchronize()
    assert mx.mx_workspace_status(wsb) == 0
    assert guards_intact(full)
    return out.view(c.M, c.N).float().cpu().numpy().astype(np.float64), plan


PLANS = [
    ("decode-cluster", dict(decode=1, split=1, cluster=4), "min"),
    ("decode-whole", dict(decode=1, split=3), "min"),
    ("decode-streamk", dict(decode=1, split=2), "full"),
    ("tile-128", dict(decode=-1, block_n=240, splits=1, block_m=128), "full"),
    ("tile-256", dict(decode=-1, block_n=240, splits=1, block_m=256), "full"),
    ("tile-splitk-ws", dict(decode=-1, block_n=128, splits=4), "full"),
    ("tile-splitk-cluster", dict(decode=-1, block_n=128, splits=4), "min"),
    ("pair", dict(decode=-1, block_m=2), "full"),
]


@pytest.mark.parametrize("name,tune,ws", PLANS)
@pytest.mark.parametrize("M", [1, 17, 64, 300])
@pytest.mark.parametrize("with_bias", [True, False])
def test_residual_epilogue(mx, name, tune, ws, M, with_bias):
    if name.startswith("decode") and M > 64:
        pytest.skip("decode kernels take M <= 64")
    N, K = 544, 640
    c = Case(M, N, K, 0, 0, 1, seed=13000 + M + (7 if with_bias else 0))
    bias = c.bias if with_bias else None
    res = synth.bf16_matrix(13100 + M, M, N, 1.0)
    y, plan = run_residual(mx, c, res, bias, ws=ws, **tune)
    y_ref, t = oracle.gemm_residual(c.a_codes, c.a_scales, 0, c.b_codes, c.b_scales, 0, bias, res, M, N, K)
    ok = oracle.within_tolerance(y, y_ref, t)
    assert ok.all(), f"{name} M={M}: {(~ok).sum()} outside tolerance (plan {plan})"
