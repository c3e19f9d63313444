"""mx_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Callers with a fixed memory arena, or behind a C plugin interface without a
device allocator, cannot give mx_gemm its workspace; this
entry point uses scratch that lives in the library instead.  The test calls it
through the C ABI twice in a row and checks each result against mx_gemm's on
the same inputs, with the acceptance bound the other GEMM tests use.  The file
name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import Case, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(lib, c, a, sa, b, sb, bias, out):
    P = ctypes.c_void_p
    return lib.mx_gemm_noalloc(P(a.data_ptr()), P(sa.data_ptr()), c.a_fmt, P(b.data_ptr()), P(sb.data_ptr()),
                               c.b_fmt, None if bias is None else P(bias.data_ptr()), c.epi, P(out.data_ptr()),
                               c.M, c.N, c.K, P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K,b_fmt,epi", [(16, 256, 512, 0, 1), (40, 512, 2048, 0, 2), (8, 256, 1024, 1, 3)])
def test_noalloc_matches_mx_gemm_twice(mx, M, N, K, b_fmt, epi):
    lib = mx.load()
    c = Case(M, N, K, 0, b_fmt, epi, seed=300 + M)
    a, sa, b, sb = to_dev(c.a_codes), to_dev(c.a_scales), to_dev(c.b_codes), to_dev(c.b_scales)
    bias = None if c.bias is None else c.bias.cuda()
    ref_out = mx.out_buffer(M, N, epi)
    ws = mx.workspace()
    mx.mx_gemm(a, sa, c.a_fmt, b, sb, c.b_fmt, bias, epi, ref_out, M, N, K, ws)
    torch.cuda.synchronize()
    y_ref = ref_out.float().cpu().numpy().astype(np.float64)
    _, t = c.ref()
    for call in range(2):
        out = torch.full_like(ref_out, float("nan"))
        assert _noalloc(lib, c, a, sa, b, sb, bias, out) == 0, f"call {call}"
        torch.cuda.synchronize()
        y = out.float().cpu().numpy().astype(np.float64)
        ok = oracle.within_tolerance(y, y_ref, t)
        assert ok.all(), f"call {call}: {(~ok).sum()} outputs differ from mx_gemm beyond the bound"
        c.check(y, f"noalloc call {call}")


def test_noalloc_rejects_bad_arguments(mx):
    lib = mx.load()
    assert lib.mx_gemm_noalloc(None, None, 0, None, None, 0, None, 0, None, 16, 256, 512, None) == mx.MX_ERR_NULL


def test_bf16_act_noalloc(mx):
    # bf16 activations (MX_A_BF16_E8M0_1X32): the fused decode path needs no
    # scratch; outside it the shared scratch would be overwritten by
    # concurrent calls, so the call refuses
    M, N, K = 16, 256, 512
    c = Case(M, N, K, 0, 0, 1, seed=82)
    b = torch.from_numpy(c.b_codes).cuda()
    sb = torch.from_numpy(c.b_scales).cuda()
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    mx.mx_gemm_noalloc(c.x.cuda(), None, 2, b, sb, 0, c.bias.cuda(), 1, out, M, N, K)
    torch.cuda.synchronize()
    c.check(out.float().cpu().numpy().astype(np.float64), "noalloc fused")
    M2 = 200
    c2 = Case(M2, N, K, 0, 0, 1, seed=83)
    out2 = torch.empty(M2, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MxError) as err:
        mx.mx_gemm_noalloc(c2.x.cuda(), None, 2, torch.from_numpy(c2.b_codes).cuda(),
                           torch.from_numpy(c2.b_scales).cuda(), 0, c2.bias.cuda(), 1, out2, M2, N, K)
    assert err.value.status == mx.MX_ERR_WORKSPACE
