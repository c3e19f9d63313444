"""Helpers of the GPU parity tests: seeded problems, oracle references,
guard-banded output buffers and the tolerance check."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

EPI_NEEDS_BIAS = (1, 2)
SENTINEL = 0x7FA5  # a bf16 NaN pattern no kernel writes
WS_GUARD, WS_SENTINEL = 256, 0xA5  # workspace guard bands (256 bytes keep its alignment)


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda() if dtype is None else t.to(dtype).cuda()


def guarded(numel: int, dtype=torch.bfloat16, guard: int = 64):
    """A buffer with `guard` sentinel elements on both sides; returns (full, view)."""
    full = torch.empty(numel + 2 * guard, dtype=torch.int16, device="cuda")
    full.fill_(SENTINEL if SENTINEL < 0x8000 else SENTINEL - 0x10000)
    view = full[guard:guard + numel].view(dtype)
    return full, view


def guards_intact(full: torch.Tensor, guard: int = 64) -> bool:
    h = full.cpu().numpy()
    return bool((h[:guard] == SENTINEL).all() and (h[-guard:] == SENTINEL).all())


class Case:
    """One seeded GEMM problem with its oracle reference."""

    def __init__(self, M, N, K, a_fmt, b_fmt, epi, seed=0, with_bias=True, x=None, w=None):
        self.M, self.N, self.K = M, N, K
        self.a_fmt, self.b_fmt, self.epi = a_fmt, b_fmt, epi
        xs, ws, bs = synth.problem(seed, M, N, K)
        self.x = xs if x is None else x
        self.w = ws if w is None else w
        use_bias = epi in EPI_NEEDS_BIAS or (epi == 3 and with_bias)
        self.bias = bs if use_bias else None
        self.a_codes, self.a_scales = oracle.quant_act(self.x, a_fmt)
        self.b_codes, self.b_scales = oracle.quant_weight(self.w, b_fmt)
        self.nout = N // 2 if epi == 3 else N
        self._ref = None

    def ref(self):
        if self._ref is None:
            self._ref = oracle.gemm(self.a_codes, self.a_scales, self.a_fmt, self.b_codes, self.b_scales,
                                    self.b_fmt, self.bias, self.epi, self.M, self.N, self.K)
        return self._ref

    def run_gpu(self, mx, block_n=0, splits=0, stream=None, max_ctas=0, block_m=0, ws="full", decode=0,
                decode_ctas=0, per_sm=0, split=0, cluster=0, bf16_act=False):
        """Runs the GEMM on the GPU.  ws="full" hands mx_gemm the workspace its
        fastest plan wants (K splits reduced through the workspace); ws="min"
        hands it the 256-byte minimum (K splits reduced over a cluster, or
        whole tiles); ws="codes" the workspace the plan on codes wants.  decode / decode_ctas go to mx_set_decode_tuning.
        bf16_act=True hands mx_gemm the bf16 activations themselves
        (MX_A_BF16_E8M0_1X32) instead of the oracle's codes and scales."""
        a_fmt = self.a_fmt
        if bf16_act:
            assert self.a_fmt == 0, "bf16 activations stand in for the 1x32 E8M0 codes"
            a_fmt = 2
            a = self.x.cuda()
            sa = None
        else:
            a = to_dev(self.a_codes)
            sa = to_dev(self.a_scales)
        b = to_dev(self.b_codes)
        sb = to_dev(self.b_scales)
        bias = None if self.bias is None else self.bias.cuda()
        full, out = guarded(self.M * self.nout)
        mx.mx_set_tuning(block_n, splits, max_ctas, block_m)
        mx.mx_set_decode_tuning(decode, decode_ctas, per_sm, 0, split, cluster)
        try:
            if ws == "full":
                wsb = mx.workspace(self.M, self.N, self.K, a_fmt, self.b_fmt, self.epi)
            elif ws == "codes":
                # what the plan on codes wants: with bf16 activations, no room
                # to quantise them ahead
                wsb = mx.workspace(self.M, self.N, self.K, self.a_fmt, self.b_fmt, self.epi)
            else:
                wsb = mx.workspace()
            # the workspace sits between two 256-byte guard bands of a
            # sentinel byte, checked untouched afterwards
            ws_full = torch.full((wsb.numel() + 2 * WS_GUARD,), WS_SENTINEL, dtype=torch.uint8, device="cuda")
            ws_full[WS_GUARD:WS_GUARD + wsb.numel()] = 0
            wsb = ws_full[WS_GUARD:WS_GUARD + wsb.numel()]
            plan = mx.mx_gemm_plan_info(self.M, self.N, self.K, a_fmt, self.b_fmt, self.epi, wsb.numel())
            self.last_ws = wsb
            self.last_plan = plan
            mx.mx_gemm(a, sa, a_fmt, b, sb, self.b_fmt, bias, self.epi, out, self.M, self.N, self.K, wsb,
                       stream=stream)
        finally:
            mx.mx_set_tuning(0, 0)
            mx.mx_set_decode_tuning(0, 0, 0, 0, 0, 0)
        torch.cuda.synchronize()
        assert mx.mx_workspace_status(wsb) == 0, "a bounded wait ran out"
        assert guards_intact(full), "write outside the output"
        wg = ws_full.cpu().numpy()
        assert (wg[:WS_GUARD] == WS_SENTINEL).all() and (wg[-WS_GUARD:] == WS_SENTINEL).all(), \
            "write outside the workspace"
        # everything after the 256-byte status block (arrival counters, and the
        # decode kernel's fp32 accumulators) is back to zero: the last arrival
        # of every tile reset its own
        if plan["k_reduction"] == "workspace":
            counters = wsb[256:256 + 4 * plan["tiles"]]
            assert int(counters.count_nonzero().item()) == 0, "arrival counters not reset"
        if plan["k_reduction"] == "workspace-atomic":
            # the decode kernel's stream-K accumulators and counters
            assert int(wsb[256:].count_nonzero().item()) == 0, "workspace not left zeroed"
        return out.view(self.M, self.nout).float().cpu().numpy().astype(np.float64)

    def check(self, y_gpu, what=""):
        y, t = self.ref()
        ok = oracle.within_tolerance(y_gpu, y, t)
        if not ok.all():
            bad = np.argwhere(~ok)
            i, j = bad[0]
            err = np.abs(y_gpu - y)
            bound = oracle.tolerance_bound(y, t)
            worst = np.unravel_index(np.argmax(err / np.maximum(bound, 1e-300)), err.shape)
            raise AssertionError(
                f"{what}: {len(bad)} of {ok.size} outside tolerance; first ({i},{j}) gpu={y_gpu[i, j]!r} "
                f"ref={y[i, j]!r}; worst {worst} gpu={y_gpu[worst]!r} ref={y[worst]!r} bound={bound[worst]!r}")
