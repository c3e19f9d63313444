"""mx_gemm_grouped (routed experts in one launch) against the oracle's grouped
GEMM, element by element within |y_gpu - y| <= 2^-8 |y| + 1e-5 T: tokens
sorted by expert with ragged and empty groups, e2m1 (the W4A8 MoE layout of
the DeepSeek-V4 mono runner page) and e4m3 32 x 32 expert weights, W4A4,
every epilogue, tile widths, and persistent CTAs walking tiles of several
groups."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import guarded, guards_intact, to_dev

pytestmark = pytest.mark.gpu
E8, E2 = 0, 1
NONE, BIAS, GELU, SWIGLU, RESIDUAL = 0, 1, 2, 3, 4


class Grouped:
    def __init__(self, counts, N, K, a_fmt, b_fmt, epi, seed, with_bias=True):
        self.counts, self.N, self.K = list(counts), N, K
        self.a_fmt, self.b_fmt, self.epi = a_fmt, b_fmt, epi
        self.offsets = np.concatenate([[0], np.cumsum(self.counts)]).astype(np.int64)
        self.M = int(self.offsets[-1])
        G = len(self.counts)
        x = synth.bf16_matrix(seed, max(self.M, 1), K, synth.X_SIGMA)[:self.M]
        self.a, self.sa = oracle.quant_act(x, a_fmt) if self.M else (None, None)
        self.bc, self.sb, self.bias = [], [], []
        for g in range(G):
            c, s = oracle.quant_weight(synth.bf16_matrix(seed + 10 + g, N, K, synth.W_SIGMA), b_fmt)
            self.bc.append(c)
            self.sb.append(s)
            self.bias.append(synth.f32_vector(seed + 100 + g, N, synth.BIAS_SIGMA))
        self.use_bias = epi in (BIAS, GELU) or (epi in (SWIGLU, RESIDUAL) and with_bias)
        self.nout = N // 2 if epi == SWIGLU else N
        self.res = synth.bf16_matrix(seed + 7, max(self.M, 1), self.nout, 1.0)[:self.M] if epi == RESIDUAL else None

    def ref(self):
        bias = self.bias if self.use_bias else None
        if self.epi != RESIDUAL:
            return oracle.gemm_grouped(self.a, self.sa, self.a_fmt, self.bc, self.sb, self.b_fmt, bias, self.epi,
                                       self.offsets, self.N, self.K)
        y = np.zeros((self.M, self.N))
        t = np.zeros((self.M, self.N))
        for g in range(len(self.counts)):
            r0, r1 = self.offsets[g], self.offsets[g + 1]
            if r1 > r0:
                y[r0:r1], t[r0:r1] = oracle.gemm_residual(
                    np.ascontiguousarray(self.a[r0:r1]), np.ascontiguousarray(self.sa[r0:r1]), self.a_fmt,
                    self.bc[g], self.sb[g], self.b_fmt, None if bias is None else bias[g], self.res[r0:r1],
                    int(r1 - r0), self.N, self.K)
        return y, t

    def run(self, mx, block_n=0, max_ctas=0):
        full, out = guarded(max(self.M, 1) * self.nout)
        if self.epi == RESIDUAL and self.M:
            out[:self.M * self.nout].copy_(self.res.reshape(-1).cuda())
        b = to_dev(np.concatenate(self.bc, 0))
        sb = to_dev(np.concatenate(self.sb, 0))
        bias = torch.cat(self.bias).cuda() if self.use_bias else None
        a = to_dev(self.a) if self.M else torch.zeros(16, dtype=torch.uint8, device="cuda")
        sa = to_dev(self.sa) if self.M else torch.zeros(16, dtype=torch.uint8, device="cuda")
        ws = mx.workspace()
        mx.mx_set_tuning(block_n, 0, max_ctas, 0)
        try:
            mx.mx_gemm_grouped(a, sa, self.a_fmt, b, sb, self.b_fmt, bias, self.epi, out, self.offsets, self.N,
                               self.K, ws)
        finally:
            mx.mx_set_tuning(0, 0)
        torch.cuda.synchronize()
        assert mx.mx_workspace_status(ws) == 0
        assert guards_intact(full), "write outside the output"
        return out[:self.M * self.nout].view(self.M, self.nout).float().cpu().numpy().astype(np.float64), out

    def check(self, y_gpu, what):
        y, t = self.ref()
        ok = oracle.within_tolerance(y_gpu, y, t)
        if not ok.all():
            i, j = np.argwhere(~ok)[0]
            raise AssertionError(f"{what}: {(~ok).sum()} of {ok.size} outside tolerance; first ({i},{j}) "
                                 f"gpu={y_gpu[i, j]!r} ref={y[i, j]!r} T={t[i, j]!r}")


COUNTS = [130, 0, 77, 256, 1]


@pytest.mark.parametrize("epi", [NONE, BIAS, GELU, SWIGLU, RESIDUAL])
@pytest.mark.parametrize("b_fmt", [E2, E8])
def test_grouped_formats_and_epilogues(mx, b_fmt, epi):
    N, K = 640, 512
    c = Grouped(COUNTS, N, K, 0, b_fmt, epi, seed=17000 + 10 * b_fmt + epi)
    y, _ = c.run(mx)
    c.check(y, f"grouped fmt{b_fmt} epi{epi}")


@pytest.mark.parametrize("block_n,max_ctas", [(128, 0), (256, 0), (0, 1), (0, 3), (240, 7)])
def test_grouped_tiles_and_persistent_ctas(mx, block_n, max_ctas):
    # CTAs that walk tiles of several groups, empty groups between them
    N, K = 544, 640
    c = Grouped([1, 0, 0, 200, 64, 0, 129], N, K, 0, E2, BIAS, seed=17100 + block_n + max_ctas)
    y, _ = c.run(mx, block_n=block_n, max_ctas=max_ctas)
    c.check(y, f"grouped BN={block_n} ctas={max_ctas}")


@pytest.mark.parametrize("epi", [NONE, SWIGLU])
def test_grouped_w4a4(mx, epi):
    N, K = 640, 768
    c = Grouped([33, 160, 0, 5], N, K, 3, E2, epi, seed=17200 + epi)
    y, _ = c.run(mx)
    c.check(y, f"grouped W4A4 epi{epi}")


def test_grouped_moe_decode_counts(mx):
    # a decode step: a few tokens per expert, most experts empty, 16 experts
    N, K = 1024, 1024
    counts = [0, 2, 0, 0, 1, 0, 3, 0, 0, 0, 1, 0, 0, 1, 0, 0]
    c = Grouped(counts, N, K, 0, E2, SWIGLU, seed=17300)
    y, _ = c.run(mx)
    c.check(y, "grouped decode counts")


def test_grouped_one_group_matches_the_oracle_gemm(mx):
    N, K = 512, 1024
    c = Grouped([300], N, K, 0, E8, GELU, seed=17400)
    y, _ = c.run(mx)
    y_ref, t = oracle.gemm(c.a, c.sa, 0, c.bc[0], c.sb[0], E8, c.bias[0], GELU, 300, N, K)
    assert oracle.within_tolerance(y, y_ref, t).all()


def test_grouped_all_empty_launches_nothing(mx):
    c = Grouped([0, 0, 0], 256, 256, 0, E2, NONE, seed=17500)
    full, out = guarded(256)
    b = to_dev(np.concatenate(c.bc, 0))
    sb = to_dev(np.concatenate(c.sb, 0))
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    mx.mx_gemm_grouped(z, z, 0, b, sb, E2, None, NONE, out, [0, 0, 0, 0], 256, 256, mx.workspace())
    torch.cuda.synchronize()
    assert guards_intact(full)
    assert (full.cpu().numpy() == 0x7FA5).all(), "an empty problem wrote its output"
