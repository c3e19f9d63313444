"""mx_gemm vs the fp64 oracle, element by element, within
|y_gpu - y| <= 2^-8 |y| + 1e-5 sum_k |a_k b_k| (guard bands checked too)."""
import numpy as np
import pytest
import torch

from gpu_helpers import Case

pytestmark = pytest.mark.gpu

E8, E2, F32 = 0, 1, 2  # weight formats
NONE, BIAS, GELU, SWIGLU = 0, 1, 2, 3


def a_fmt_for(b_fmt):
    return 1 if b_fmt == F32 else 0


def test_config0_small_mxfp8_bias(mx):
    # M=16 N=256 K=512, seed 0: e4m3 1x32 activations, 32x32 weights, bias epilogue
    c = Case(16, 256, 512, 0, E8, BIAS, seed=0)
    c.check(c.run_gpu(mx), "config0")


@pytest.mark.parametrize("b_fmt,epi", [(E8, NONE), (E8, BIAS), (E8, GELU), (E8, SWIGLU),
                                       (E2, NONE), (E2, BIAS), (E2, GELU), (E2, SWIGLU),
                                       (F32, NONE), (F32, BIAS), (F32, GELU), (F32, SWIGLU)])
def test_formats_and_epilogues_multi_tile(mx, b_fmt, epi):
    # several M and N tiles with ragged tails; K not a multiple of 128 where allowed
    M = 300
    N = 640 if epi == SWIGLU else (544 if b_fmt != F32 else 520)
    K = 640 if b_fmt == E2 else 672
    c = Case(M, N, K, a_fmt_for(b_fmt), b_fmt, epi, seed=3 + b_fmt * 10 + epi)
    c.check(c.run_gpu(mx), f"fmt{b_fmt} epi{epi}")


@pytest.mark.parametrize("decode", [0, -1])
@pytest.mark.parametrize("M", [1, 2, 7, 8, 16, 31, 33, 64, 65, 127, 128, 129, 257])
def test_m_sweep(mx, M, decode):
    # automatic plan (decode kernel for M <= 64) and the tile kernel alone
    c = Case(M, 256, 512, 0, E8, BIAS, seed=M)
    c.check(c.run_gpu(mx, decode=decode), f"M={M} decode={decode}")


@pytest.mark.parametrize("block_n", [64, 128, 240, 256])
@pytest.mark.parametrize("b_fmt,epi", [(E8, GELU), (E2, SWIGLU), (F32, BIAS)])
def test_tile_widths(mx, block_n, b_fmt, epi):
    c = Case(200, 512, 512, a_fmt_for(b_fmt), b_fmt, epi, seed=block_n + b_fmt)
    c.check(c.run_gpu(mx, block_n=block_n, splits=1), f"BN={block_n}")


@pytest.mark.parametrize("splits", [2, 3, 5, 8, 16])
@pytest.mark.parametrize("block_n", [64, 128, 240, 256])
def test_split_k_cluster_reduction(mx, splits, block_n):
    # minimum workspace: the splits of a tile reduce over a thread-block cluster
    c = Case(40, 512, 2048, 0, E8, BIAS, seed=splits * 7 + block_n)
    c.check(c.run_gpu(mx, block_n=block_n, splits=splits, ws="min"), f"S={splits} BN={block_n}")


@pytest.mark.parametrize("splits", [2, 3, 5, 8, 16, 23, 32])
@pytest.mark.parametrize("block_n", [64, 128, 240, 256])
def test_split_k_workspace_reduction(mx, splits, block_n):
    # full workspace: partials and arrival counters in the workspace, the last
    # CTA of each tile reduces; more splits than a cluster can hold
    c = Case(40, 512, 4096, 0, E8, BIAS, seed=splits * 5 + block_n)
    c.check(c.run_gpu(mx, block_n=block_n, splits=splits), f"S={splits} BN={block_n}")


def test_split_k_workspace_more_units_than_ctas(mx):
    # persistent CTAs that each take several (tile, split) units, the
    # accumulator of one overlapping the partial write-out of the previous
    c = Case(24, 1024, 4096, 0, E8, GELU, seed=77)
    for ctas in (1, 5, 37):
        c.check(c.run_gpu(mx, block_n=128, splits=12, max_ctas=ctas), f"ctas={ctas}")


@pytest.mark.parametrize("ws", ["full", "min"])
@pytest.mark.parametrize("b_fmt,epi", [(E2, SWIGLU), (F32, NONE), (E8, GELU), (E8, NONE)])
def test_split_k_formats(mx, b_fmt, epi, ws):
    # decode-shaped, with the K tail landing in the last split
    M, N = (16, 256) if epi == SWIGLU else (5, 288)
    K = 1536 if b_fmt == E2 else 1568
    c = Case(M, N, K, a_fmt_for(b_fmt), b_fmt, epi, seed=41 + epi)
    c.check(c.run_gpu(mx, block_n=128, splits=4, ws=ws), f"split fmt{b_fmt} epi{epi} ws={ws}")


@pytest.mark.parametrize("ws", ["full", "min"])
def test_split_k_bit_reproducible(mx, ws):
    c = Case(64, 256, 4096, 0, E8, NONE, seed=9)
    y1 = c.run_gpu(mx, block_n=128, splits=8, ws=ws)
    y2 = c.run_gpu(mx, block_n=128, splits=8, ws=ws)
    assert np.array_equal(y1, y2)
    c.check(y1, f"split reproducible ws={ws}")


def test_split_k_workspace_and_cluster_agree_bitwise(mx):
    # both reductions add the same fp32 partials in split order
    c = Case(33, 512, 3072, 0, E8, BIAS, seed=12)
    y_ws = c.run_gpu(mx, block_n=128, splits=6, ws="full")
    y_cl = c.run_gpu(mx, block_n=128, splits=6, ws="min")
    assert np.array_equal(y_ws, y_cl)


@pytest.mark.parametrize("ws", ["full", "min"])
def test_tile_kernel_decode_config1_shape(mx, ws):
    # the decode shape of the fused q_a + kv projection at M = 8 on the tile
    # kernel (decode kernel off): K split through the workspace or a cluster
    c = Case(8, 2048, 7168, 0, E8, NONE, seed=1)
    y = c.run_gpu(mx, decode=-1, ws=ws)
    assert c.last_plan["kernel"] == "tile" and c.last_plan["splits"] > 1
    c.check(y, f"config1 M=8 tile kernel ws={ws}")


def test_gemm_identity_weight_through_gpu(mx):
    # W = I (e4m3 1.0, E8M0 127) -> out = dequantised x, rounded once to bf16
    M, K = 64, 256
    c = Case(M, K, K, 0, E8, NONE, seed=77)
    eye = np.zeros((K, K), np.uint8)
    eye[np.arange(K), np.arange(K)] = 0x38
    c.b_codes = eye
    c.b_scales = np.full((K // 32, K // 32), 127, np.uint8)
    c._ref = None
    y = c.run_gpu(mx)
    yref, _ = c.ref()
    assert np.array_equal(y, torch.from_numpy(yref).to(torch.bfloat16).double().numpy())


def test_gemm_scale_bump_doubles_one_block_through_gpu(mx):
    M, N, K = 32, 128, 256
    c = Case(M, N, K, 0, E8, NONE, seed=5)
    y0 = c.run_gpu(mx)
    c.check(y0, "before bump")
    c.b_scales = c.b_scales.copy()
    c.b_scales[:, :] = 127
    c.b_codes = np.where(np.arange(K)[None, :] < 32, c.b_codes, 0).astype(np.uint8)  # only K block 0
    c._ref = None
    y1 = c.run_gpu(mx)
    c.check(y1, "block 0 only")
    c.b_scales = c.b_scales.copy()
    c.b_scales[:, 0] = 128
    c._ref = None
    y2 = c.run_gpu(mx)
    c.check(y2, "bumped")
    # exactly doubled (power of two scaling commutes with fp32 and bf16 rounding)
    assert np.array_equal(y2, 2 * y1)


@pytest.mark.parametrize("block_n", [64, 128, 240, 256])
@pytest.mark.parametrize("b_fmt,epi", [(E8, BIAS), (E2, SWIGLU), (F32, GELU)])
def test_persistent_many_tiles_per_cta(mx, block_n, b_fmt, epi):
    # a capped grid makes every CTA walk several tiles: exercises the smem ring
    # and the (double-buffered) TMEM accumulator phases across tiles
    M, N, K = 300, (640 if epi == SWIGLU else 544), 640
    c = Case(M, N, K, a_fmt_for(b_fmt), b_fmt, epi, seed=90 + block_n + b_fmt)
    for ctas in (1, 3):
        c.check(c.run_gpu(mx, block_n=block_n, splits=1, max_ctas=ctas), f"BN={block_n} ctas={ctas}")


@pytest.mark.parametrize("b_fmt,epi", [(E8, NONE), (E8, GELU), (E2, SWIGLU), (E2, BIAS), (F32, SWIGLU), (F32, GELU)])
def test_two_row_block_tiles(mx, b_fmt, epi):
    # 256-row tiles (two 128-row MMA blocks sharing each weight tile), with a
    # ragged M tail inside the second block and several tiles per CTA
    M = 300
    N = 640 if epi == SWIGLU else 544
    K = 640 if b_fmt == E2 else 672
    c = Case(M, N, K, a_fmt_for(b_fmt), b_fmt, epi, seed=500 + b_fmt * 10 + epi)
    plan_out = None
    for ctas in (0, 2):
        c.check(c.run_gpu(mx, block_n=240, splits=1, max_ctas=ctas, block_m=256), f"BM=256 ctas={ctas}")


def test_auto_plan_uses_two_row_blocks_for_large_m(mx):
    plan = mx.mx_gemm_plan(4096, 4096, 4096, 0, 0, 2)
    assert plan["block_n"] == 240 and plan["splits"] == 1


@pytest.mark.parametrize("plan", ["tile", "decode", "split-ws", "split-cluster"])
@pytest.mark.parametrize("b_fmt,epi", [(E2, SWIGLU), (E8, GELU), (F32, SWIGLU), (E8, SWIGLU)])
def test_epilogue_far_tails(mx, plan, b_fmt, epi):
    # biases spread over [-120, 120] push the gate / GELU pre-activations into
    # the far tails, where e^-v leaves the fp32 range: SiLU(g) and GELU(v)
    # there are tiny (down to bf16 subnormals), and must come out as such
    M = 300 if plan == "tile" else 16
    N, K = 512, 512
    c = Case(M, N, K, a_fmt_for(b_fmt), b_fmt, epi, seed=70 + b_fmt * 10 + epi)
    gen = torch.Generator().manual_seed(5)
    if epi == SWIGLU:
        gate = torch.linspace(-120.0, 120.0, N // 2)[torch.randperm(N // 2, generator=gen)]
        up = torch.randn(N // 2, generator=gen) * 3
        c.bias = torch.cat([gate, up]).float()
    else:
        c.bias = torch.linspace(-120.0, 120.0, N)[torch.randperm(N, generator=gen)].float()
    c._ref = None
    kw = {"tile": dict(decode=-1), "decode": dict(decode=1),
          "split-ws": dict(decode=-1, block_n=128, splits=4),
          "split-cluster": dict(decode=-1, block_n=128, splits=4, ws="min")}[plan]
    y = c.run_gpu(mx, **kw)
    yref, _ = c.ref()
    if epi == SWIGLU:
        # outputs far below fp32's e^-88 reach, down to bf16 subnormals (the
        # fp64 tanh form of GELU is exactly 0 there, so GELU is checked for
        # finite, in-tolerance tails only)
        tiny = (np.abs(yref) < 2.0 ** -120) & (yref != 0)
        assert tiny.any(), "the case does not reach the far tail"
    assert np.isfinite(y).all()
    c.check(y, f"tails {plan} fmt{b_fmt} epi{epi}")
