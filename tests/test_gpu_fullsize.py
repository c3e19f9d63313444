"""Every workload at its full size, launched the way bench.py times it (CUDA
graph replays of quantisation + GEMM, programmatic dependent launch with
weight prefetch), checked against the fp64 oracle on sampled outputs.

The oracle never sees a value produced on the GPU: it regenerates the sampled
rows of x and W from the seeded generator, quantises them itself, and computes
those outputs; the GPU quantises and multiplies the full matrices.  The samples
follow the launch plan the library chose: at least one row inside every tile
of rows (all rows for the decode kernels, whose one tile holds every token)
and one whole 32-column block inside every tile of output columns, the ragged
last tiles included; for SwiGLU the matching gate and up rows of W come with
each block.  Whole 32-column blocks keep 32 x 32 weight scales regenerable."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

E8, E2, F32 = 0, 1, 2
NONE, BIAS, GELU, SWIGLU = 0, 1, 2, 3

# (name, M, N, K, b_fmt, epi, seed, with_bias[, a_fmt]); seeds as in bench.py
WORKLOADS = [
    ("decode q_a+kv M=1", 1, 2048, 7168, E8, NONE, 1, False),
    ("decode q_a+kv M=8", 8, 2048, 7168, E8, NONE, 1, False),
    ("decode q_a+kv M=32", 32, 2048, 7168, E8, NONE, 1, False),
    ("decode q_a+kv M=64", 64, 2048, 7168, E8, NONE, 1, False),
    ("DiT/ViT MLP bias+GELU", 4096, 4096, 4096, E8, GELU, 2, True),
    ("W4A8 gate_up SwiGLU M=16", 16, 34816, 5120, E2, SWIGLU, 3, False),
    ("W4A8 gate_up SwiGLU M=4096", 4096, 34816, 5120, E2, SWIGLU, 3, False),
    ("fp8 lm_head", 16, 248320, 5120, F32, NONE, 4, False),
    ("W4A8 down projection M=16", 16, 5120, 17408, E2, NONE, 5, False),
    ("W4A8 down projection M=4096", 4096, 5120, 17408, E2, NONE, 5, False),
    ("W4A4 gate_up SwiGLU M=4096", 4096, 34816, 5120, E2, SWIGLU, 3, False, 3),
]


def plan_tiles(plan, M, swiglu):
    """(rows per tile, output columns per tile) of the plan that ran."""
    if plan["kernel"] == "decode":
        # one tile of tokens; 128 weight rows per output tile, a gate and an
        # up sub-tile of 128 each for SwiGLU
        return M, 128
    bn = plan["block_n"]
    return plan["block_m"], (bn // 2 if swiglu else bn)


def sample_rows(M, tile_m, rng):
    """One random row inside every tile of rows, plus the first and last row."""
    if tile_m >= M:
        return np.arange(M, dtype=np.int64)
    rows = {0, M - 1}
    for r0 in range(0, M, tile_m):
        rows.add(int(rng.integers(r0, min(r0 + tile_m, M))))
    return np.array(sorted(rows), np.int64)


def sample_blocks(nout, tile_n, rng):
    """One whole 32-column block inside every tile of output columns (the
    block holding a tile's last column when no block fits inside it), plus the
    first and last block."""
    assert nout % 32 == 0
    blocks = {0, nout // 32 - 1}
    for c0 in range(0, nout, tile_n):
        c1 = min(c0 + tile_n, nout)
        first, last = -(-c0 // 32), c1 // 32 - 1  # blocks wholly inside [c0, c1)
        blocks.add(int(rng.integers(first, last + 1)) if first <= last else (c1 - 1) // 32)
    return np.array(sorted(blocks), np.int64)


@pytest.mark.parametrize("name,M,N,K,b_fmt,epi,seed,with_bias,a_fmt",
                         [w if len(w) == 9 else w + (1 if w[4] == F32 else 0,) for w in WORKLOADS],
                         ids=[w[0] for w in WORKLOADS])
def test_full_size_sampled(mx, name, M, N, K, b_fmt, epi, seed, with_bias, a_fmt):
    dev = "cuda"
    # ---- GPU: the whole problem, as the bench runs it
    w = synth.bf16_matrix(seed + 1, N, K, synth.W_SIGMA, device=dev)
    wc, ws = mx.weight_buffers(N, K, b_fmt)
    mx.mx_quant_weight(w, wc, ws, b_fmt)
    del w
    x = synth.bf16_matrix(seed, M, K, synth.X_SIGMA, device=dev)
    bias = synth.f32_vector(seed + 2, N, synth.BIAS_SIGMA, device=dev) if with_bias else None
    ac, asc = mx.act_buffers(M, K, a_fmt)
    out = mx.out_buffer(M, N, epi)
    wsb = mx.workspace(M, N, K, a_fmt, b_fmt, epi)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())  # inputs and workspace were made on the default stream
    mx.mx_set_launch_flags(mx.MX_LAUNCH_PDL | mx.MX_LAUNCH_PREFETCH_WEIGHTS)
    try:
        with torch.cuda.stream(stream):
            mx.mx_quant_act(x, ac, asc, a_fmt, stream=stream)
            mx.mx_gemm(ac, asc, a_fmt, wc, ws, b_fmt, bias, epi, out, M, N, K, wsb, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            mx.mx_quant_act(x, ac, asc, a_fmt, stream=stream)
            mx.mx_gemm(ac, asc, a_fmt, wc, ws, b_fmt, bias, epi, out, M, N, K, wsb, stream=stream)
        with torch.cuda.stream(stream):
            for _ in range(3):
                out.fill_(float("nan"))
                g.replay()
        stream.synchronize()
    finally:
        mx.mx_set_launch_flags(mx.MX_LAUNCH_PDL)
    assert mx.mx_workspace_status(wsb) == mx.MX_OK
    y_gpu = out.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(y_gpu).all(), "unwritten outputs"
    del g

    # ---- oracle: sampled rows x sampled 32-column blocks, from its own quantisation
    plan = mx.mx_gemm_plan_info(M, N, K, a_fmt, b_fmt, epi, wsb.numel())
    tile_m, tile_n = plan_tiles(plan, M, epi == SWIGLU)
    rng = np.random.default_rng(seed * 7919 + M)
    rows = sample_rows(M, tile_m, rng)
    nout = N // 2 if epi == SWIGLU else N
    blocks = sample_blocks(nout, tile_n, rng)
    assert len(blocks) >= -(-nout // tile_n) and len(rows) >= min(M, -(-M // tile_m))
    cols = (blocks[:, None] * 32 + np.arange(32)[None, :]).ravel()
    w_rows = np.concatenate([cols, cols + N // 2]) if epi == SWIGLU else cols
    # the sampled rows are drawn on the device (the generator is counter based,
    # so they are the rows the GPU multiplied) and handed to the oracle
    xs = synth.bf16_rows(seed, K, synth.X_SIGMA, rows, device=dev).cpu()
    wsel = synth.bf16_rows(seed + 1, K, synth.W_SIGMA, w_rows, device=dev).cpu()
    a_codes, a_scales = oracle.quant_act(xs, a_fmt)
    b_codes, b_scales = oracle.quant_weight(wsel, b_fmt)
    bsel = None
    if with_bias:
        bsel = synth.f32_vector(seed + 2, N, synth.BIAS_SIGMA)[torch.from_numpy(w_rows)]
    y, t = oracle.gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bsel, epi, len(rows), len(w_rows), K)
    got = y_gpu[np.ix_(rows, cols)]
    ok = oracle.within_tolerance(got, y, t)
    if not ok.all():
        i, j = np.argwhere(~ok)[0]
        raise AssertionError(f"{name}: {(~ok).sum()} of {ok.size} sampled outputs outside tolerance; "
                             f"row {rows[i]} col {cols[j]} gpu={got[i, j]!r} ref={y[i, j]!r} T={t[i, j]!r}")
