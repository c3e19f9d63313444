/*
 * mxgemm.h -- C ABI of libmxgemm.so: block-scaled low-precision projection
 * GEMM  y[M, N] = x[M, K] . W^T  with a fused bf16 epilogue, for NVIDIA B200
 * (sm_100a), and the activation-quantisation producer that feeds it.
 *
 * The operation is the one the source pages share:
 *   - the projection itself, y[b, rows] = x[b, cols] . W^T with W stored
 *     [N, K] row-major (cortiq-engine 0.5.39 dit.rs, Proj::matmat; the wgpu
 *     ViT page's `gemm_nt_coop`, "y[n, m] = x[n, k] . w[m, k]^T");
 *   - e4m3 weights with uint8 E8M0 scales over 32 x 32 blocks, layout
 *     [N/32, K/32] (vLLM DeepSeek-V4 mono runner page, AttnWeights: wqkv
 *     [2048, 7168], wqkv_scale [64, 224]);
 *   - MXFP4 (fp4x2) weights [N, K/2] with 1 x 32 E8M0 scales [N, K/32] and a
 *     fused [gate; up] weight ("w13" with 2 * inter rows, MonoLayerWeights on
 *     the same page; the sly-radiance README's fused gate_up N = 34816 in the
 *     radiance_mxfp4_fp8.hip row) feeding a W4A8 GEMM with fp8 activations;
 *   - an fp8 lm_head quantised per output channel with a per-token fp8
 *     activation (sly-radiance README, radiance_lmhead_fp8.py row);
 *   - bias / bias+GELU epilogues fused into the FP8 GEMM (flash-rt GR00T
 *     frontend docstring: "bias / bias+GELU in the hipBLASLt FP8 epilogue"),
 *     bias added before the activation (vit.rs, vt_bias_act), and the SwiGLU
 *     silu(gate) * up of the FFN (dit.rs, `silu` and the FFN block).
 *
 * Conventions shared by every call
 *   - All matrix pointers are DEVICE pointers owned by the caller; dense,
 *     row-major, no padding between rows.  The library allocates nothing,
 *     never synchronises the device (except mx_workspace_status) and launches
 *     only on the given stream, so the calls that take a workspace can be
 *     captured in a CUDA graph.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *   - Every pointer must be 16-byte aligned; e2m1 weight codes 32-byte aligned.
 *   - Errors found while validating return at once and launch nothing.  A
 *     launch failure returns MX_ERR_CUDA.  A device other than sm_100 returns
 *     MX_ERR_ARCH.  A kernel whose bounded waits ran out writes a bit into the
 *     workspace status word (read it with mx_workspace_status).
 *   - Thread safety: all calls are re-entrant; the only global state is a
 *     per-device property cache filled under std::call_once and the optional
 *     tuning override (mx_set_tuning).
 */
#ifndef MXGEMM_H
#define MXGEMM_H

#include <stddef.h>

#if defined(__GNUC__)
#define MX_API __attribute__((visibility("default")))
#else
#define MX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mx_status {
    MX_OK = 0,
    MX_ERR_NULL = 1,      /* a required pointer is NULL                       */
    MX_ERR_SHAPE = 2,     /* a size is out of range or not a required multiple */
    MX_ERR_ALIGN = 3,     /* a pointer is not aligned as required              */
    MX_ERR_FORMAT = 4,    /* unknown format / epilogue, or an invalid pairing  */
    MX_ERR_WORKSPACE = 5, /* workspace missing or smaller than required        */
    MX_ERR_ARCH = 6,      /* current device is not sm_100                      */
    MX_ERR_CUDA = 7,      /* a CUDA call or kernel launch failed               */
    MX_ERR_TIMEOUT = 8    /* a kernel gave up on a bounded wait (status word)  */
} mx_status;

/* Activation operand formats (A = x codes, always e4m3fn). */
typedef enum mx_a_fmt {
    /* e4m3 codes [M, K] + uint8 E8M0 scales [M, K/32] (one per row and
     * 32-wide K block): scale = 2^(e - 127) = 2^ceil(log2(amax / 448)). */
    MX_A_E4M3_E8M0_1X32 = 0,
    /* e4m3 codes [M, K] + fp32 scale per row (token) [M] = amax_row / 448. */
    MX_A_E4M3_F32_ROW = 1,
    /* bf16 activations [M, K] handed to mx_gemm as they are (a_codes = x,
     * a_scales unused, may be NULL): the GEMM quantises them itself, each
     * 1 x 32 block exactly as mx_quant_act does for MX_A_E4M3_E8M0_1X32 (the
     * same codes and scales bit for bit), and multiplies those.  mx_gemm
     * quantises into its workspace first and then multiplies
     * (mx_gemm_workspace_size counts that space; back to back the two
     * launches overlap under MX_LAUNCH_PDL).  For decode shapes (M <= 64,
     * K % 128 == 0) whose workspace has no room for the codes -- the 256-byte
     * minimum, or mx_gemm_noalloc -- the decode kernel quantises them itself
     * in the same launch.  Pairs with the E8M0 weight formats.  Not an output
     * format of mx_quant_act. */
    MX_A_BF16_E8M0_1X32 = 2,
    /* W4A4: e2m1 codes packed two per byte [M, K/2] (low nibble = even k) +
     * uint8 E8M0 scales [M, K/32], k the smallest integer with
     * amax <= 6 * 2^k (the rule of the e2m1 weights), codes RNE onto the e2m1
     * grid.  Pairs with MX_B_E2M1_E8M0_1X32 only (the native MXFP4 W4A4 GEMM,
     * the sly-radiance README's AITER gemm_afp4wfp4 path) and runs at the
     * tensor cores' fp4 rate (tcgen05.mma kind::mxf4, K = 64 per
     * instruction); M > 64 and M <= 64 both take the tile kernel, no K split.
     * mx_quant_act produces it from bf16. */
    MX_A_E2M1_E8M0_1X32 = 3
} mx_a_fmt;

/* Weight operand formats (B = W, stored [N, K]). */
typedef enum mx_b_fmt {
    /* e4m3 codes [N, K] + uint8 E8M0 scales [N/32, K/32] over 32 x 32 blocks. */
    MX_B_E4M3_E8M0_32X32 = 0,
    /* e2m1 codes packed two per byte [N, K/2] (low nibble = even k) + uint8
     * E8M0 scales [N, K/32] (one per row and 32-wide K block). */
    MX_B_E2M1_E8M0_1X32 = 1,
    /* e4m3 codes [N, K] + fp32 scale per output channel [N] = amax_row / 448. */
    MX_B_E4M3_F32_ROW = 2
} mx_b_fmt;

/* Fused epilogues, computed in fp32 and rounded once to bf16. */
typedef enum mx_epi {
    MX_EPI_NONE = 0,           /* y = acc                                         */
    MX_EPI_BIAS = 1,           /* y = acc + bias[n]                               */
    MX_EPI_BIAS_GELU_TANH = 2, /* v = acc + bias[n]; y = 0.5 v (1 + tanh(
                                  sqrt(2/pi) (v + 0.044715 v^3)))                */
    MX_EPI_SWIGLU = 3,         /* W = [gate; up] with N rows (gate rows 0..N/2-1,
                                  up rows N/2..N-1); out [M, N/2]:
                                  y[m, j] = silu(g) * u, g = acc[m, j] (+ bias[j]),
                                  u = acc[m, j + N/2] (+ bias[j + N/2]),
                                  silu(v) = v / (1 + e^-v)                        */
    MX_EPI_RESIDUAL = 4,       /* in place: out[m, n] = out[m, n] + (acc + bias[n]),
                                  bias optional, computed in fp32 and rounded once
                                  to bf16: the residual update x += y + b of the
                                  ViT page's `vt_add`.  out holds the residual
                                  stream on entry and must not overlap the
                                  activations or weights                          */
    MX_EPI_SWIGLU_MXQ = 5      /* MX_EPI_SWIGLU with its result handed on as the
                                  next GEMM's MX operand (the sly README's fused
                                  silu_mul_quant): y = bf16(silu(g) * u) is not
                                  stored; out receives its 1 x 32 E8M0
                                  quantisation, e4m3 codes [M, N/2] followed by
                                  E8M0 scales [M, N/64] from byte M * N/2 of
                                  out -- bit for bit what mx_quant_act gives for
                                  that y, ready for MX_A_E4M3_E8M0_1X32         */
} mx_epi;

/*
 * mx_quant_act -- activation quantisation bf16 -> e4m3 (the producer of the
 * GEMM's A operand; the sly-radiance README's fused producers emit such a
 * `(q_fp8, scale)` pair for the W4A8 GEMM, radiance_fused_norm.py row).
 *
 *   x       [M, K] bf16, device.
 *   codes   [M, K] uint8 (e4m3fn), device, written.
 *   scales  MX_A_E4M3_E8M0_1X32: [M, K/32] uint8 E8M0 -- per block of 32,
 *           e = clamp(127 + k, 0, 254) with k the smallest integer such that
 *           amax <= 448 * 2^k (an all-zero block gets e = 0); codes are
 *           round-to-nearest-even of x * 2^-k (exact scaling, so never
 *           saturating), the sign of zero kept.
 *           MX_A_E4M3_F32_ROW: [M] fp32 -- s = amax_row / 448 (IEEE division;
 *           1.0 for an all-zero row); codes = RNE_satfinite(x / s).
 *           MX_A_E2M1_E8M0_1X32: codes [M, K/2] packed e2m1 (low nibble =
 *           even k), scales [M, K/32] E8M0 with k the smallest integer such
 *           that amax <= 6 * 2^k; codes RNE onto {0, .5, 1, 1.5, 2, 3, 4, 6}
 *           of x * 2^-k, the sign kept.
 *   Requires M >= 1, K >= 32, K % 32 == 0.  The result is bit-exact: it is the
 *   unique rounding the definition gives.
 */
MX_API mx_status mx_quant_act(const void* x, int M, int K, void* codes, void* scales, mx_a_fmt fmt, void* stream);

/*
 * mx_quant_weight -- one-off weight preparation bf16 [N, K] -> the chosen
 * B format (the pages load weights already in these layouts; this call makes
 * them from bf16, e.g. "quantized to fp8 per output channel after loading",
 * sly-radiance README, radiance_lmhead_fp8.py row).
 *
 *   MX_B_E4M3_E8M0_32X32: codes [N, K] uint8, scales [N/32, K/32] uint8;
 *     same exponent rule as the activations over each 32 x 32 block.
 *     Requires N % 32 == 0, K % 32 == 0.
 *   MX_B_E2M1_E8M0_1X32: codes [N, K/2] uint8 (two e2m1 per byte, low nibble =
 *     even k), scales [N, K/32] uint8; k = smallest integer with
 *     amax <= 6 * 2^k, codes = RNE onto {0, .5, 1, 1.5, 2, 3, 4, 6}.
 *     Requires K % 32 == 0.
 *   MX_B_E4M3_F32_ROW: codes [N, K] uint8, scales [N] fp32 = amax_row / 448.
 */
MX_API mx_status mx_quant_weight(const void* w, int N, int K, void* codes, void* scales, mx_b_fmt fmt, void* stream);

/*
 * mx_add_rms_quant -- residual add, RMSNorm and 1 x 32 E8M0 quantisation of
 * each row: the producer that hands the next GEMM its MX operand (sly-radiance
 * README, Contents table, radiance_fused_norm.py row: the fused add_rms_quant
 * op returns (q_fp8, scale) for the W4A8 linear; RMSNorm with a plain weight as
 * the DiT page's `rms_norm` defines it, x * rsqrt(mean x^2 + eps) * w).  Read
 * as the unfused chain it replaces, for each row m:
 *   r = bf16(x + residual), written back into `residual` (in place);
 *   y = bf16(r * rsqrt(mean_k r^2 + eps) * w);
 *   codes + scales = the 1 x 32 E8M0 quantisation of y, bit for bit what
 *   mx_quant_act gives for that y; y itself goes to y_out when it is not NULL.
 *
 *   x         [M, K] bf16, device, read.
 *   residual  [M, K] bf16, device, read and overwritten with r (may be x).
 *   w         [K] bf16, device, read.
 *   eps       >= 0.
 *   y_out     [M, K] bf16, device, written; NULL = not wanted.
 *   codes     [M, K] uint8 e4m3, device, written.
 *   scales    [M, K/32] uint8 E8M0, device, written.
 * The sum of squares is taken in fp32, so y can differ from an fp64 chain by
 * one bf16 rounding where it falls near a bf16 midpoint; codes and scales are
 * always those of the y written.  Requires M >= 1, 32 <= K <= 16384,
 * K % 32 == 0; x, residual, w, codes and y_out 16-byte aligned.  Errors as
 * mx_quant_act; no workspace.
 */
MX_API mx_status mx_add_rms_quant(const void* x, void* residual, const void* w, float eps, int M, int K,
                                  void* y_out, void* codes, void* scales, void* stream);

/*
 * mx_gemm_workspace_size -- bytes of workspace that let mx_gemm run its fastest
 * plan for this problem on the current device: a 256-byte status block, plus,
 * when K is split across CTAs, one arrival counter per output tile and the
 * split-K storage.  For M <= 64 (the decode kernel) that is one fp32
 * accumulator per tile of 128 output columns (tiles x M x 128 x 4 bytes, twice
 * that for SwiGLU); for larger decode-like shapes of the tile kernel, the fp32
 * partials of every split (splits x min(M,128) x tile width x 4 bytes per
 * tile).  mx_gemm accepts any workspace of at least 256 bytes and plans within
 * what it is given (with less, the decode kernel runs whole tiles, or K splits
 * are reduced over thread-block clusters).  The caller zero-fills the
 * workspace once when allocating it; kernels leave it as they found it (the
 * last CTA of a tile resets its counter and clears its accumulator) unless a
 * bounded wait ran out, after which the workspace must be zero-filled again.
 * Use one workspace per stream with work in flight.  For
 * MX_A_BF16_E8M0_1X32 activations that do not take the fused decode path the
 * size includes the quantised activations (M x K code bytes and M x K/32
 * scale bytes, each rounded up to 256 bytes).  Returns 256 when no sm_100
 * device is current.
 *
 * The contract follows the scratch of the vLLM DeepSeek-V4 mono runner page
 * (MonoRunner.scratch): caller-visible device scratch per problem shape,
 * zero-filled when first allocated, allocated on an eager call and never
 * while a stream is being captured (the runner raises an error if a width is
 * first reached inside a capture), so that captured launches see only
 * pointers.  Its arrival counters reset themselves, like the runner's
 * kernel-advanced epoch words, so the same workspace serves every replay.
 */
MX_API size_t mx_gemm_workspace_size(int M, int N, int K, mx_a_fmt a_fmt, mx_b_fmt b_fmt, mx_epi epi);

/*
 * mx_gemm -- out = epilogue(x . W^T) with block-scaled low-precision operands.
 *
 *   a_codes, a_scales, a_fmt   activation operand (see mx_a_fmt).
 *   b_codes, b_scales, b_fmt   weight operand (see mx_b_fmt).
 *   bias     fp32 [N] (device); required for BIAS and BIAS_GELU_TANH, optional
 *            (NULL = none) for SWIGLU, must be NULL for NONE.
 *   epi      fused epilogue (mx_epi).
 *   out      bf16 [M, N] ([M, N/2] for SWIGLU), device, written; rounded to
 *            nearest even from the fp32 epilogue value.
 *   M, N, K  problem size (N counts gate and up rows for SWIGLU).
 *   workspace, ws_bytes   caller-owned device scratch, 16-byte aligned, at
 *            least 256 bytes (MX_ERR_WORKSPACE otherwise) and ideally
 *            mx_gemm_workspace_size(...) bytes; zero-filled once.
 *
 *   Each 32-wide K block contributes 2^(ea-127) * 2^(eb-127) * sum(a * w) for
 *   E8M0 formats; the fp32-row pair gives sx[m] * sw[n] * sum(a * w).
 *   Accumulation is fp32 on the tensor cores.  Accepted error against the
 *   exact value: |y - y_exact| <= 2^-8 |y_exact| + 1e-5 sum_k |a_k w_k|.
 *
 *   Valid (a_fmt, b_fmt) pairs: (E8M0_1X32 or BF16_E8M0_1X32,
 *   E4M3_E8M0_32X32), (E8M0_1X32 or BF16_E8M0_1X32, E2M1_E8M0_1X32),
 *   (F32_ROW, E4M3_F32_ROW).  With BF16_E8M0_1X32 the result is the one the
 *   same call gives on mx_quant_act's codes and scales.
 *   Requires M >= 1, N >= 1, K >= 32, K % 32 == 0; N % 32 == 0 for 32 x 32
 *   scales; K % 128 == 0 for e2m1 weights; N % 64 == 0 for SWIGLU.
 */
MX_API mx_status mx_gemm(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                  const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out, int M, int N,
                  int K, void* workspace, size_t ws_bytes, void* stream);

/*
 * mx_gemm_grouped -- `groups` independent GEMMs that share N, K, formats and
 * epilogue in one launch: the routed experts of a mixture-of-experts layer
 * (vLLM DeepSeek-V4 mono runner page, MonoLayerWeights: w13 [experts,
 * 2 inter, hidden / 2] and w2 [experts, hidden, inter / 2] fp4x2 with their
 * 1 x 32 E8M0 scales [experts * rows, hidden / 32]).  The tokens come sorted
 * by group: activation rows offsets[g] .. offsets[g + 1] - 1 go through group
 * g's weights and bias, and the result lands in the same rows of out.
 *
 *   a_codes, a_scales  [M, K] activations of every group, M = offsets[groups];
 *                      MX_A_E4M3_E8M0_1X32 or MX_A_E2M1_E8M0_1X32 (W4A4).
 *   b_codes, b_scales  the groups' weights back to back: codes [groups * N,
 *                      K] (e4m3) or [groups * N, K/2] (e2m1), scales as the
 *                      B format lays out groups * N rows ([groups * N / 32,
 *                      K/32] for 32 x 32 blocks, [groups * N, K/32] for 1 x 32).
 *   bias               fp32 [groups, N] or NULL (rules of mx_gemm).
 *   epi                any mx_epi but MX_EPI_SWIGLU_MXQ.
 *   out                [M, N] bf16 ([M, N/2] for SWIGLU).
 *   offsets            HOST array of groups + 1 ints: 0 = offsets[0] <=
 *                      offsets[1] <= ... ; a group may be empty.
 *   workspace          as mx_gemm (the 256-byte minimum is enough).
 * Requires 1 <= groups <= 256; shapes, alignment and format pairs as mx_gemm
 * (F32_ROW and bf16 activations are not taken).  The groups' tiles share one
 * persistent launch of the tile kernel, whatever the rows per group, so
 * small groups do not each pay a launch.  M = 0 (every group empty) returns
 * MX_OK and launches nothing.
 */
MX_API mx_status mx_gemm_grouped(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                                 const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out,
                                 int groups, const int* offsets, int N, int K, void* workspace, size_t ws_bytes,
                                 void* stream);
#define MX_MAX_GROUPS 256

/*
 * mx_gemm_noalloc -- mx_gemm for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for users of this
 * library who cannot hand mx_gemm a workspace: runtimes that give kernels a
 * fixed arena and forbid hidden allocations, and plain-C plugin hosts with no
 * device allocator.
 *
 * Same arguments, results and tolerance as mx_gemm, minus the workspace.  The
 * scratch is a MX_NOALLOC_SCRATCH_BYTES array inside the library, held by
 * every GPU that loads it until the process exits; a plan that would need
 * more scratch than that returns MX_ERR_WORKSPACE (so do MX_A_BF16_E8M0_1X32
 * activations outside the decode shapes, which would quantise into it; decode
 * shapes quantise inside the decode kernel).  Only the scratch's status
 * word is used (calls never keep split-K partials there), so decode-sized
 * problems take the cluster-reduced split plan.  The call allocates and
 * frees nothing.  Its first call on a device looks the array's device address
 * up (cudaGetSymbolAddress, with that device current) and keeps it for that
 * device's context; after a device reset or anything else that replaces the
 * context, the next call looks the address up anew.  All calls share the array, which keeps what
 * the last call left there (only a give-up of a bounded wait writes it, and no
 * kernel reads it back), so calls that overlap on the GPU race on it.  A
 * give-up cannot be read back through this call; use mx_gemm with a workspace
 * when that matters.
 */
#define MX_NOALLOC_SCRATCH_BYTES 4096
MX_API mx_status mx_gemm_noalloc(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                                 const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out,
                                 int M, int N, int K, void* stream);

/* Human-readable name of a status code (static storage). */
MX_API const char* mx_status_string(mx_status s);

/*
 * mx_workspace_status -- synchronises `stream`, reads the workspace status
 * word and returns MX_OK if it is zero, MX_ERR_TIMEOUT if a kernel gave up on
 * a bounded wait (the word is then cleared), MX_ERR_CUDA on a CUDA error.
 * The word is the first 4 bytes of the workspace; kernels only OR bits into
 * it.  It plays the part of the status words in the vLLM DeepSeek-V4 mono
 * runner page's device mailbox (MonoRunner's epoch tensor: an epoch, a mark
 * per CTA and counters that the kernels themselves advance), read back on
 * the host between launches rather than by a later kernel.
 */
MX_API mx_status mx_workspace_status(void* workspace, void* stream);

/*
 * mx_debug_watchdog -- test hook for the bounded waits: launches one block
 * that waits on an mbarrier nobody arrives on, gives up after `timeout_us`
 * microseconds, records the give-up in the workspace status word and exits
 * normally.  Returns the launch status; read the result with
 * mx_workspace_status.  Never faults or traps.
 */
MX_API mx_status mx_debug_watchdog(void* workspace, size_t ws_bytes, unsigned timeout_us, void* stream);

/*
 * mx_set_tuning -- process-wide override of the tile choice for tuning and
 * tests: block_n in {0 (auto), 64, 128, 256} columns of W per tile; splits in
 * {0 (auto), 1 .. 16} K-splits (a thread-block cluster of that size reduces
 * them on chip); max_ctas caps the persistent grid (0 = one CTA per SM);
 * block_m in {0 (auto), 128, 256, MX_TUNE_BM_PAIR} output rows per tile (256 =
 * two 128-row MMA blocks sharing each weight tile; only with block_n 240 and
 * no K split; MX_TUNE_BM_PAIR = 256 x 240 tiles over pairs of CTAs on two SMs,
 * cta_group::2 MMAs; block_n 0 or 240, no K split; max_ctas caps the CTAs).
 * Not for concurrent use with other threads' mx_gemm calls.
 */
MX_API void mx_set_tuning(int block_n, int splits, int max_ctas, int block_m);
#define MX_TUNE_BM_PAIR 2

/*
 * mx_set_launch_flags -- process-wide launch options (default MX_LAUNCH_PDL).
 *   MX_LAUNCH_PDL: launch the kernels with programmatic dependent launch.  A
 *     kernel may then start its set-up while the previous kernel in the stream
 *     is finishing; every access to global memory still waits until that
 *     kernel has completed, so results are the same as without the flag.
 *   MX_LAUNCH_PREFETCH_WEIGHTS (only with MX_LAUNCH_PDL): mx_gemm may read the
 *     weight codes and scales before the previous kernel in the stream has
 *     completed.  Set it only when that kernel never writes the weights (the
 *     usual case for inference, where weights are constant); activations,
 *     bias, scales of the activations and the output are still ordered.
 *   MX_LAUNCH_DETERMINISTIC: bitwise-reproducible results from run to run.
 *     Without it, decode-sized GEMMs (M <= 64) whose K is split across CTAs
 *     add the fp32 partials of a tile with atomic adds in arrival order (the
 *     results stay within the stated tolerance but may differ in the last
 *     bit between runs); with it they run whole tiles per CTA, or the tile
 *     kernel with its fixed-order split-K reductions.
 */
#define MX_LAUNCH_PDL 1u
#define MX_LAUNCH_PREFETCH_WEIGHTS 2u
#define MX_LAUNCH_DETERMINISTIC 4u
MX_API void mx_set_launch_flags(unsigned flags);

/*
 * mx_set_decode_tuning -- process-wide override of the decode kernel choice,
 * for tuning and tests.  The decode kernel puts the weights on the MMA's
 * 128-row side and the tokens on its N side.  mode 0: automatic (the decode
 * kernel for M <= 64, unless mx_set_tuning overrides are set); 1 (or more):
 * the decode kernel whenever it can run the problem (M <= 64; K % 128 == 0
 * for E8M0 formats), even with mx_set_tuning overrides or few tiles; -1:
 * never.
 * ctas: its grid size (0 = one CTA per SM).  ctas_per_sm: its shared-memory
 * budget -- 2 (at most 113 KB, so the next launch's CTAs can start beside this
 * launch's), 1 (a deep weight ring for long-running problems), 0 = choose.
 * prefetch_stages: with MX_LAUNCH_PREFETCH_WEIGHTS, how many weight stages
 * each CTA may request before the previous kernel has completed (0 = as many
 * as its ring holds).  split: how a tile's K range is shared between CTAs --
 * 0 automatic (a cluster per tile when there are fewer tiles than SMs, else
 * whole tiles), 1 a thread-block cluster per tile (partials reduced in
 * distributed shared memory, in rank order), 2 stream-K (equal ranges of
 * (tile, K block) units over `ctas` CTAs; cut tiles reduced with fp32 atomic
 * adds in the workspace, arrival order), 3 whole tiles.  cluster_size: CTAs
 * per cluster for split 0 / 1 (2..8; 0 = fill the SMs).  Not for concurrent
 * use with other threads' mx_gemm calls.
 */
MX_API void mx_set_decode_tuning(int mode, int ctas, int ctas_per_sm, int prefetch_stages, int split,
                                 int cluster_size);

/*
 * mx_debug_set_timeline -- tracing: install (or, with NULL, remove) a device
 * buffer into which every later mx_gemm launch writes, per CTA (linear index
 * blockIdx.y * gridDim.x + blockIdx.x), 16 uint64 slots: %globaltimer
 * nanoseconds at kernel start, setup done, first TMA issued, first stage
 * landed, last MMA committed, accumulator ready, tile stored / partial
 * parked, cluster barrier 1, reduction done, cluster barrier 2, kernel end,
 * then the SM id (slot 11).  The last 256 slots of the buffer hold the
 * first 64 K-steps of CTA 0 (TMA issued, stage landed, MMAs committed, scale
 * copies issued; 64 slots each); the per-CTA records fill what is in front of
 * them ((bytes / 8 - 256) / 16 CTAs), later CTAs are not recorded.  A buffer
 * smaller than 272 slots disables tracing.  Process-wide; for profiling only.
 * The kernels record only in a library built with MXG_TRACE=1 (the package's
 * build step writes that variant as libmxgemm_trace.so); the default build
 * accepts the call and records nothing, because the per-iteration checks of
 * the tracing code slow short launches even when no buffer is installed.
 */
MX_API void mx_debug_set_timeline(void* buffer, size_t bytes);

/*
 * mx_gemm_plan -- the tile choice mx_gemm would make for this problem on the
 * current device: writes block_n, splits, grid size (CTAs) and the number of
 * accumulator buffers.  For logging and benchmarks; launches nothing.
 */
MX_API mx_status mx_gemm_plan(int M, int N, int K, mx_a_fmt a_fmt, mx_b_fmt b_fmt, mx_epi epi, int* block_n,
                       int* splits, int* grid, int* acc_bufs);

/*
 * mx_gemm_plan_info -- the full launch plan mx_gemm would choose for this
 * problem on the current device when handed `ws_bytes` of workspace
 * ((size_t)-1: as much as its fastest plan wants).  For logging, benchmarks
 * and tests; launches nothing.
 */
typedef struct mx_plan_info {
    int kernel;      /* 0: tile kernel (activation-row x weight-row tiles);
                        1: decode kernel (weights as the MMA's 128-row side);
                        3: tile kernel over CTA pairs (256 x 240 tiles,
                           cta_group::2 MMAs) */
    int block_m;     /* activation rows per tile (decode kernel: tokens per MMA) */
    int block_n;     /* weight rows per tile (decode kernel: 128 per sub-tile) */
    int splits;      /* K splits per tile (decode kernel: about how many CTAs
                        share one tile) */
    int k_reduction; /* 0 none; 1 thread-block cluster (distributed shared
                        memory, fixed order); 2 workspace partials (fixed
                        order); 3 workspace fp32 atomic adds (arrival order) */
    int grid;        /* CTAs launched */
    int acc_bufs;    /* TMEM accumulator buffers */
    int stages;      /* shared-memory ring depth */
    int tiles;       /* output tiles */
    size_t ws_bytes; /* workspace this plan needs */
    int ctas_per_sm; /* CTAs the kernel's shared-memory budget lets one SM hold */
    int act_quant;   /* MX_A_BF16_E8M0_1X32: 1 quantised inside the decode
                        kernel, 2 quantised into the workspace first; else 0 */
} mx_plan_info;
MX_API mx_status mx_gemm_plan_info(int M, int N, int K, mx_a_fmt a_fmt, mx_b_fmt b_fmt, mx_epi epi,
                                   size_t ws_bytes, mx_plan_info* info);

#ifdef __cplusplus
}
#endif

#endif /* MXGEMM_H */
