// mx_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/mxgemm.h"

namespace mxg {

// Epilogues whose weight is a fused [gate; up] with N rows and N/2 outputs.
inline bool epi_swiglu(int epi) { return epi == MX_EPI_SWIGLU || epi == MX_EPI_SWIGLU_MXQ; }

// Status word bits written by kernels into the workspace.
constexpr unsigned kStatusTimeout = 1u;

// Bounded waits give up after this many nanoseconds of %globaltimer.
#ifndef MXG_WATCHDOG_NS
#define MXG_WATCHDOG_NS 2000000000ull
#endif

// Kernel tracing (mx_debug_set_timeline) is compiled in only with
// -DMXG_TRACE=1: even switched off at run time, its per-iteration checks
// added about 1 us to a 7 us decode launch.
#ifndef MXG_TRACE
#define MXG_TRACE 0
#endif

struct DeviceInfo {
    int device = -1;
    int sms = 0;
    int major = 0, minor = 0;
    size_t smem_optin = 0;
};

// Cached properties of the current device; returns cudaSuccess or the error.
cudaError_t current_device(DeviceInfo* out);

// ---- quantisation launchers (mx_quant.cu) ---------------------------------
cudaError_t launch_add_rms_quant(const void* x, void* res, const void* w, float eps, int M, int K, void* y_out,
                                 void* codes, void* scales, cudaStream_t st);
cudaError_t launch_quant_e8m0_1x32(const void* x, long long rows, int K, uint8_t* codes, uint8_t* scales,
                                   cudaStream_t st);
cudaError_t launch_quant_f32_row(const void* x, int rows, int K, uint8_t* codes, float* scales, cudaStream_t st);
cudaError_t launch_quant_w_e4m3_32x32(const void* w, int N, int K, uint8_t* codes, uint8_t* scales,
                                      cudaStream_t st);
cudaError_t launch_quant_w_e2m1_1x32(const void* w, int N, int K, uint8_t* codes, uint8_t* scales,
                                     cudaStream_t st);

// ---- GEMM (mx_gemm.cu) -------------------------------------------------------
// Activation formats with E8M0 block scales (codes given, or bf16 quantised by the GEMM).
inline bool a_fmt_e8m0(int fmt) { return fmt == MX_A_E4M3_E8M0_1X32 || fmt == MX_A_BF16_E8M0_1X32; }

// bf16 activations are quantised inside the decode kernel while M x tiles is
// at most this (each tile's CTAs quantise the tokens of their K range), and
// by the quantisation kernel ahead of it otherwise.  Zero: with room in the
// workspace, quantising ahead (a separate launch that programmatic
// dependent launch overlaps with the GEMM's start) measured faster over
// back-to-back decode steps (37.8 against 38.2 us for 4 x M in {1, 8, 32,
// 64} at N 2048, K 7168), so the decode kernel quantises only when the
// workspace has no room for the codes.
constexpr long long kFusedQuantMaxWork = 0;

// Workspace bytes of bf16 activations quantised ahead of the GEMM: codes
// [M, K] then scales [M, K/32], each rounded up to 256 bytes.
inline size_t act_quant_bytes(int M, int K)
{
    const size_t codes = (static_cast<size_t>(M) * K + 255) / 256 * 256;
    const size_t scales = (static_cast<size_t>(M) * (K / 32) + 255) / 256 * 256;
    return codes + scales;
}

// Most groups one grouped launch takes (the group table travels in the
// kernel's parameters).
constexpr int kMaxGroups = 256;

struct GemmProblem {
    const void* a_codes;
    const void* a_scales;
    int a_fmt;
    const void* b_codes;
    const void* b_scales;
    int b_fmt;
    const float* bias;
    int epi;
    void* out;
    int M, N, K;
    unsigned* status;
    // grouped launch: `groups` problems sharing N, K, formats and epilogue;
    // host offsets[0 .. groups] of their activation rows (M = offsets[groups])
    int groups = 0;
    const int* offsets = nullptr;
};

struct GemmPlan {
    int block_n = 0;
    int splits = 1;
    int grid_x = 0, grid_y = 0;
    int acc_bufs = 0;
    int units = 0;
    int a_rows = 128;  // activation rows loaded per stage (64 when M <= 64, 256 for two 128-row blocks)
    int block_m = 128; // output rows per tile
    int gsplit = 0;    // K splits reduced through the workspace (1) or a thread-block cluster (0)
    int part_rows = 0; // rows of one workspace partial tile
    size_t ws_bytes = 0;  // workspace this plan needs
    int stages = 0;       // shared-memory ring depth
    // decode kernel (kernel == 1): weights are the MMA's 128-row side, tokens its N
    int kernel = 0;       // 0 = tile kernel (mx_gemm.cu), 1 = decode kernel, weights on the MMA's M side
                          // (mx_decode.cu), 3 = tile kernel over CTA pairs (mx_gemm_pair.cu)
    int tiles = 0;        // decode: tiles of 128 output columns
    int whole_tiles = 0;  // decode: CTAs take whole tiles (no cross-CTA reduction)
    int reduce = 0;       // decode: some tile's K range is split between CTAs (workspace accumulators)
    int one_per_sm = 0;   // decode: one CTA per SM with a deep weight ring (else two CTAs per SM)
    int cluster = 1;      // decode: CTAs per cluster sharing one tile's K range (1 = none)
    // bf16 activations (MX_A_BF16_E8M0_1X32): quantised inside the decode
    // kernel (act_quant = 1) or into the workspace at byte quant_off by the
    // quantisation kernel before the GEMM (act_quant = 2)
    int act_quant = 0;
    size_t quant_off = 0;
    // MX_EPI_SWIGLU_MXQ: the SwiGLU output quantised inside the decode
    // kernel's epilogue (out_quant = 1), or stored as bf16 into the workspace
    // at byte out_off and quantised from there (out_quant = 2)
    int out_quant = 0;
    size_t out_off = 0;
};

// How the decode kernel shares a tile's K range between CTAs.
enum DecSplit { kDecAuto = 0, kDecCluster = 1, kDecStreamK = 2, kDecWholeTiles = 3 };

// Workspace layout: [0, 256) status word and reserved; then one arrival
// counter per output tile (256-byte aligned block); then the fp32 split-K
// partials.  Counters are zero between launches (the last arrival resets).
constexpr size_t kWorkspaceHeader = 256;

// Plans the launch; `ws_bytes` is the workspace available (plans that need
// more are not considered).
cudaError_t plan_gemm(const GemmProblem& pb, const DeviceInfo& dev, size_t ws_bytes, GemmPlan* plan);
cudaError_t launch_gemm(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st);
// grouped problems (pb.groups > 0): the tile kernel over every group's tiles
cudaError_t plan_gemm_grouped(const GemmProblem& pb, const DeviceInfo& dev, GemmPlan* plan);
cudaError_t launch_watchdog_probe(unsigned* status, unsigned timeout_us, cudaStream_t st);

void set_tuning(int block_n, int splits, int max_ctas, int block_m);
void set_decode_tuning(int mode, int ctas, int per_sm, int prefetch_stages, int split, int cluster);
int decode_prefetch_stages();  // 0 = no limit

// 2-D tensor map over a row-major [rows, inner] matrix with the 128-byte
// swizzle (mx_gemm.cu).
bool make_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows);

// ---- tile kernel over CTA pairs (mx_gemm_pair.cu) -----------------------------
constexpr int kTuneBmPair = 2;  // mx_set_tuning block_m value that asks for it
int max_active_pairs(bool scaled, bool swiglu);
bool plan_pair(const GemmProblem& pb, int sms, int max_ctas, GemmPlan* plan);
cudaError_t launch_pair(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st);

// ---- decode kernel (mx_decode.cu) -------------------------------------------
int decode_tokens_tile(int M, bool short_launch);
size_t decode_ws_bytes(int tiles, int nsub, int M);
bool plan_decode(const GemmProblem& pb, int split, int grid, int cluster, int per_sm, int sms, GemmPlan* plan);
cudaError_t launch_decode(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st);
void set_timeline(void* buf, size_t bytes);
constexpr int kTimelineCtaSlots = 16;  // per-CTA records ahead of the 4 x 64 per-stage detail
unsigned long long* timeline_buffer(int* ctas);  // installed trace buffer (null = off)
void set_launch_flags(unsigned flags);
unsigned launch_flags();

// Argument checks of mx_gemm (everything but the workspace); no CUDA calls.
mx_status validate_gemm(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                        const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out, int M,
                        int N, int K);

}  // namespace mxg
