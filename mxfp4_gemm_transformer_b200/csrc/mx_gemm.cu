// mx_gemm.cu -- the block-scaled projection GEMM for sm_100a.
//
//   out[m, n] = epilogue( sum_kb 2^(ea-127) 2^(eb-127) sum_{k in kb} a[m,k] w[n,k] )
//
// One warp-specialised kernel per (tile width, scaling, SwiGLU) choice:
//   warp 0      TMA producer: A tile 128 x 128 B and B tile BN x 128 B per
//               K-step (128 elements) into a multi-stage shared-memory ring.
//   warp 1      TMEM allocator and the single MMA-issuing thread:
//               tcgen05.mma kind::mxf8f6f4 (block scaled, e4m3 x e4m3 or
//               e4m3 x e2m1) or kind::f8f6f4 (per-row fp32 scales), M = 128,
//               N = BN, K = 32 per instruction, fp32 accumulators in TMEM.
//   warp 2      scale-factor producer: reads the row-major E8M0 scales, expands
//               32 x 32 weight blocks to per-row scales, and writes the
//               128-row chunks in the layout tcgen05.cp copies to TMEM
//               (byte (r % 32) * 16 + (r / 32) * 4 + kblock).
//   warps 4-11  epilogue: tcgen05.ld of the accumulator (thread = row, two
//               warps per TMEM lane quadrant taking alternate 32-column
//               chunks), per-row/column fp32 scales, bias, GELU-tanh or SwiGLU
//               in fp32, round to bf16, and a store transposed through the
//               warp's 2 KB of shared memory so that it covers whole row
//               segments.
// Accumulators are double-buffered in TMEM when they fit, so the epilogue of
// one tile overlaps the mainloop of the next (persistent CTAs, one per SM).
//
// When there are fewer output tiles than SMs (decode-sized M), K is split.
// With a large enough caller workspace every (tile, split) unit writes its
// fp32 partial tile there and bumps the tile's counter; the CTA that arrives
// last sums the partials in split order (deterministic), runs the epilogue
// and resets the counter, so no CTA ever waits for another.  Without that
// workspace the splits of a tile form a thread-block cluster instead: every
// CTA parks its partial in its own shared memory and each reduces a slice of
// columns over distributed shared memory, in fixed rank order.
//
// Every wait is bounded (%globaltimer): a wait that runs out sets a bit in the
// caller's workspace status word, tells the other roles to stop, and the
// kernel tears down normally.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mx_internal.h"
#include "mx_ptx.cuh"
#include "mx_kernel_common.cuh"

namespace mxg {

struct GemmArgs {
    CUtensorMap tmA;    // e4m3 codes [M, K], box {128, rows}
    CUtensorMap tmB;    // W codes [N, K], box {128, rows per load}
    const uint8_t* sa;   // E8M0 [M, K/32]
    const uint8_t* sb;   // E8M0 [N/32, K/32] or [N, K/32]
    const float* sxa;    // fp32 [M]
    const float* swb;    // fp32 [N]
    const float* bias;   // fp32 [N] or null
    __nv_bfloat16* out;  // [M, Nout]
    unsigned* status;
    float* part;                   // split-K partials [tiles][splits][part_rows][BN] (workspace mode)
    unsigned* counters;            // per-tile arrival counters, zero between launches
    unsigned long long* timeline;  // optional per-CTA %globaltimer stamps (null = off)
    int prefetch_w;                // weights may be read before the previous kernel completes
    int timeline_ctas;
    int M, N, K, Nout, KB, num_kb;
    int tiles_m, tiles_n, splits, units;
    int gsplit;     // K splits reduced through the workspace (else through a cluster)
    int part_rows;  // rows of one partial tile: min(tile rows, M)
    int b_fmt, epi, n_half;
    uint32_t idesc;
    uint32_t tx_bytes;
    // Grouped launch (routed experts), groups > 0: group g takes activation
    // rows g_row[g] .. g_row[g+1]-1 through weight rows g*N .. g*N+N-1 (and
    // bias g*N ..), and owns units g_unit[g] .. g_unit[g+1]-1 of the walk, its
    // M tiles times tiles_n; b_rows = every group's weight rows (load bound).
    int groups, b_rows;
    int g_row[kMaxGroups + 1];
    int g_unit[kMaxGroups + 1];
};

static_assert(sizeof(GemmArgs) <= 4096, "kernel parameters must fit the 4 KB parameter space");

// Where one output tile lies: activation rows m0 .. m_end-1 (m_end bounds the
// rows of its group), weight rows from b0, column tile tn, the group's bias.
struct TileXY {
    int m0, m_end, b0, tn;
    const float* bias;
};

__device__ __forceinline__ TileXY tile_xy(const GemmArgs& p, int tile, int bm)
{
    if (p.groups == 0) {
        const int tm = tile % p.tiles_m;
        return TileXY{tm * bm, p.M, 0, tile / p.tiles_m, p.bias};
    }
    // the group whose units hold this tile: the last g with g_unit[g] <= tile
    // (empty groups own no units, so a run of equal starts resolves to the
    // group after it)
    int lo = 0, hi = p.groups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.g_unit[mid] <= tile) lo = mid;
        else hi = mid;
    }
    const int r0 = p.g_row[lo], r1 = p.g_row[lo + 1];
    const int tiles_m = (r1 - r0 + bm - 1) / bm;
    const int local = tile - p.g_unit[lo];
    return TileXY{r0 + (local % tiles_m) * bm, r1, lo * p.N, local / tiles_m,
                  p.bias ? p.bias + static_cast<size_t>(lo) * p.N : nullptr};
}

// AR = rows of the activation tile loaded per stage:
//   64   decode (M <= 64): the MMA still reads 128 rows; accumulator rows >= 64
//        come from stale shared memory and are never stored; frees ring space;
//   128  one 128-row block per CTA tile;
//   256  two 128-row blocks per CTA tile sharing each B tile (two M = 128 MMAs
//        per K-step), halving the operand bytes each SM loads per FLOP.
template <int BN, int SC, bool SWIGLU, int AR = 128>
struct Cfg {
    static constexpr bool SCALED = SC != 0;  // E8M0 block scales (1: kind::mxf8f6f4, 2: kind::mxf4)
    static constexpr bool F4 = SC == 2;      // both operands packed e2m1, K = 64 per MMA
    static constexpr int MB = AR == 256 ? 2 : 1;  // 128-row MMA blocks per tile
    static constexpr int BM = 128 * MB;
    static constexpr int BK = 128;  // K elements per stage (128 bytes per row in smem)
    static constexpr int A_BYTES = AR * BK;
    static constexpr int B_BYTES = BN * BK;
    static constexpr int SFB_CHUNKS = (BN + 127) / 128;
    // K elements per stage: 128 one-byte codes per row, or 256 packed e2m1
    // (kind::mxf4), whose stage then carries two scale chunks of 4 K blocks
    static constexpr int KPS = F4 ? 256 : 128;
    static constexpr int SF_CHUNK = 512 * (MB + SFB_CHUNKS);
    static constexpr int SF_BYTES = SCALED ? SF_CHUNK * (F4 ? 2 : 1) : 0;
    static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES + SF_BYTES + 1023) / 1024) * 1024;
    static constexpr int SMEM_LIMIT = 232448;
    // output staging: one 32 x 32 bf16 chunk per epilogue warp, transposed through
    // shared memory so that the global stores cover whole row segments (none for
    // the decode variants, which store directly)
    static constexpr int STAGING_BYTES = AR == 64 ? 0 : 8 * 2048;
    static constexpr int RESERVED = 1024 + 4096 + STAGING_BYTES + 1024;  // barriers, column params, staging, slack
    static constexpr int STAGES_FIT = (SMEM_LIMIT - RESERVED) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static constexpr int SF_COLS = SCALED ? 4 * MB + 4 * SFB_CHUNKS : 0;
    // TMEM: row blocks of one accumulator start on 32-column boundaries when
    // that fits; two accumulators (epilogue overlap) when they fit as well
    static constexpr int BN32 = (BN + 31) / 32 * 32;
    static constexpr int RB_STRIDE = ((MB - 1) * BN32 + BN + SF_COLS <= 512) ? BN32 : BN;
    static constexpr int ACC_COLS = (MB - 1) * RB_STRIDE + BN;  // columns of one accumulator
    static constexpr int ACC_BUFS = (2 * ((ACC_COLS + 31) / 32 * 32) + SF_COLS <= 512 ||
                                     2 * ACC_COLS + SF_COLS <= 512) ? 2 : 1;
    static constexpr int ACC_STRIDE = (ACC_BUFS == 2 && (ACC_COLS + 31) / 32 * 32 + ACC_COLS + SF_COLS <= 512)
                                          ? (ACC_COLS + 31) / 32 * 32
                                          : ACC_COLS;
    static constexpr int SF_BASE = (ACC_BUFS - 1) * ACC_STRIDE + ACC_COLS;
    static constexpr int COLS_USED = SF_BASE + SF_COLS;
    static constexpr int TMEM_COLS = COLS_USED <= 32    ? 32
                                     : COLS_USED <= 64  ? 64
                                     : COLS_USED <= 128 ? 128
                                     : COLS_USED <= 256 ? 256
                                                        : 512;
    static constexpr int OUT_COLS = SWIGLU ? BN / 2 : BN;
    static constexpr int RED_STRIDE = BN + 4;  // fp32 row stride of the split-K partial (bank spread)
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + RESERVED;
    static_assert(STAGES >= 2, "shared memory too small for two stages");
    static_assert(MB == 2 || 128 * RED_STRIDE * 4 <= STAGES * STAGE_BYTES, "cluster split-K partial must fit in the ring");
    static_assert(COLS_USED <= 512, "TMEM overflow");
};

// Per-CTA pipeline milestones (tracing; written only when a timeline buffer
// is installed with mx_debug_set_timeline).
enum Stamp {
    kStampStart = 0, kStampReady, kStampFirstTma, kStampFirstFull, kStampLastCommit, kStampAccFull,
    kStampTileDone, kStampClusterSync1, kStampReduced, kStampClusterSync2, kStampEnd, kStampSmid,
    kStampCount = 16
};
static_assert(kStampCount == kTimelineCtaSlots, "timeline layout");

// Per-stage detail for CTA 0 (first 64 K-steps it handles), stored after the
// per-CTA records: [0..63] TMA issued, [64..127] stage landed (MMA side),
// [128..191] MMAs committed, [192..255] scale copies issued.
__device__ __forceinline__ void stamp_stage(const GemmArgs& p, int row, int i)
{
    if (MXG_TRACE && p.timeline && i < 64 && blockIdx.x == 0 && blockIdx.y == 0)
        p.timeline[static_cast<size_t>(p.timeline_ctas) * kStampCount + row * 64 + i] = globaltimer_ns();
}

__device__ __forceinline__ void stamp(const GemmArgs& p, int which)
{
    if (MXG_TRACE && p.timeline) {
        const int cta = static_cast<int>(blockIdx.y * gridDim.x + blockIdx.x);
        if (cta < p.timeline_ctas) {
            unsigned long long v;
            if (which == kStampSmid) {
                uint32_t sm;
                asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
                v = sm;
            } else {
                v = globaltimer_ns();
            }
            p.timeline[cta * kStampCount + which] = v;
        }
    }
}

struct EpiCtx {
    int epi;
    bool f32row;
    float sx;  // per-row activation scale (fp32-row format)
    const float* swb;
    const float* bias;
    int n_half;
};

// Per-column parameters of one output column: bias of the gate/plain and up
// columns, and (fp32-row formats) the weight scales of both.
struct ColParams {
    float bg, bu, wg, wu;
};

template <bool SWIGLU>
__device__ __forceinline__ ColParams col_params(const EpiCtx& c, int n)
{
    ColParams cp{0.f, 0.f, 1.f, 1.f};
    if (c.bias) {
        cp.bg = __ldcg(c.bias + n);
        if (SWIGLU) cp.bu = __ldcg(c.bias + n + c.n_half);
    }
    if (c.f32row) {
        cp.wg = __ldcg(c.swb + n);
        if (SWIGLU) cp.wu = __ldcg(c.swb + n + c.n_half);
    }
    return cp;
}

template <bool SWIGLU>
__device__ __forceinline__ float epi_apply(const EpiCtx& c, float g, float u, const ColParams& cp)
{
    if (c.f32row) {
        g *= c.sx * cp.wg;
        if (SWIGLU) u *= c.sx * cp.wu;
    }
    if (SWIGLU) return sigmoid_mul(g + cp.bg, g + cp.bg) * (u + cp.bu);
    if (c.epi == MX_EPI_NONE) return g;
    g += cp.bg;
    return c.epi == MX_EPI_BIAS_GELU_TANH ? gelu_tanh(g) : g;
}

// value of output column n from gate/plain accumulator g and up accumulator u
template <bool SWIGLU>
__device__ __forceinline__ float epi_value(const EpiCtx& c, float g, float u, int n, float res = 0.f)
{
    if (c.f32row) {
        g *= c.sx * __ldcg(c.swb + n);
        if (SWIGLU) u *= c.sx * __ldcg(c.swb + n + c.n_half);
    }
    if (SWIGLU) {
        if (c.bias) {
            g += __ldcg(c.bias + n);
            u += __ldcg(c.bias + n + c.n_half);
        }
        return sigmoid_mul(g, g) * u;
    }
    if (c.epi == MX_EPI_NONE) return g;
    if (c.bias) g += __ldcg(c.bias + n);
    if (c.epi == MX_EPI_RESIDUAL) return g + res;
    return c.epi == MX_EPI_BIAS_GELU_TANH ? gelu_tanh(g) : g;
}

constexpr int kThreads = 128 + kEpiThreads;

// ---------------------------------------------------------------------------

template <int BN, int SC, bool SWIGLU, int AR>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmArgs p)
{
    using C = Cfg<BN, SC, SWIGLU, AR>;
    constexpr bool SCALED = C::SCALED;
    constexpr bool F4 = C::F4;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + C::STAGES;
    uint64_t* acc_full = empty + C::STAGES;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* final_bar = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_holder + 2);  // workspace split-K
    float* colp = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES + 1024);  // [4][256]
    uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES + 1024 + 4096;                  // [8 warps][2 KB]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool split_mode = p.splits > 1 && !p.gsplit;  // cluster reduction

    if (threadIdx.x == 0) {
        prefetch_tmap(&p.tmA);
        prefetch_tmap(&p.tmB);
        stamp(p, kStampStart);
        stamp(p, kStampSmid);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], SCALED ? 1 + 32 : 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    if (threadIdx.x == 0) stamp(p, kStampReady);
    const uint32_t tmem_sfa = tmem + C::SF_BASE;    // 4 columns per 128-row A block
    const uint32_t tmem_sfb = tmem_sfa + 4 * C::MB;  // 4 columns per 128-row B chunk

    // this CTA's units: persistent stride, or exactly one (tile, split) in a cluster
    const int u_first = split_mode ? static_cast<int>(blockIdx.y) * p.splits + static_cast<int>(cluster_ctarank())
                                   : static_cast<int>(blockIdx.x);
    const int u_step = split_mode ? p.units : static_cast<int>(gridDim.x);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_b = policy_evict_first();
            uint32_t stage = 0, phase = 0;
            int dbg_i = 0;
            // With weight prefetch allowed, the first ring's worth of weight
            // tiles is requested before waiting for the previous kernel; the
            // activation tiles of those stages follow once it has completed.
            int pre = 0;
            if (p.prefetch_w && u_first < p.units) {
                const int tile = u_first / p.splits, split = u_first % p.splits;
                const TileXY t = tile_xy(p, tile, C::BM);
                const int kb0 = split * p.num_kb / p.splits, kb1 = (split + 1) * p.num_kb / p.splits;
                pre = min(C::STAGES, kb1 - kb0);
                for (int i = 0; i < pre; ++i) {
                    const int kb = kb0 + i;
                    mbar_arrive_expect_tx(&full[i], p.tx_bytes);
                    uint8_t* sB = ring + i * C::STAGE_BYTES + C::A_BYTES;
                    if (SWIGLU) {
                        tma_load_2d(sB, &p.tmB, &full[i], kb * C::BK, t.b0 + t.tn * (BN / 2), pol_b);
                        tma_load_2d(sB + (BN / 2) * C::BK, &p.tmB, &full[i], kb * C::BK,
                                    t.b0 + p.n_half + t.tn * (BN / 2), pol_b);
                    } else {
                        tma_load_2d(sB, &p.tmB, &full[i], kb * C::BK, t.b0 + t.tn * BN, pol_b);
                    }
                }
            }
            pdl_wait();
            for (int u = u_first; u < p.units; u += u_step) {
                const int tile = u / p.splits, split = u % p.splits;
                const TileXY t = tile_xy(p, tile, C::BM);
                const int kb0 = split * p.num_kb / p.splits, kb1 = (split + 1) * p.num_kb / p.splits;
                for (int kb = kb0; kb < kb1; ++kb) {
                    uint8_t* sA = ring + stage * C::STAGE_BYTES;
                    uint8_t* sB = sA + C::A_BYTES;
                    if (pre > 0) {
                        // weights already requested; add the activation tile
                        --pre;
                        tma_load_2d(sA, &p.tmA, &full[stage], kb * C::BK, t.m0, pol_a);
                        if (u == u_first && kb == kb0) stamp(p, kStampFirstTma);
                        if (++stage == C::STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.status)) goto producer_done;
                    mbar_arrive_expect_tx(&full[stage], p.tx_bytes);
                    tma_load_2d(sA, &p.tmA, &full[stage], kb * C::BK, t.m0, pol_a);
                    if (u == u_first && kb == kb0) stamp(p, kStampFirstTma);
                    stamp_stage(p, 0, dbg_i++);
                    if (SWIGLU) {
                        tma_load_2d(sB, &p.tmB, &full[stage], kb * C::BK, t.b0 + t.tn * (BN / 2), pol_b);
                        tma_load_2d(sB + (BN / 2) * C::BK, &p.tmB, &full[stage], kb * C::BK,
                                    t.b0 + p.n_half + t.tn * (BN / 2), pol_b);
                    } else {
                        tma_load_2d(sB, &p.tmB, &full[stage], kb * C::BK, t.b0 + t.tn * BN, pol_b);
                    }
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        producer_done:;
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            int dbg_i = 0;
            for (int u = u_first; u < p.units; u += u_step) {
                const int split = u % p.splits;
                const int kb0 = split * p.num_kb / p.splits, kb1 = (split + 1) * p.num_kb / p.splits;
                if (!wait_bar(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status)) goto mma_done;
                tc_fence_after();
                const uint32_t d = tmem + acc * C::ACC_STRIDE;
                uint32_t accumulate = 0;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bar(&full[stage], phase, abort_flag, p.status)) goto mma_done;
                    tc_fence_after();
                    if (SCALED) fence_proxy_async_smem();
                    if (u == u_first && kb == kb0) stamp(p, kStampFirstFull);
                    stamp_stage(p, 1, dbg_i);
                    const uint32_t sA = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint32_t sB = sA + C::A_BYTES;
                    if (SCALED && !F4) {
                        const uint32_t sf = sB + C::B_BYTES;
#pragma unroll
                        for (int rb = 0; rb < C::MB; ++rb) tc_cp_32x128b_x4(tmem_sfa + 4 * rb, sdesc_sf(sf + 512 * rb));
#pragma unroll
                        for (int j = 0; j < C::SFB_CHUNKS; ++j)
                            tc_cp_32x128b_x4(tmem_sfb + 4 * j, sdesc_sf(sf + 512 * (C::MB + j)));
                    }
                    const int krem = p.K - kb * C::KPS;
                    const int ksteps = F4 ? (krem >= 256 ? 4 : krem / 64) : (krem >= C::BK ? 4 : krem / 32);
                    for (int kk = 0; kk < ksteps; ++kk) {
                        if (F4 && (kk & 1) == 0) {
                            // one scale chunk (4 K blocks of 32) per two K = 64 MMAs; the
                            // copy is ordered after the previous MMAs that read the columns
                            const uint32_t sf = sB + C::B_BYTES + (kk >> 1) * C::SF_CHUNK;
#pragma unroll
                            for (int rb = 0; rb < C::MB; ++rb)
                                tc_cp_32x128b_x4(tmem_sfa + 4 * rb, sdesc_sf(sf + 512 * rb));
#pragma unroll
                            for (int j = 0; j < C::SFB_CHUNKS; ++j)
                                tc_cp_32x128b_x4(tmem_sfb + 4 * j, sdesc_sf(sf + 512 * (C::MB + j)));
                        }
                        const uint64_t bd = sdesc_sw128(sB + kk * 32);
#pragma unroll
                        for (int rb = 0; rb < C::MB; ++rb) {
                            const uint64_t ad = sdesc_sw128(sA + rb * 16384 + kk * 32);
                            const uint32_t drb = d + rb * C::RB_STRIDE;
                            if (SCALED) {
                                // scale id: the byte (or, for kind::mxf4, the byte pair)
                                // of the chunk's 32-bit column this MMA's K blocks use
                                const uint32_t sid = F4 ? static_cast<uint32_t>((kk & 1) * 2) : static_cast<uint32_t>(kk);
                                const uint32_t id = p.idesc | (sid << 4) | (sid << 29);
                                if (F4) mma_mxf4(drb, ad, bd, id, tmem_sfa + 4 * rb, tmem_sfb, accumulate);
                                else mma_mx(drb, ad, bd, id, tmem_sfa + 4 * rb, tmem_sfb, accumulate);
                            } else {
                                mma_f8(drb, ad, bd, p.idesc, accumulate);
                            }
                        }
                        accumulate = 1;
                    }
                    tc_commit(&empty[stage]);
                    stamp_stage(p, 2, dbg_i++);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                tc_commit(&acc_full[acc]);
                stamp(p, kStampLastCommit);
                if (u + u_step >= p.units) pdl_launch_dependents();
                if (C::ACC_BUFS == 2) {
                    acc ^= 1u;
                    if (acc == 0) acc_phase ^= 1u;
                } else {
                    acc_phase ^= 1u;
                }
            }
        mma_done:;
        }
    } else if (warp == 2) {
        // ------------------------------------------------ scale-factor producer
        // Every lane fills 16 bytes of each 128-row chunk: rows lane + 32 g,
        // bytes g * 4 .. g * 4 + 3 = the stage's four 32-wide K blocks.  With
        // K % 128 == 0 the copies are asynchronous 4-byte cp.async (zero-fill
        // for rows past the end) and each lane's arrival is tied to their
        // completion; otherwise bytes are gathered with plain loads.
        if (SCALED) {
            uint32_t stage = 0, phase = 0;
            int dbg_i = 0;
            const int KB = p.KB;
            const bool vec4 = (KB & 3) == 0;
            auto issue_a = [&](uint8_t* sf, int m0, int k4) {
#pragma unroll
                for (int rb = 0; rb < C::MB; ++rb) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int m = m0 + rb * 128 + lane + 32 * g;
                        const bool ok = m < p.M;
                        const uint8_t* src = p.sa + static_cast<size_t>(ok ? m : 0) * KB + k4;
                        cp_async_4(sf + 512 * rb + lane * 16 + g * 4, src, ok ? 4u : 0u);
                    }
                }
            };
            auto b_row = [&](int r, const TileXY& t) {
                if (SWIGLU)
                    return t.b0 + ((r < BN / 2) ? t.tn * (BN / 2) + r : p.n_half + t.tn * (BN / 2) + (r - BN / 2));
                return t.b0 + t.tn * BN + r;
            };
            auto issue_b = [&](uint8_t* sf, const TileXY& t, int k4) {
#pragma unroll
                for (int j = 0; j < C::SFB_CHUNKS; ++j) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int r = 128 * j + lane + 32 * g;  // row within the B tile
                        const int n = b_row(r, t);
                        const bool ok = r < BN && n < p.b_rows;
                        const int nn = ok ? n : 0;
                        const uint8_t* src = (p.b_fmt == MX_B_E4M3_E8M0_32X32)
                                                 ? p.sb + static_cast<size_t>(nn >> 5) * KB + k4
                                                 : p.sb + static_cast<size_t>(nn) * KB + k4;
                        cp_async_4(sf + 512 * (C::MB + j) + lane * 16 + g * 4, src, ok ? 4u : 0u);
                    }
                }
            };
            // weight scales of the first ring's worth of stages may be requested
            // before the previous kernel completes (weight prefetch allowed)
            int pre = 0;
            if (vec4 && p.prefetch_w && u_first < p.units) {
                const int tile = u_first / p.splits, split = u_first % p.splits;
                const TileXY t = tile_xy(p, tile, C::BM);
                const int kb0 = split * p.num_kb / p.splits, kb1 = (split + 1) * p.num_kb / p.splits;
                pre = min(C::STAGES, kb1 - kb0);
                for (int i = 0; i < pre; ++i) {
                    uint8_t* sf = ring + i * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
                    const int kbase = (kb0 + i) * (C::KPS / 32);
#pragma unroll
                    for (int c = 0; c < (F4 ? 2 : 1); ++c)
                        if (kbase + 4 * c < KB) issue_b(sf + c * C::SF_CHUNK, t, kbase + 4 * c);
                }
            }
            pdl_wait();
            for (int u = u_first; u < p.units; u += u_step) {
                const int tile = u / p.splits, split = u % p.splits;
                const TileXY t = tile_xy(p, tile, C::BM);
                const int kb0 = split * p.num_kb / p.splits, kb1 = (split + 1) * p.num_kb / p.splits;
                for (int kb = kb0; kb < kb1; ++kb) {
                    uint8_t* sf = ring + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
                    const int k4 = kb * (C::KPS / 32);  // first 32-wide K block of this stage
                    if (pre > 0) {
                        --pre;
#pragma unroll
                        for (int c = 0; c < (F4 ? 2 : 1); ++c)
                            if (k4 + 4 * c < KB) issue_a(sf + c * C::SF_CHUNK, t.m0, k4 + 4 * c);
                        cp_async_arrive_noinc(&full[stage]);
                    } else {
                        if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.status)) goto sf_done;
                        if (F4) {
                            // two chunks of 4 K blocks; a chunk wholly past K is not
                            // read (its MMAs are not issued)
#pragma unroll
                            for (int c = 0; c < 2; ++c)
                                if (k4 + 4 * c < KB) {
                                    issue_a(sf + c * C::SF_CHUNK, t.m0, k4 + 4 * c);
                                    issue_b(sf + c * C::SF_CHUNK, t, k4 + 4 * c);
                                }
                            cp_async_arrive_noinc(&full[stage]);
                        } else if (vec4) {
                            issue_a(sf, t.m0, k4);
                            issue_b(sf, t, k4);
                            cp_async_arrive_noinc(&full[stage]);
                            if (lane == 0) stamp_stage(p, 3, dbg_i);
                            ++dbg_i;
                        } else {
                            uint32_t v[4];
#pragma unroll
                            for (int rb = 0; rb < C::MB; ++rb) {
#pragma unroll
                                for (int g = 0; g < 4; ++g) {
                                    const int m = t.m0 + rb * 128 + lane + 32 * g;
                                    uint32_t w = 0;
                                    if (m < p.M) {
                                        const uint8_t* src = p.sa + static_cast<size_t>(m) * KB + k4;
#pragma unroll
                                        for (int j = 0; j < 4; ++j)
                                            if (k4 + j < KB) w |= static_cast<uint32_t>(__ldcg(src + j)) << (8 * j);
                                    }
                                    v[g] = w;
                                }
                                *reinterpret_cast<uint4*>(sf + 512 * rb + lane * 16) = make_uint4(v[0], v[1], v[2], v[3]);
                            }
#pragma unroll
                            for (int j = 0; j < C::SFB_CHUNKS; ++j) {
#pragma unroll
                                for (int g = 0; g < 4; ++g) {
                                    const int r = 128 * j + lane + 32 * g;
                                    const int n = b_row(r, t);
                                    uint32_t w = 0;
                                    if (r < BN && n < p.b_rows) {
                                        const uint8_t* src = (p.b_fmt == MX_B_E4M3_E8M0_32X32)
                                                                 ? p.sb + static_cast<size_t>(n >> 5) * KB + k4
                                                                 : p.sb + static_cast<size_t>(n) * KB + k4;
#pragma unroll
                                        for (int jj = 0; jj < 4; ++jj)
                                            if (k4 + jj < KB) w |= static_cast<uint32_t>(__ldcg(src + jj)) << (8 * jj);
                                    }
                                    v[g] = w;
                                }
                                *reinterpret_cast<uint4*>(sf + 512 * (C::MB + j) + lane * 16) =
                                    make_uint4(v[0], v[1], v[2], v[3]);
                            }
                            fence_proxy_async_smem();
                            mbar_arrive(&full[stage]);
                        }
                    }
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        sf_done:;
        }
    } else if (warp >= 4) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quadrant this warp may read
        const int half = (warp - 4) >> 2;   // which alternate 32-column chunks it takes
        const int et = threadIdx.x - 128;   // index among the epilogue threads
        const int row = q * 32 + lane;
        uint32_t acc = 0, acc_phase = 0;
        pdl_wait();
        const bool f32row = !SCALED;
        for (int u = u_first; u < p.units; u += u_step) {
            const int tile = u / p.splits;
            const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
            const bool ready = wait_bar(&acc_full[acc], acc_phase, abort_flag, p.status);
            // All epilogue warps meet here every tile, whether or not their wait
            // succeeded, and leave together: the barrier ORs every thread's
            // "stop" so the decision is uniform and no warp is left waiting on
            // a later barrier.  It also means every warp is done with the
            // previous tile's column parameters.
            if (named_bar_or(1, kEpiThreads, !ready || *abort_flag)) break;
            tc_fence_after();
            if (threadIdx.x == 128) stamp(p, kStampAccFull);
            if (split_mode) {
                // park the fp32 partial (valid rows only) for the cluster reduction
                const int m = tm * C::BM + row;
                if (half == 0 && tm * C::BM + q * 32 < p.M) {
                    const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
                    float* red = reinterpret_cast<float*>(ring);
                    for (int c = 0; c < BN; c += 32) {
                        uint32_t g[32];
                        tmem_ld32(taddr + c, g);
                        tmem_ld_wait();
                        if (m < p.M) {
                            float4* dst = reinterpret_cast<float4*>(red + row * C::RED_STRIDE + c);
                            const int c4 = min(32, BN - c) / 4;  // float4s of this chunk inside the tile
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (j < c4)
                                    dst[j] = make_float4(__uint_as_float(g[4 * j]), __uint_as_float(g[4 * j + 1]),
                                                         __uint_as_float(g[4 * j + 2]), __uint_as_float(g[4 * j + 3]));
                        }
                    }
                }
                break;  // one unit per CTA in split mode
            }
            if (p.gsplit) {
                // write this unit's fp32 partial, free the accumulator, count the
                // arrival; the tile's last arrival reduces
                const int split = u % p.splits;
                const int rows_valid = min(C::BM, p.M - tm * C::BM);
                float* dst = p.part + static_cast<size_t>(tile * p.splits + split) * p.part_rows * BN;
#pragma unroll 1
                for (int rb = 0; rb < C::MB; ++rb) {
                    if (rb * 128 + q * 32 >= rows_valid) continue;  // warp-uniform: no valid row
                    const int r = rb * 128 + row;
                    const uint32_t taddr =
                        tmem + acc * C::ACC_STRIDE + rb * C::RB_STRIDE + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
                    for (int c = half * 32; c < BN; c += 64) {
                        uint32_t g[32];
                        tmem_ld32(taddr + c, g);
                        tmem_ld_wait();
                        if (r < rows_valid) {
                            float4* d4 = reinterpret_cast<float4*>(dst + static_cast<size_t>(r) * BN + c);
                            const int c4 = min(32, BN - c) / 4;  // float4s of this chunk inside the tile
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (j < c4)
                                    d4[j] = make_float4(__uint_as_float(g[4 * j]), __uint_as_float(g[4 * j + 1]),
                                                        __uint_as_float(g[4 * j + 2]), __uint_as_float(g[4 * j + 3]));
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[acc]);
                if (C::ACC_BUFS == 2) {
                    acc ^= 1u;
                    if (acc == 0) acc_phase ^= 1u;
                } else {
                    acc_phase ^= 1u;
                }
                __threadfence();  // this thread's partial is visible device-wide before the count
                named_bar_sync(1, kEpiThreads);
                if (et == 0) {
                    const unsigned before = atomicAdd(p.counters + tile, 1u);
                    const bool last = before == static_cast<unsigned>(p.splits - 1);
                    if (last) p.counters[tile] = 0u;  // every split of the tile has arrived: reset
                    *last_flag = last ? 1 : 0;
                }
                named_bar_sync(1, kEpiThreads);
                if (*last_flag) {
                    __threadfence();
                    const int G = C::OUT_COLS / 4;  // groups of 4 output columns
                    const float* base = p.part + static_cast<size_t>(tile) * p.splits * p.part_rows * BN;
                    const size_t sstride = static_cast<size_t>(p.part_rows) * BN;
                    EpiCtx ec{p.epi, !SCALED, 1.0f, p.swb, p.bias, p.n_half};
                    for (int e = et; e < rows_valid * G; e += kEpiThreads) {
                        const int r = e / G;
                        const int col = (e % G) * 4;
                        const int n0 = tn * C::OUT_COLS + col;
                        if (n0 >= p.Nout) continue;
                        const float* src = base + static_cast<size_t>(r) * BN + col;
                        float4 sg = make_float4(0.f, 0.f, 0.f, 0.f), su = make_float4(0.f, 0.f, 0.f, 0.f);
                        // up to 8 (SwiGLU: 4) splits' loads in flight, added in split order
                        constexpr int kBatch = SWIGLU ? 4 : 8;
                        for (int s0 = 0; s0 < p.splits; s0 += kBatch) {
                            float4 v[kBatch], w[kBatch];
#pragma unroll
                            for (int i = 0; i < kBatch; ++i) {
                                if (s0 + i < p.splits) {
                                    const float* ps = src + static_cast<size_t>(s0 + i) * sstride;
                                    v[i] = __ldcg(reinterpret_cast<const float4*>(ps));
                                    if (SWIGLU) w[i] = __ldcg(reinterpret_cast<const float4*>(ps + BN / 2));
                                }
                            }
#pragma unroll
                            for (int i = 0; i < kBatch; ++i) {
                                if (s0 + i < p.splits) {
                                    sg.x += v[i].x; sg.y += v[i].y; sg.z += v[i].z; sg.w += v[i].w;
                                    if (SWIGLU) { su.x += w[i].x; su.y += w[i].y; su.z += w[i].z; su.w += w[i].w; }
                                }
                            }
                        }
                        const int m = tm * C::BM + r;
                        if (!SCALED) ec.sx = __ldcg(p.sxa + m);
                        const float gv[4] = {sg.x, sg.y, sg.z, sg.w};
                        const float uv[4] = {su.x, su.y, su.z, su.w};
                        __nv_bfloat16* o = p.out + static_cast<size_t>(m) * p.Nout + n0;
                        if (n0 + 4 <= p.Nout && (p.Nout & 3) == 0) {
                            uint2 v2;
                            float rv[4] = {0.f, 0.f, 0.f, 0.f};
                            if (p.epi == MX_EPI_RESIDUAL) {
                                const uint2 q2 = *reinterpret_cast<const uint2*>(o);
                                rv[0] = __uint_as_float(q2.x << 16);
                                rv[1] = __uint_as_float(q2.x & 0xFFFF0000u);
                                rv[2] = __uint_as_float(q2.y << 16);
                                rv[3] = __uint_as_float(q2.y & 0xFFFF0000u);
                            }
                            v2.x = pack_bf16x2(epi_value<SWIGLU>(ec, gv[0], uv[0], n0, rv[0]),
                                               epi_value<SWIGLU>(ec, gv[1], uv[1], n0 + 1, rv[1]));
                            v2.y = pack_bf16x2(epi_value<SWIGLU>(ec, gv[2], uv[2], n0 + 2, rv[2]),
                                               epi_value<SWIGLU>(ec, gv[3], uv[3], n0 + 3, rv[3]));
                            *reinterpret_cast<uint2*>(o) = v2;
                        } else {
                            for (int j = 0; j < 4; ++j)
                                if (n0 + j < p.Nout) store_out(o + j, p.epi, epi_value<SWIGLU>(ec, gv[j], uv[j], n0 + j));
                        }
                    }
                }
                if (threadIdx.x == 128) stamp(p, kStampTileDone);
                continue;
            }
            // stage this tile's per-column parameters in shared memory
            const TileXY t = tile_xy(p, tile, C::BM);
            const int n_base = t.tn * C::OUT_COLS;
            for (int i = et; i < C::OUT_COLS; i += kEpiThreads) {
                const int n = n_base + i;
                const bool ok = n < p.Nout;
                colp[i] = (ok && t.bias) ? __ldcg(t.bias + n) : 0.f;
                colp[256 + i] = (SWIGLU && ok && t.bias) ? __ldcg(t.bias + n + p.n_half) : 0.f;
                colp[512 + i] = (f32row && ok) ? __ldcg(p.swb + n) : 1.f;
                colp[768 + i] = (SWIGLU && f32row && ok) ? __ldcg(p.swb + n + p.n_half) : 1.f;
            }
            named_bar_sync(1, kEpiThreads);
#pragma unroll 1
            for (int rb = 0; rb < C::MB; ++rb) {
                const int m = t.m0 + rb * 128 + row;
                if (t.m0 + rb * 128 + q * 32 >= t.m_end) continue;  // warp-uniform: no valid row
                const uint32_t taddr =
                    tmem + acc * C::ACC_STRIDE + rb * C::RB_STRIDE + (static_cast<uint32_t>(q * 32) << 16);
                const bool row_ok = m < t.m_end;
                const float sx = (f32row && row_ok) ? __ldcg(p.sxa + m) : 1.f;
                __nv_bfloat16* out_row = p.out + static_cast<size_t>(row_ok ? m : 0) * p.Nout + n_base;
#pragma unroll 1
                for (int c = half * 32; c < C::OUT_COLS; c += 64) {
                    uint32_t g[32], h[32];
                    tmem_ld32(taddr + c, g);
                    if (SWIGLU) tmem_ld32(taddr + BN / 2 + c, h);
                    tmem_ld_wait();
                    uint32_t pk[16];
                    if (SWIGLU) {
                        if (f32row) epi_chunk<MX_EPI_SWIGLU, true, true>(g, h, sx, colp, c, pk);
                        else epi_chunk<MX_EPI_SWIGLU, true, false>(g, h, sx, colp, c, pk);
                    } else if (p.epi == MX_EPI_BIAS_GELU_TANH) {
                        if (f32row) epi_chunk<MX_EPI_BIAS_GELU_TANH, false, true>(g, h, sx, colp, c, pk);
                        else epi_chunk<MX_EPI_BIAS_GELU_TANH, false, false>(g, h, sx, colp, c, pk);
                    } else if (p.epi == MX_EPI_BIAS) {
                        if (f32row) epi_chunk<MX_EPI_BIAS, false, true>(g, h, sx, colp, c, pk);
                        else epi_chunk<MX_EPI_BIAS, false, false>(g, h, sx, colp, c, pk);
                    } else if (p.epi == MX_EPI_RESIDUAL) {
                        float res[32];
                        load_row32_bf16(p.out, p.Nout, t.m_end, m, n_base + c,
                                        min(min(32, C::OUT_COLS - c), p.Nout - (n_base + c)), res);
                        if (f32row) epi_chunk_residual<true>(g, sx, colp, c, res, pk);
                        else epi_chunk_residual<false>(g, sx, colp, c, res, pk);
                    } else {
                        if (f32row) epi_chunk<MX_EPI_NONE, false, true>(g, h, sx, colp, c, pk);
                        else epi_chunk<MX_EPI_NONE, false, false>(g, h, sx, colp, c, pk);
                    }
                    const int cw = min(32, C::OUT_COLS - c);  // columns of this chunk in the tile
                    const int n_left = p.Nout - (n_base + c);
                    if (C::STAGING_BYTES > 0) {
                        store_chunk_staged(staging + (warp - 4) * 2048, pk, lane, p.out, p.Nout, t.m_end,
                                           t.m0 + rb * 128 + q * 32, n_base + c, min(cw, n_left));
                    } else if (row_ok) {
                        if (cw == 32 && n_left >= 32 && (p.Nout & 7) == 0) {
                            uint4* d4 = reinterpret_cast<uint4*>(out_row + c);
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4)
                                d4[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                        } else {
                            for (int j = 0; j < cw && j < n_left; ++j) {
                                const uint32_t w2 = pk[j >> 1];
                                reinterpret_cast<uint16_t*>(out_row)[c + j] =
                                    static_cast<uint16_t>((j & 1) ? (w2 >> 16) : (w2 & 0xFFFFu));
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            if (threadIdx.x == 128) stamp(p, kStampTileDone);
            if (C::ACC_BUFS == 2) {
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
    }
    __syncwarp();

    if (split_mode) {
        // every CTA of the cluster has parked its partial
        cluster_sync_all();
        if (threadIdx.x == 128) stamp(p, kStampClusterSync1);
        if (warp >= 4 && !*abort_flag) {
            const int tile = static_cast<int>(blockIdx.y);
            const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
            const int rank = static_cast<int>(cluster_ctarank());
            const int rows = min(C::BM, p.M - tm * C::BM);
            const int U = C::OUT_COLS / 4;  // groups of 4 output columns
            const int u0 = rank * U / p.splits, u1 = (rank + 1) * U / p.splits;
            const int width = u1 - u0;
            const uint32_t red_s = smem_u32(ring);
            const int t = threadIdx.x - 128;
            for (int e = t; e < rows * width; e += kEpiThreads) {
                const int r = e / width;
                const int col = (u0 + e % width) * 4;
                float4 s = make_float4(0.f, 0.f, 0.f, 0.f), su = make_float4(0.f, 0.f, 0.f, 0.f);
                const uint32_t off = static_cast<uint32_t>((r * C::RED_STRIDE + col) * 4);
                // issue the remote loads of up to 8 peers back to back, then add
                // them in rank order (the sum order is fixed: deterministic)
                for (int p0 = 0; p0 < p.splits; p0 += 8) {
                    float4 v[8], w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (p0 + i < p.splits) {
                            const uint32_t base = map_peer_smem(red_s, static_cast<uint32_t>(p0 + i));
                            v[i] = ld_dsmem_f4(base + off);
                            if (SWIGLU) w[i] = ld_dsmem_f4(base + off + static_cast<uint32_t>((BN / 2) * 4));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (p0 + i < p.splits) {
                            s.x += v[i].x; s.y += v[i].y; s.z += v[i].z; s.w += v[i].w;
                            if (SWIGLU) { su.x += w[i].x; su.y += w[i].y; su.z += w[i].z; su.w += w[i].w; }
                        }
                    }
                }
                const int m = tm * C::BM + r;
                EpiCtx ec{p.epi, !SCALED, 1.0f, p.swb, p.bias, p.n_half};
                if (!SCALED) ec.sx = __ldcg(p.sxa + m);
                const int n0 = tn * C::OUT_COLS + col;
                const float gv[4] = {s.x, s.y, s.z, s.w};
                const float uv[4] = {su.x, su.y, su.z, su.w};
                __nv_bfloat16* dst = p.out + static_cast<size_t>(m) * p.Nout + n0;
                if (n0 + 4 <= p.Nout && (p.Nout & 3) == 0) {
                    uint2 o;
                    float rv[4] = {0.f, 0.f, 0.f, 0.f};
                    if (p.epi == MX_EPI_RESIDUAL) {
                        const uint2 q2 = *reinterpret_cast<const uint2*>(dst);
                        rv[0] = __uint_as_float(q2.x << 16);
                        rv[1] = __uint_as_float(q2.x & 0xFFFF0000u);
                        rv[2] = __uint_as_float(q2.y << 16);
                        rv[3] = __uint_as_float(q2.y & 0xFFFF0000u);
                    }
                    o.x = pack_bf16x2(epi_value<SWIGLU>(ec, gv[0], uv[0], n0, rv[0]),
                                      epi_value<SWIGLU>(ec, gv[1], uv[1], n0 + 1, rv[1]));
                    o.y = pack_bf16x2(epi_value<SWIGLU>(ec, gv[2], uv[2], n0 + 2, rv[2]),
                                      epi_value<SWIGLU>(ec, gv[3], uv[3], n0 + 3, rv[3]));
                    *reinterpret_cast<uint2*>(dst) = o;
                } else {
                    for (int j = 0; j < 4; ++j)
                        if (n0 + j < p.Nout) store_out(dst + j, p.epi, epi_value<SWIGLU>(ec, gv[j], uv[j], n0 + j));
                }
            }
        }
        if (threadIdx.x == 128) stamp(p, kStampReduced);
        // nobody leaves while a peer may still read its shared memory
        cluster_sync_all();
        if (threadIdx.x == 128) stamp(p, kStampClusterSync2);
    }

    // ---------------------------------------------------- teardown
    __syncthreads();
    if (threadIdx.x == 0) stamp(p, kStampEnd);
    if (warp == 1) {
        if (lane == 0) {
            // every MMA this thread issued has completed before TMEM is freed
            tc_commit(final_bar);
            wait_bar_final(final_bar, 0, p.status);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// watchdog probe: waits on a barrier nobody arrives on, gives up, reports.

__global__ void watchdog_probe_kernel(unsigned* status, unsigned long long timeout_ns)
{
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
        if (globaltimer_ns() - t0 > timeout_ns) {
            atomicOr(status, kStatusTimeout);
            break;
        }
    }
}

cudaError_t launch_watchdog_probe(unsigned* status, unsigned timeout_us, cudaStream_t st)
{
    watchdog_probe_kernel<<<1, 32, 0, st>>>(status, static_cast<unsigned long long>(timeout_us) * 1000ull);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// host side: tensor maps, planning, launch

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

bool make_map(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int g_tune_bn = 0, g_tune_splits = 0, g_tune_ctas = 0, g_tune_bm = 0;
int g_dec_mode = 0, g_dec_ctas = 0, g_dec_per_sm = 0, g_dec_prefetch = 0, g_dec_split = 0, g_dec_cluster = 0;
unsigned g_launch_flags = MX_LAUNCH_PDL;
unsigned long long* g_timeline = nullptr;
int g_timeline_ctas = 0;

// Kernel attributes are per device: set them the first time a device uses
// this kernel (before any stream capture, since the first call is eager).
template <int BN, int SC, bool SWIGLU, int AR>
cudaError_t prepare_kernel()
{
    using C = Cfg<BN, SC, SWIGLU, AR>;
    auto kern = gemm_kernel<BN, SC, SWIGLU, AR>;
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && !done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

// The compiled variants: (tile width, activation rows) x scaling (sc: 0 fp32
// row / column scales, 1 E8M0 kind::mxf8f6f4, 2 E8M0 kind::mxf4 W4A4) x SwiGLU.
template <class Op>
auto dispatch(int bn, int ar, int sc, bool swiglu, Op op) -> decltype(op.template run<128, 1, false, 128>())
{
#define MXG_DISPATCH(B, A)                                                                                    \
    if (bn == B && ar == A && sc != 2)                                                                        \
        return sc ? (swiglu ? op.template run<B, 1, true, A>() : op.template run<B, 1, false, A>())             \
                  : (swiglu ? op.template run<B, 0, true, A>() : op.template run<B, 0, false, A>());
#define MXG_DISPATCH_F4(B, A)                                                                                 \
    if (bn == B && ar == A && sc == 2) return swiglu ? op.template run<B, 2, true, A>() : op.template run<B, 2, false, A>();
    MXG_DISPATCH(64, 128)
    MXG_DISPATCH(128, 128)
    MXG_DISPATCH(240, 128)
    MXG_DISPATCH(256, 128)
    MXG_DISPATCH(128, 64)
    MXG_DISPATCH(256, 64)
    MXG_DISPATCH(240, 256)
    MXG_DISPATCH_F4(240, 128)
    MXG_DISPATCH_F4(256, 128)
    MXG_DISPATCH_F4(240, 256)
#undef MXG_DISPATCH
#undef MXG_DISPATCH_F4
    return op.invalid();
}

struct AccBufsOp {
    template <int BN, int SC, bool SWIGLU, int AR>
    int run() const { return Cfg<BN, SC, SWIGLU, AR>::ACC_BUFS; }
    int invalid() const { return 0; }
};

struct RingOp {
    template <int BN, int SC, bool SWIGLU, int AR>
    long long run() const
    {
        return static_cast<long long>(Cfg<BN, SC, SWIGLU, AR>::STAGES) * Cfg<BN, SC, SWIGLU, AR>::STAGE_BYTES;
    }
    long long invalid() const { return 0; }
};

// How many clusters of `cluster` CTAs of a kernel variant the device runs at
// once (cached per device, variant and cluster size).
struct ClustersOp {
    int cluster;
    template <int BN, int SC, bool SWIGLU, int AR>
    int run() const
    {
        using C = Cfg<BN, SC, SWIGLU, AR>;
        static std::mutex mu;
        static int cache[64][17] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64 || cluster < 1 || cluster > 16) return 0;
        {
            std::lock_guard<std::mutex> lk(mu);
            if (cache[dev][cluster]) return cache[dev][cluster];
        }
        if (prepare_kernel<BN, SC, SWIGLU, AR>() != cudaSuccess) return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cluster * 64, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<BN, SC, SWIGLU, AR>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        std::lock_guard<std::mutex> lk(mu);
        cache[dev][cluster] = n > 0 ? n : -1;
        return n;
    }
    int invalid() const { return 0; }
};

int max_active_clusters_for(int bn, int ar, int sc, bool swiglu, int cluster)
{
    return dispatch(bn, ar, sc, swiglu, ClustersOp{cluster});
}

// Whether the parked split-K partial (rows x (BN + 4) fp32) fits in the ring.
bool split_fits(int bn, int ar, int sc, bool swiglu, int rows)
{
    const long long ring = dispatch(bn, ar, sc, swiglu, RingOp{});
    return ring > 0 && static_cast<long long>(rows) * (bn + 4) * 4 <= ring;
}

struct LaunchOp {
    const GemmArgs* args;
    const GemmPlan* plan;
    cudaStream_t st;
    template <int BN, int SC, bool SWIGLU, int AR>
    cudaError_t run() const
    {
        using C = Cfg<BN, SC, SWIGLU, AR>;
        auto kern = gemm_kernel<BN, SC, SWIGLU, AR>;
        cudaError_t e = prepare_kernel<BN, SC, SWIGLU, AR>();
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(plan->grid_x, plan->grid_y, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        int na = 0;
        if (plan->splits > 1 && !plan->gsplit) {
            attr[na].id = cudaLaunchAttributeClusterDimension;
            attr[na].val.clusterDim.x = plan->splits;
            attr[na].val.clusterDim.y = 1;
            attr[na].val.clusterDim.z = 1;
            ++na;
        }
        if (launch_flags() & MX_LAUNCH_PDL) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        return cudaLaunchKernelEx(&cfg, kern, *args);
    }
    cudaError_t invalid() const { return cudaErrorInvalidValue; }
};


struct StagesOp {
    template <int BN, int SC, bool SWIGLU, int AR>
    int run() const { return Cfg<BN, SC, SWIGLU, AR>::STAGES; }
    int invalid() const { return 0; }
};

}  // namespace

bool make_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows)
{
    return make_map(tm, dt, base, inner, rows, row_bytes, box_inner, box_rows);
}

void set_decode_tuning(int mode, int ctas, int per_sm, int prefetch_stages, int split, int cluster)
{
    g_dec_mode = mode;
    g_dec_ctas = ctas;
    g_dec_per_sm = per_sm;
    g_dec_prefetch = prefetch_stages;
    g_dec_split = split;
    g_dec_cluster = cluster;
}

int decode_prefetch_stages() { return g_dec_prefetch; }

// Buffer layout: per-CTA records of kStampCount slots, then the 256-slot
// per-stage detail of CTA 0 at the very end; the CTA count is what fits in
// front of it (a buffer too small for the detail disables tracing).
void set_timeline(void* buf, size_t bytes)
{
    const size_t slots = bytes / sizeof(unsigned long long);
    if (!buf || slots < 256 + kStampCount) {
        g_timeline = nullptr;
        g_timeline_ctas = 0;
        return;
    }
    g_timeline = static_cast<unsigned long long*>(buf);
    g_timeline_ctas = static_cast<int>((slots - 256) / kStampCount);
}

unsigned long long* timeline_buffer(int* ctas)
{
    *ctas = g_timeline_ctas;
    return g_timeline;
}

void set_launch_flags(unsigned flags) { g_launch_flags = flags; }
unsigned launch_flags() { return g_launch_flags; }

void set_tuning(int block_n, int splits, int max_ctas, int block_m)
{
    g_tune_bm = block_m;
    g_tune_bn = block_n;
    g_tune_splits = splits;
    g_tune_ctas = max_ctas;
}

// Workspace bytes of a workspace-reduced split plan.
size_t gsplit_ws_bytes(int tiles, int splits, int part_rows, int bn)
{
    const size_t counters = (static_cast<size_t>(tiles) * 4 + 255) / 256 * 256;
    return kWorkspaceHeader + counters + static_cast<size_t>(tiles) * splits * part_rows * bn * 4;
}

// Tile choice.  Large problems (at least as many output tiles as SMs) run
// persistent, one CTA per SM.  Smaller ones split K: through the workspace
// (partials + last-arrival reduction; any number of CTAs) when the caller's
// workspace holds the partials, else over a thread-block cluster (all of a
// tile's splits must fit on the device at once).  Among the tile widths and
// split counts, take the one with the lowest estimated time.
cudaError_t plan_gemm(const GemmProblem& pb, const DeviceInfo& dev, size_t ws_bytes, GemmPlan* plan)
{
    if (pb.epi == MX_EPI_SWIGLU_MXQ) {
        // The SwiGLU GEMM whose output is handed on as MX codes: quantised in
        // the decode kernel's epilogue (a warp's lanes hold one 1 x 32 block
        // of a token), else stored as bf16 into the workspace behind what the
        // plan needs and quantised from there by the activation quantiser.
        GemmProblem q = pb;
        q.epi = MX_EPI_SWIGLU;
        cudaError_t e = plan_gemm(q, dev, ws_bytes, plan);
        if (e != cudaSuccess) return e;
        if (plan->kernel == 1) {
            plan->out_quant = 1;
            return cudaSuccess;
        }
        const size_t tbytes = static_cast<size_t>(pb.M) * (pb.N / 2) * 2;
        const size_t avail = ws_bytes > tbytes + kWorkspaceHeader ? ws_bytes - tbytes : kWorkspaceHeader;
        *plan = GemmPlan();
        e = plan_gemm(q, dev, avail, plan);
        if (e != cudaSuccess) return e;
        plan->out_quant = 2;
        plan->out_off = (plan->ws_bytes + 255) / 256 * 256;
        plan->ws_bytes = plan->out_off + tbytes;
        return cudaSuccess;
    }
    if (pb.a_fmt == MX_A_BF16_E8M0_1X32) {
        // bf16 activations: the plan for the equivalent codes.  The codes are
        // made once, into the workspace behind what the plan needs, by the
        // quantisation kernel before the GEMM; the decode kernel can quantise
        // them itself, used while M x tiles <= kFusedQuantMaxWork and
        // whenever the workspace has no room for the codes (every tile's CTAs
        // then quantise the same tokens again, work that competes with the
        // MMA issue).
        GemmProblem q = pb;
        q.a_fmt = MX_A_E4M3_E8M0_1X32;
        cudaError_t e = plan_gemm(q, dev, ws_bytes, plan);
        if (e != cudaSuccess) return e;
        const bool fusable = plan->kernel == 1;  // the decode kernel quantises tokens
        if (fusable && static_cast<long long>(pb.M) * plan->tiles <= kFusedQuantMaxWork) {
            plan->act_quant = 1;
            return cudaSuccess;
        }
        const GemmPlan fused = *plan;
        const size_t qbytes = act_quant_bytes(pb.M, pb.K);
        const size_t avail = ws_bytes > qbytes + kWorkspaceHeader ? ws_bytes - qbytes : kWorkspaceHeader;
        *plan = GemmPlan();
        e = plan_gemm(q, dev, avail, plan);
        if (e != cudaSuccess) return e;
        plan->act_quant = 2;
        plan->quant_off = (plan->ws_bytes + 255) / 256 * 256;
        plan->ws_bytes = plan->quant_off + qbytes;
        // no room for the codes, or room only for a different kernel (e.g.
        // stream-K's accumulators no longer fit): quantise inside the decode
        // kernel the full workspace plans for
        if (fusable && (plan->ws_bytes > ws_bytes || plan->kernel != fused.kernel)) {
            *plan = fused;
            plan->act_quant = 1;
        }
        return cudaSuccess;
    }
    const bool swiglu = epi_swiglu(pb.epi);
    const int sc = pb.a_fmt == MX_A_E4M3_E8M0_1X32 ? 1 : (pb.a_fmt == MX_A_E2M1_E8M0_1X32 ? 2 : 0);
    const int nout = swiglu ? pb.N / 2 : pb.N;
    const int num_kb = (pb.K + 127) / 128;
    const int tiles_m = (pb.M + 127) / 128;
    const int sms = dev.sms > 0 ? dev.sms : 148;
    auto tiles_for = [&](int bn) {
        const int oc = swiglu ? bn / 2 : bn;
        return tiles_m * ((nout + oc - 1) / oc);
    };
    auto ar_for = [&](int bn) { return (pb.M <= 64 && (bn == 128 || bn == 256)) ? 64 : 128; };
    const int part_rows = std::min(pb.M, 128);

    // Decode-sized M: the decode kernel (weights on the MMA's 128-row side).
    // One CTA moves a 128-K block of weights only about every half
    // microsecond, so an SM needs two CTAs' pipelines to keep up with HBM:
    //  * fewer tiles than SMs (short, latency-bound launches): a tile's K
    //    range is split over a thread-block cluster, one CTA per SM, so the
    //    next launch's CTAs can start beside this one's;
    //  * otherwise about two CTAs per SM: a cluster of 2 per tile when the
    //    tiles alone cannot fill two per SM, else whole tiles over 2 x SMs
    //    CTAs.
    // All of these are deterministic and need no workspace; the stream-K
    // split (workspace atomics) is used only when asked for.
    const bool tuned = g_tune_bn != 0 || g_tune_splits != 0 || g_tune_bm != 0 || g_tune_ctas != 0;
    if (pb.M <= 64 && g_dec_mode >= 0 && (g_dec_mode >= 1 || !tuned) && sc != 2) {
        const bool det = (launch_flags() & MX_LAUNCH_DETERMINISTIC) != 0;
        const int nout_d = swiglu ? pb.N / 2 : pb.N;
        const int tiles_d = (nout_d + 127) / 128;
        const bool short_launch = tiles_d * 2 <= sms;
        const int grid = g_dec_ctas > 0 ? g_dec_ctas : (short_launch ? sms : 2 * sms);
        const int per_sm = g_dec_per_sm > 0 ? g_dec_per_sm : 2;
        int split = g_dec_split;
        if (split == kDecStreamK && det) split = kDecAuto;
        int cluster = g_dec_cluster > 0 ? g_dec_cluster
                                        : std::min(8, (short_launch ? sms : 2 * sms) / std::max(1, tiles_d));
        // A short launch whose CTAs would each stream many K blocks (the W4A8
        // down projection at M = 16: 40 tiles x 136 K blocks) fills two CTAs
        // per SM instead, in clusters of at most 6 (measured there: 15.2 us
        // against 23.8 us for clusters of 3, one CTA per SM; clusters of 7 at
        // two per SM ran at 25 us).
        const int num_kb_d = (pb.K + 127) / 128;
        if (g_dec_cluster == 0 && short_launch && num_kb_d > 16 * cluster)
            cluster = std::min(6, 2 * sms / std::max(1, tiles_d));
        GemmPlan dp;
        if ((split == kDecAuto || split == kDecCluster) && tiles_d * cluster <= 2 * sms &&
            plan_decode(pb, kDecCluster, grid, cluster, per_sm, sms, &dp)) {
            *plan = dp;
            return cudaSuccess;
        }
        dp = GemmPlan();
        if (split != kDecStreamK && plan_decode(pb, kDecWholeTiles, grid, 1, per_sm, sms, &dp) &&
            (dp.grid_x * 10 >= sms * 8 || split == kDecWholeTiles)) {
            *plan = dp;
            return cudaSuccess;
        }
        // too few whole tiles to fill the SMs and no cluster split: stream-K
        // when the workspace holds its accumulators (and results may depend on
        // the arrival order), else the tile kernel below
        dp = GemmPlan();
        if ((split == kDecStreamK || (split == kDecAuto && !det)) &&
            plan_decode(pb, kDecStreamK, grid, 1, per_sm, sms, &dp) && dp.ws_bytes <= ws_bytes) {
            *plan = dp;
            return cudaSuccess;
        }
    }

    // 256 x 240 tiles over CTA pairs (cta_group::2 MMAs), on request
    if (g_tune_bm == kTuneBmPair && g_tune_splits <= 1 && (g_tune_bn == 0 || g_tune_bn == 240) && sc != 2 &&
        plan_pair(pb, sms, g_tune_ctas, plan))
        return cudaSuccess;

    // An MMA instruction costs about the same issue time up to N = 128 and
    // only ~40% more at N = 256, so wide tiles are the most efficient; 240
    // keeps two accumulators (and the epilogue overlap) inside TMEM.
    int bn = 240;
    int splits = 1;
    int gsplit = 0;
    const bool forced_bn = g_tune_bn == 64 || g_tune_bn == 128 || g_tune_bn == 240 || g_tune_bn == 256;
    if (forced_bn) bn = g_tune_bn;
    if (g_tune_splits > 0) {
        splits = std::min(g_tune_splits, num_kb);
        if (splits > 1 && gsplit_ws_bytes(tiles_for(bn), splits, part_rows, bn) <= ws_bytes)
            gsplit = 1;
        else
            splits = std::min(splits, 16);
    } else if (tiles_m == 1 && tiles_for(bn) < sms && num_kb >= 2) {
        // Decode-sized M: the weights are streamed once.  Estimate each choice
        // as weight bytes per CTA over the slower of the CTA's MMA streaming
        // rate (weight bytes per MMA issue cycle: ~120 cycles per instruction
        // up to N = 128, ~171 at N = 256, K = 32 bytes) and its share of HBM,
        // plus the split-K tail: a fixed cost and, for the workspace
        // reduction, the partial bytes the last-arriving CTA reads.
        const double w_bytes = static_cast<double>(pb.N) * pb.K * (pb.b_fmt == MX_B_E2M1_E8M0_1X32 ? 0.5 : 1.0);
        const double hbm_bytes_per_cycle = 3400.0;  // ~6.5 TB/s at ~1.9 GHz, whole GPU
        const double reduce_bytes_per_cycle = 32.0;  // one CTA reading partials from L2
        double best = 1e30;
        int best_bn = forced_bn ? bn : 256, best_s = 1, best_g = 0;
        const int cands[3] = {256, 128, 64};
        for (int ci = 0; ci < 3; ++ci) {
            const int b = cands[ci];
            if (forced_bn && b != bn) continue;
            if (swiglu && b == 64) continue;
            const int t = tiles_for(b);
            if (t > sms) continue;
            const double mma_rate = (b >= 256 ? 256.0 * 32 / 171 : b * 32.0 / 120);
            for (int s = 1; s <= std::min(32, num_kb); ++s) {
                if (t * s > sms) break;
                const int ar = ar_for(b);
                const int ctas = t * s;
                const double rate = std::min(mma_rate, hbm_bytes_per_cycle / ctas);
                // up to half the SMs: the next launch's CTAs fit beside this
                // one's and stream their weights during its tail
                const double overlap = 2 * ctas <= sms ? 0.0 : 1500.0;
                const double stream = w_bytes / ctas / rate + overlap;
                // each reduction that is possible for this (width, splits)
                for (int g = 0; g < 2; ++g) {
                    double tail = 0.0;
                    if (s > 1 && g == 1) {
                        if (gsplit_ws_bytes(t, s, part_rows, b) > ws_bytes) continue;
                        tail = 3000.0 + static_cast<double>(s) * part_rows * b * 4 / reduce_bytes_per_cycle;
                    } else if (s > 1) {
                        if (s > 16) continue;
                        if (max_active_clusters_for(b, ar, sc, swiglu, s) < t) continue;
                        if (!split_fits(b, ar, sc, swiglu, pb.M)) continue;
                        tail = 2500.0 + static_cast<double>(part_rows) * b * 4 / reduce_bytes_per_cycle;
                    } else if (g == 1) {
                        continue;
                    }
                    const double cycles = stream + tail;
                    if (cycles < best * 0.97) {
                        best = cycles;
                        best_bn = b;
                        best_s = s;
                        best_g = g;
                    }
                }
            }
        }
        bn = best_bn;
        splits = best_s;
        gsplit = best_g;
    }
    if (splits < 1) splits = 1;
    if (sc == 2) {
        // W4A4 (kind::mxf4): compiled for 240- and 256-wide tiles of 128 or
        // 256 rows, without K splits
        bn = g_tune_bn == 256 ? 256 : 240;
        splits = 1;
    }
    if (splits == 1) gsplit = 0;

    // Tile height: two 128-row blocks per tile (halving operand bytes per FLOP)
    // when K is not split, the tile is 240 wide and there are at least as many
    // 256-row tiles as SMs; 64 loaded rows for decode-sized M.
    int a_rows = ar_for(bn);
    if (sc == 2) a_rows = 128;
    const int oc = swiglu ? bn / 2 : bn;
    const int tiles_n = (nout + oc - 1) / oc;
    const bool tall_ok = splits == 1 && bn == 240;
    if (g_tune_bm == 256 && tall_ok)
        a_rows = 256;
    else if (g_tune_bm == 0 && tall_ok && pb.M > 128 && ((pb.M + 255) / 256) * tiles_n >= sms)
        a_rows = 256;
    const int block_m = a_rows == 256 ? 256 : 128;
    const int tiles = ((pb.M + block_m - 1) / block_m) * tiles_n;

    plan->block_n = bn;
    plan->a_rows = a_rows;
    plan->block_m = block_m;
    plan->splits = splits;
    plan->gsplit = gsplit;
    plan->part_rows = gsplit ? part_rows : 0;
    plan->ws_bytes = gsplit ? gsplit_ws_bytes(tiles, splits, part_rows, bn) : kWorkspaceHeader;
    plan->units = tiles * splits;
    plan->acc_bufs = dispatch(bn, a_rows, sc, swiglu, AccBufsOp{});
    plan->stages = dispatch(bn, a_rows, sc, swiglu, StagesOp{});
    if (splits > 1 && !gsplit) {
        plan->grid_x = splits;
        plan->grid_y = tiles;
    } else {
        const int cap = g_tune_ctas > 0 ? std::min(g_tune_ctas, sms) : sms;
        plan->grid_x = std::min(plan->units, cap);
        plan->grid_y = 1;
    }
    return cudaSuccess;
}

// Grouped problems run on the tile kernel: tiles of 128 activation rows of
// one group by 240 weight rows (the variant with two accumulators, so one
// tile's epilogue overlaps the next tile's main loop), no K split, one
// persistent CTA per SM.  mx_set_tuning may pick 128 / 256 columns (240 / 256
// for W4A4) and cap the CTAs.
cudaError_t plan_gemm_grouped(const GemmProblem& pb, const DeviceInfo& dev, GemmPlan* plan)
{
    const bool swiglu = epi_swiglu(pb.epi);
    const int sc = pb.a_fmt == MX_A_E2M1_E8M0_1X32 ? 2 : 1;
    int bn = 240;
    if (g_tune_bn == 256 || (sc == 1 && g_tune_bn == 128)) bn = g_tune_bn;
    const int oc = swiglu ? bn / 2 : bn;
    const int tiles_n = ((swiglu ? pb.N / 2 : pb.N) + oc - 1) / oc;
    long long units = 0;
    for (int g = 0; g < pb.groups; ++g) units += (pb.offsets[g + 1] - pb.offsets[g] + 127) / 128 * tiles_n;
    if (units > (1LL << 30)) return cudaErrorInvalidValue;
    *plan = GemmPlan();
    plan->kernel = 0;
    plan->block_n = bn;
    plan->a_rows = 128;
    plan->block_m = 128;
    plan->splits = 1;
    plan->gsplit = 0;
    plan->units = static_cast<int>(units);
    plan->tiles = static_cast<int>(units);
    int grid = static_cast<int>(std::min<long long>(units, dev.sms));
    if (g_tune_ctas > 0) grid = std::min(grid, g_tune_ctas);
    plan->grid_x = std::max(grid, 1);
    plan->grid_y = 1;
    plan->ws_bytes = kWorkspaceHeader;
    plan->acc_bufs = dispatch(bn, 128, sc, swiglu, AccBufsOp{});
    plan->stages = dispatch(bn, 128, sc, swiglu, StagesOp{});
    return plan->acc_bufs > 0 ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_gemm(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st)
{
    if (plan.act_quant == 2) {
        // bf16 activations outside the decode kernel: quantise them into the
        // workspace, then the GEMM on those codes
        uint8_t* ws = reinterpret_cast<uint8_t*>(pb.status);
        uint8_t* codes = ws + plan.quant_off;
        uint8_t* scales = codes + (static_cast<size_t>(pb.M) * pb.K + 255) / 256 * 256;
        cudaError_t e = launch_quant_e8m0_1x32(pb.a_codes, pb.M, pb.K, codes, scales, st);
        if (e != cudaSuccess) return e;
        GemmProblem q = pb;
        q.a_fmt = MX_A_E4M3_E8M0_1X32;
        q.a_codes = codes;
        q.a_scales = scales;
        GemmPlan p2 = plan;
        p2.act_quant = 0;
        return launch_gemm(q, p2, st);
    }
    if (plan.out_quant == 2) {
        // SwiGLU into the workspace as bf16, then its 1 x 32 quantisation into
        // out (codes, then scales)
        uint8_t* ws = reinterpret_cast<uint8_t*>(pb.status);
        __nv_bfloat16* tmp = reinterpret_cast<__nv_bfloat16*>(ws + plan.out_off);
        GemmProblem q = pb;
        q.epi = MX_EPI_SWIGLU;
        q.out = tmp;
        GemmPlan p2 = plan;
        p2.out_quant = 0;
        cudaError_t e = launch_gemm(q, p2, st);
        if (e != cudaSuccess) return e;
        uint8_t* codes = static_cast<uint8_t*>(pb.out);
        return launch_quant_e8m0_1x32(tmp, pb.M, pb.N / 2, codes, codes + static_cast<size_t>(pb.M) * (pb.N / 2), st);
    }
    if (plan.kernel == 1) return launch_decode(pb, plan, st);
    if (plan.kernel == 3) return launch_pair(pb, plan, st);
    const bool swiglu = epi_swiglu(pb.epi);
    const int sc = pb.a_fmt == MX_A_E4M3_E8M0_1X32 ? 1 : (pb.a_fmt == MX_A_E2M1_E8M0_1X32 ? 2 : 0);
    const bool scaled = sc != 0;
    const int bn = plan.block_n;
    const int out_cols = swiglu ? bn / 2 : bn;

    GemmArgs a;
    memset(&a, 0, sizeof(a));
    const bool f4 = pb.a_fmt == MX_A_E2M1_E8M0_1X32;  // W4A4, kind::mxf4
    const uint32_t b_rows = swiglu ? bn / 2 : bn;
    // weight rows behind the map: every group's when the problems are grouped
    const uint64_t nb = pb.groups > 0 ? static_cast<uint64_t>(pb.groups) * pb.N : static_cast<uint64_t>(pb.N);
    if (f4) {
        // both operands packed two per byte, loaded as plain bytes: a 128-byte
        // row of a stage holds 256 K elements
        if (!make_map(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.a_codes, pb.K / 2, pb.M, pb.K / 2, 128,
                      static_cast<uint32_t>(plan.a_rows)) ||
            !make_map(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.b_codes, pb.K / 2, nb, pb.K / 2, 128, b_rows))
            return cudaErrorInvalidValue;
    } else if (!make_map(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.a_codes, pb.K, pb.M, pb.K, 128,
                         static_cast<uint32_t>(plan.a_rows))) {
        return cudaErrorInvalidValue;
    } else if (pb.b_fmt == MX_B_E2M1_E8M0_1X32) {
        if (!make_map(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, pb.b_codes, pb.K, nb, pb.K / 2, 128, b_rows))
            return cudaErrorInvalidValue;
    } else {
        if (!make_map(&a.tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.b_codes, pb.K, nb, pb.K, 128, b_rows))
            return cudaErrorInvalidValue;
    }
    a.b_rows = static_cast<int>(nb);
    if (pb.groups > 0) {
        // the group table: rows and first unit of every group (empty groups
        // own no units); tiles are block_m rows of one group by out_cols
        const int tiles_n = ((swiglu ? pb.N / 2 : pb.N) + out_cols - 1) / out_cols;
        int unit = 0;
        a.groups = pb.groups;
        for (int g = 0; g < pb.groups; ++g) {
            a.g_row[g] = pb.offsets[g];
            a.g_unit[g] = unit;
            unit += (pb.offsets[g + 1] - pb.offsets[g] + plan.block_m - 1) / plan.block_m * tiles_n;
        }
        a.g_row[pb.groups] = pb.offsets[pb.groups];
        a.g_unit[pb.groups] = unit;
        if (unit != plan.units) return cudaErrorInvalidValue;
    }
    a.sa = scaled ? static_cast<const uint8_t*>(pb.a_scales) : nullptr;
    a.sb = scaled ? static_cast<const uint8_t*>(pb.b_scales) : nullptr;
    a.sxa = scaled ? nullptr : static_cast<const float*>(pb.a_scales);
    a.swb = scaled ? nullptr : static_cast<const float*>(pb.b_scales);
    a.bias = pb.bias;
    a.out = static_cast<__nv_bfloat16*>(pb.out);
    a.status = pb.status;
    a.gsplit = plan.gsplit;
    a.part_rows = plan.part_rows;
    if (plan.gsplit) {
        uint8_t* ws = reinterpret_cast<uint8_t*>(pb.status);
        const int tiles = plan.units / plan.splits;
        a.counters = reinterpret_cast<unsigned*>(ws + kWorkspaceHeader);
        a.part = reinterpret_cast<float*>(ws + kWorkspaceHeader + (static_cast<size_t>(tiles) * 4 + 255) / 256 * 256);
    }
    a.timeline = g_timeline;
    a.prefetch_w = (g_launch_flags & MX_LAUNCH_PDL) && (g_launch_flags & MX_LAUNCH_PREFETCH_WEIGHTS) ? 1 : 0;
    a.timeline_ctas = g_timeline_ctas;
    a.M = pb.M;
    a.N = pb.N;
    a.K = pb.K;
    a.Nout = swiglu ? pb.N / 2 : pb.N;
    a.KB = pb.K / 32;
    a.num_kb = f4 ? (pb.K + 255) / 256 : (pb.K + 127) / 128;
    a.tiles_m = pb.groups > 0 ? 1 : (pb.M + plan.block_m - 1) / plan.block_m;
    a.tiles_n = (a.Nout + out_cols - 1) / out_cols;
    a.splits = plan.splits;
    a.units = plan.units;
    a.b_fmt = pb.b_fmt;
    a.epi = pb.epi;
    a.n_half = pb.N / 2;
    const uint32_t b_code = (pb.b_fmt == MX_B_E2M1_E8M0_1X32) ? 5u : 0u;  // e2m1 : e4m3
    if (f4)  // kind::mxf4: E2M1 is format 1 for both operands; K = 64 per MMA
        a.idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(bn >> 3) << 17) | (1u << 23) |
                  (static_cast<uint32_t>(128 >> 4) << 24);
    else if (scaled)
        a.idesc = (0u << 7) | (b_code << 10) | (static_cast<uint32_t>(bn >> 3) << 17) | (1u << 23) |
                  (static_cast<uint32_t>(128 >> 4) << 24);
    else
        a.idesc = (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(bn >> 3) << 17) |
                  (static_cast<uint32_t>(128 >> 4) << 24);
    // transaction bytes count the global-side size: a 128-element e2m1 row is
    // 64 bytes even though it lands as 128 bytes (16 codes + 8 pad bytes per
    // 16-byte chunk) in shared memory
    const uint32_t b_row_bytes = (pb.b_fmt == MX_B_E2M1_E8M0_1X32 && !f4) ? 64u : 128u;
    a.tx_bytes = static_cast<uint32_t>(plan.a_rows * 128) + static_cast<uint32_t>(bn) * b_row_bytes;

    return dispatch(bn, plan.a_rows, sc, swiglu, LaunchOp{&a, &plan, st});
}

}  // namespace mxg
