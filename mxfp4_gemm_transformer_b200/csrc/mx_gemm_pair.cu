// mx_gemm_pair.cu -- the block-scaled GEMM over CTA pairs (tcgen05 cta_group::2).
//
// The prefill / large-M path of the MX projection GEMM (sly README, Contents
// table, the MXFP4 / FP8 GEMM rows; GR00T page, fused-epilogue tier).  It
// computes the same thing as the tile kernel in mx_gemm.cu: out = epilogue(
// sum_k dec(A) dec(W)) with the E8M0 block scales applied inside the MMA, or
// the fp32 row / column scales in the epilogue.
//
// Layout of the work: an output tile is 256 rows x 240 MMA columns (for
// SwiGLU 120 gate + 120 up columns -> 120 outputs) and belongs to a cluster of
// two CTAs on two SMs.  CTA r holds rows r*128 .. r*128+127 of the tile's
// activations and MMA columns r*120 .. r*120+119 of its weights, one 128-wide
// K block per stage (16 KB + 15 KB, six stages); the even CTA issues M = 256,
// N = 240 MMAs that read both CTAs' shared memory and write the accumulator
// rows of each CTA into that CTA's TMEM.  Each SM therefore loads half the
// operand bytes of a 256 x 240 tile per FLOP, like the one-CTA 256-row tile,
// but with a ring twice as deep and a 128 x 240 accumulator per CTA, so two
// accumulators fit in TMEM and the epilogue of one tile runs under the main
// loop of the next.
//
// Warp roles (both CTAs unless noted):
//   warp 0      TMA: this CTA's A and B halves; completion is counted on the
//               even CTA's `full` barrier (which expects both CTAs' bytes);
//   warp 1      even CTA: MMA issue (scale copies, 4 MMAs per stage, commits
//               multicast to both CTAs' `empty` / `acc_full` barriers);
//               both: TMEM allocation;
//   warp 2      scale factors by cp.async into the tcgen05.cp layout: this
//               CTA's 128 A rows and all 240 B rows (the MMA reads the B
//               scales of every column from each CTA's TMEM);
//   warp 3      odd CTA: forwards the completion of its scale copies to the
//               even CTA's `full` barrier (cp.async can only signal a local
//               barrier);
//   warps 4-11  epilogue of this CTA's 128 rows, then a release of the
//               accumulator to the even CTA's `acc_empty` (16 arrivals).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "mx_internal.h"
#include "mx_kernel_common.cuh"
#include "mx_ptx.cuh"

namespace mxg {
namespace {

struct PairArgs {
    CUtensorMap tmA;     // e4m3 codes [M, K], box {128, 128}
    CUtensorMap tmB;     // W codes [N, K], box {128, 120}
    const uint8_t* sa;   // E8M0 [M, K/32]
    const uint8_t* sb;   // E8M0 [N/32, K/32] or [N, K/32]
    const float* sxa;    // fp32 [M]
    const float* swb;    // fp32 [N]
    const float* bias;   // fp32 [N] or null
    __nv_bfloat16* out;  // [M, Nout]
    unsigned* status;
    int prefetch_w;  // weights may be read before the previous kernel completes
    int M, N, K, Nout, KB, num_kb;
    int tiles_m, tiles;
    int b_fmt, epi, n_half;
    uint32_t idesc;
    uint32_t tx_bytes;  // both CTAs' A + B bytes of one stage
    unsigned long long* timeline;  // per-stage detail of the first pair (trace builds), null = off
};

// Trace builds: %globaltimer of the first 64 K-steps of the first pair, rows
// 0 even CTA's loads issued, 1 stage seen by the MMA thread, 2 its MMAs
// issued and committed, 3 odd CTA's scale copies forwarded.
__device__ __forceinline__ void pair_stamp(const PairArgs& p, int row, int i)
{
    if (MXG_TRACE && p.timeline && i < 64 && blockIdx.x < 2) p.timeline[row * 64 + i] = globaltimer_ns();
}

constexpr int kPairThreads = 128 + kEpiThreads;

template <bool SCALED, bool SWIGLU>
struct PairCfg {
    static constexpr int BN = 240;       // MMA columns of a tile
    static constexpr int BH = BN / 2;    // weight rows each CTA loads
    static constexpr int BK = 128;
    static constexpr int A_BYTES = 128 * BK;
    static constexpr int B_BYTES = BH * BK;
    static constexpr int SFB_CHUNKS = 2;  // B scales of all 240 columns, 128 rows a chunk
    static constexpr int SF_BYTES = SCALED ? 512 * (1 + SFB_CHUNKS) : 0;
    static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES + SF_BYTES + 1023) / 1024) * 1024;
    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int STAGING_BYTES = kEpiWarps * 2048;  // output transpose, 2 KB per epilogue warp
    static constexpr int RESERVED = 1024 + 4096 + STAGING_BYTES + 1024;  // barriers, column params, staging, slack
    static constexpr int STAGES_FIT = (SMEM_LIMIT - RESERVED) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static constexpr int ACC_STRIDE = 256;  // two accumulators of 240 columns
    static constexpr int SF_BASE = ACC_STRIDE + BN;
    static constexpr int TMEM_COLS = 512;
    static constexpr int OUT_COLS = SWIGLU ? BN / 2 : BN;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + RESERVED;
    static_assert(SF_BASE + (SCALED ? 4 + 4 * SFB_CHUNKS : 0) <= TMEM_COLS, "TMEM overflow");
    static_assert(STAGES >= 2, "shared memory too small for two stages");
    static_assert(3 * 8 * 8 + 5 * 8 + 16 <= 1024, "barrier block overflow");
};

template <bool SCALED, bool SWIGLU>
__global__ void __launch_bounds__(kPairThreads, 1) gemm_pair_kernel(const __grid_constant__ PairArgs p)
{
    using C = PairCfg<SCALED, SWIGLU>;
    extern __shared__ uint8_t smem_raw[];
    // Both CTAs run the same code with the same static shared memory, so the
    // aligned base (and every operand offset the pair MMA relies on) matches.
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* empty = full + 8;
    uint64_t* sf_full = empty + 8;      // odd CTA: its scale copies of a stage have landed
    uint64_t* acc_full = sf_full + 8;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* final_bar = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    float* colp = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES + 1024);  // [4][256]
    uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES + 1024 + 4096;                  // [8 warps][2 KB]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank() & 1u;
    const bool leader = rank == 0;
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int pairs = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        prefetch_tmap(&p.tmA);
        prefetch_tmap(&p.tmB);
        for (int s = 0; s < C::STAGES; ++s) {
            // even CTA: its producer's arrive.expect_tx (+ its scale warp's 32
            // cp.async arrivals + the odd CTA's forwarded one)
            mbar_init(&full[s], SCALED ? 1 + 32 + 1 : 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_full[s], 32);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * kEpiWarps);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    // both CTAs' barriers are initialised and TMEM allocated before any
    // cross-CTA arrival, copy or MMA
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint32_t tmem_sfa = tmem + C::SF_BASE;  // 4 columns: this CTA's 128 A rows
    const uint32_t tmem_sfb = tmem_sfa + 4;       // 4 columns per 128 B rows, all 240 rows
    // the even CTA's barriers, as shared::cluster addresses
    const uint32_t full_lead = map_peer_smem(smem_u32(full), 0);
    const uint32_t acc_empty_lead = map_peer_smem(smem_u32(acc_empty), 0);

    // weight rows (of W [N, K]) this CTA loads for tile column tn
    auto b_row0 = [&](int tn) {
        if (SWIGLU) return rank == 0 ? tn * C::BH : p.n_half + tn * C::BH;
        return tn * C::BN + static_cast<int>(rank) * C::BH;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_a = policy_evict_last();
            const uint64_t pol_b = policy_evict_first();
            uint32_t stage = 0, phase = 0;
            int pre = 0;
            if (p.prefetch_w && pair < p.tiles) {
                const int tn = pair / p.tiles_m;
                pre = min(C::STAGES, p.num_kb);
                for (int i = 0; i < pre; ++i) {
                    if (leader) mbar_arrive_expect_tx(&full[i], p.tx_bytes);
                    tma_load_2d_pair(ring + i * C::STAGE_BYTES + C::A_BYTES, &p.tmB, full_lead + 8u * i, i * C::BK,
                                     b_row0(tn), pol_b);
                }
            }
            pdl_wait();
            bool last_issued = false;
            int dbg_i = 0;
            for (int t = pair; t < p.tiles; t += pairs) {
                const int tm = t % p.tiles_m, tn = t / p.tiles_m;
                const int m0 = tm * 256 + static_cast<int>(rank) * 128;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    uint8_t* sA = ring + stage * C::STAGE_BYTES;
                    if (pre > 0) {
                        --pre;  // weights already requested; add the activation tile
                    } else {
                        if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.status)) goto producer_done;
                        if (leader) mbar_arrive_expect_tx(&full[stage], p.tx_bytes);
                        tma_load_2d_pair(sA + C::A_BYTES, &p.tmB, full_lead + 8u * stage, kb * C::BK, b_row0(tn),
                                         pol_b);
                    }
                    tma_load_2d_pair(sA, &p.tmA, full_lead + 8u * stage, kb * C::BK, m0, pol_a);
                    if (leader) pair_stamp(p, 0, dbg_i);
                    ++dbg_i;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (t + pairs >= p.tiles) last_issued = true;
            }
            // the odd CTA has no MMA thread: it lets the next kernel start once
            // its loads are out (the next kernel still waits for this one to
            // complete before reading its results)
            if (!leader && last_issued) pdl_launch_dependents();
        producer_done:;
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (leader && lane == 0) {
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            int dbg_i = 0;
            for (int t = pair; t < p.tiles; t += pairs) {
                if (!wait_bar(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status)) goto mma_done;
                tc_fence_after();
                const uint32_t d = tmem + acc * C::ACC_STRIDE;
                uint32_t accumulate = 0;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!wait_bar(&full[stage], phase, abort_flag, p.status)) goto mma_done;
                    tc_fence_after();
                    pair_stamp(p, 1, dbg_i);
                    const uint32_t sA = smem_u32(ring + stage * C::STAGE_BYTES);
                    const uint32_t sB = sA + C::A_BYTES;
                    if (SCALED) {
                        fence_proxy_async_smem();  // scale bytes were written by cp.async
                        const uint32_t sf = sB + C::B_BYTES;
                        tc_cp_32x128b_x4_pair(tmem_sfa, sdesc_sf(sf));
#pragma unroll
                        for (int j = 0; j < C::SFB_CHUNKS; ++j)
                            tc_cp_32x128b_x4_pair(tmem_sfb + 4 * j, sdesc_sf(sf + 512 * (1 + j)));
                    }
                    const int krem = p.K - kb * C::BK;
                    const int ksteps = krem >= C::BK ? 4 : krem / 32;
                    for (int kk = 0; kk < ksteps; ++kk) {
                        const uint64_t ad = sdesc_sw128(sA + kk * 32);
                        const uint64_t bd = sdesc_sw128(sB + kk * 32);
                        if (SCALED) {
                            const uint32_t id =
                                p.idesc | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29);
                            mma_mx_pair(d, ad, bd, id, tmem_sfa, tmem_sfb, accumulate);
                        } else {
                            mma_f8_pair(d, ad, bd, p.idesc, accumulate);
                        }
                        accumulate = 1;
                    }
                    tc_commit_pair_mc(&empty[stage], 0x3);
                    pair_stamp(p, 2, dbg_i++);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                tc_commit_pair_mc(&acc_full[acc], 0x3);
                if (t + pairs >= p.tiles) pdl_launch_dependents();
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            }
        mma_done:;
        }
    } else if (warp == 2) {
        // ------------------------------------------------ scale-factor producer
        // Lane l fills 16 bytes of each 128-row chunk: rows l + 32 g, bytes
        // 4 g .. 4 g + 3 = the stage's four 32-wide K blocks (the layout
        // tcgen05.cp.32x128b.warpx4 spreads over the TMEM lane quadrants).
        if (SCALED) {
            uint64_t* bar = leader ? full : sf_full;
            uint32_t stage = 0, phase = 0;
            const int KB = p.KB;
            const bool vec4 = (KB & 3) == 0;
            auto b_row = [&](int r, int tn) {  // W row of MMA column r of tile column tn
                if (SWIGLU) return (r < C::BH) ? tn * C::BH + r : p.n_half + tn * C::BH + (r - C::BH);
                return tn * C::BN + r;
            };
            auto b_src = [&](int n, int k4) {
                return (p.b_fmt == MX_B_E4M3_E8M0_32X32) ? p.sb + static_cast<size_t>(n >> 5) * KB + k4
                                                         : p.sb + static_cast<size_t>(n) * KB + k4;
            };
            auto issue_a = [&](uint8_t* sf, int m0, int k4) {
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int m = m0 + lane + 32 * g;
                    const bool ok = m < p.M;
                    cp_async_4(sf + lane * 16 + g * 4, p.sa + static_cast<size_t>(ok ? m : 0) * KB + k4, ok ? 4u : 0u);
                }
            };
            auto issue_b = [&](uint8_t* sf, int tn, int k4) {
#pragma unroll
                for (int j = 0; j < C::SFB_CHUNKS; ++j) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int r = 128 * j + lane + 32 * g;
                        const int n = b_row(r, tn);
                        const bool ok = r < C::BN && n < p.N;
                        cp_async_4(sf + 512 * (1 + j) + lane * 16 + g * 4, b_src(ok ? n : 0, k4), ok ? 4u : 0u);
                    }
                }
            };
            int pre = 0;
            if (vec4 && p.prefetch_w && pair < p.tiles) {
                const int tn = pair / p.tiles_m;
                pre = min(C::STAGES, p.num_kb);
                for (int i = 0; i < pre; ++i) issue_b(ring + i * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES, tn, i * 4);
            }
            pdl_wait();
            for (int t = pair; t < p.tiles; t += pairs) {
                const int tm = t % p.tiles_m, tn = t / p.tiles_m;
                const int m0 = tm * 256 + static_cast<int>(rank) * 128;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    uint8_t* sf = ring + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
                    const int k4 = kb * 4;
                    if (pre > 0) {
                        --pre;
                        issue_a(sf, m0, k4);
                        cp_async_arrive_noinc(&bar[stage]);
                    } else {
                        if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.status)) goto sf_done;
                        if (vec4) {
                            issue_a(sf, m0, k4);
                            issue_b(sf, tn, k4);
                            cp_async_arrive_noinc(&bar[stage]);
                        } else {
                            // K % 128 != 0: gather the bytes with plain loads
                            uint32_t v[4];
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                const int m = m0 + lane + 32 * g;
                                uint32_t w = 0;
                                if (m < p.M) {
                                    const uint8_t* src = p.sa + static_cast<size_t>(m) * KB + k4;
                                    for (int j = 0; j < 4; ++j)
                                        if (k4 + j < KB) w |= static_cast<uint32_t>(__ldcg(src + j)) << (8 * j);
                                }
                                v[g] = w;
                            }
                            *reinterpret_cast<uint4*>(sf + lane * 16) = make_uint4(v[0], v[1], v[2], v[3]);
#pragma unroll
                            for (int j = 0; j < C::SFB_CHUNKS; ++j) {
#pragma unroll
                                for (int g = 0; g < 4; ++g) {
                                    const int r = 128 * j + lane + 32 * g;
                                    const int n = b_row(r, tn);
                                    uint32_t w = 0;
                                    if (r < C::BN && n < p.N) {
                                        const uint8_t* src = b_src(n, k4);
                                        for (int jj = 0; jj < 4; ++jj)
                                            if (k4 + jj < KB) w |= static_cast<uint32_t>(__ldcg(src + jj)) << (8 * jj);
                                    }
                                    v[g] = w;
                                }
                                *reinterpret_cast<uint4*>(sf + 512 * (1 + j) + lane * 16) =
                                    make_uint4(v[0], v[1], v[2], v[3]);
                            }
                            fence_proxy_async_smem();
                            mbar_arrive(&bar[stage]);
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
    } else if (warp == 3) {
        // ------------------------------------------------ scale forwarder (odd CTA)
        if (SCALED && !leader && lane == 0) {
            uint32_t stage = 0, phase = 0;
            int dbg_i = 0;
            for (int t = pair; t < p.tiles; t += pairs) {
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!wait_bar(&sf_full[stage], phase, abort_flag, p.status)) goto fwd_done;
                    fence_proxy_async_smem();  // the even CTA's tcgen05.cp reads these bytes
                    mbar_arrive_cluster(full_lead + 8u * stage);
                    pair_stamp(p, 3, dbg_i++);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        fwd_done:;
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;            // TMEM lane quadrant this warp may read
        const int half = (warp - 4) >> 2;  // which alternate 32-column chunks it takes
        const int et = threadIdx.x - 128;
        uint32_t acc = 0, acc_phase = 0;
        pdl_wait();
        const bool f32row = !SCALED;
        for (int t = pair; t < p.tiles; t += pairs) {
            const int tm = t % p.tiles_m, tn = t / p.tiles_m;
            const bool ready = wait_bar(&acc_full[acc], acc_phase, abort_flag, p.status);
            // all epilogue warps meet here every tile and leave together (the
            // stop decision is uniform); this also retires the previous tile's
            // column parameters
            if (named_bar_or(1, kEpiThreads, !ready || *abort_flag)) break;
            tc_fence_after();
            const int n_base = tn * C::OUT_COLS;
            for (int i = et; i < C::OUT_COLS; i += kEpiThreads) {
                const int n = n_base + i;
                const bool ok = n < p.Nout;
                colp[i] = (ok && p.bias) ? __ldcg(p.bias + n) : 0.f;
                colp[256 + i] = (SWIGLU && ok && p.bias) ? __ldcg(p.bias + n + p.n_half) : 0.f;
                colp[512 + i] = (f32row && ok) ? __ldcg(p.swb + n) : 1.f;
                colp[768 + i] = (SWIGLU && f32row && ok) ? __ldcg(p.swb + n + p.n_half) : 1.f;
            }
            named_bar_sync(1, kEpiThreads);
            const int row0 = tm * 256 + static_cast<int>(rank) * 128 + q * 32;  // output row of lane 0
            if (row0 < p.M) {
                const uint32_t taddr = tmem + acc * C::ACC_STRIDE + (static_cast<uint32_t>(q * 32) << 16);
                const int m = row0 + lane;
                const float sx = (f32row && m < p.M) ? __ldcg(p.sxa + m) : 1.f;
#pragma unroll 1
                for (int c = half * 32; c < C::OUT_COLS; c += 64) {
                    uint32_t g[32], h[32];
                    tmem_ld32(taddr + c, g);
                    if (SWIGLU) tmem_ld32(taddr + C::BN / 2 + c, h);
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
                        load_row32_bf16(p.out, p.Nout, p.M, m, n_base + c,
                                        min(min(32, C::OUT_COLS - c), p.Nout - (n_base + c)), res);
                        if (f32row) epi_chunk_residual<true>(g, sx, colp, c, res, pk);
                        else epi_chunk_residual<false>(g, sx, colp, c, res, pk);
                    } else {
                        if (f32row) epi_chunk<MX_EPI_NONE, false, true>(g, h, sx, colp, c, pk);
                        else epi_chunk<MX_EPI_NONE, false, false>(g, h, sx, colp, c, pk);
                    }
                    const int lim = min(min(32, C::OUT_COLS - c), p.Nout - (n_base + c));
                    store_chunk_staged(staging + (warp - 4) * 2048, pk, lane, p.out, p.Nout, p.M, row0, n_base + c,
                                       lim);
                }
            }
            // this CTA is done with the accumulator: tell the even CTA's MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(&acc_empty[acc]);
                else mbar_arrive_cluster(acc_empty_lead + 8u * acc);
            }
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
        }
    }
    __syncwarp();

    // ---------------------------------------------------- teardown
    if (leader && warp == 1 && lane == 0) {
        // every pair MMA has completed before either CTA frees TMEM or leaves
        tc_commit_pair(final_bar);
        wait_bar_final(final_bar, 0, p.status);
    }
    __syncwarp();
    // no CTA leaves while its partner may still read or signal its shared
    // memory or write its TMEM
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, C::TMEM_COLS);
}

template <bool SCALED, bool SWIGLU>
cudaError_t prepare_pair()
{
    using C = PairCfg<SCALED, SWIGLU>;
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && !done[dev]) {
        e = cudaFuncSetAttribute(gemm_pair_kernel<SCALED, SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

template <bool SCALED, bool SWIGLU>
cudaError_t launch_pair_t(const PairArgs& a, const GemmPlan& plan, cudaStream_t st)
{
    using C = PairCfg<SCALED, SWIGLU>;
    cudaError_t e = prepare_pair<SCALED, SWIGLU>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.grid_x, 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    if (launch_flags() & MX_LAUNCH_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<SCALED, SWIGLU>, a);
}

template <bool SCALED, bool SWIGLU>
int max_pairs_t()
{
    using C = PairCfg<SCALED, SWIGLU>;
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (cache[dev]) return cache[dev] > 0 ? cache[dev] : 0;
    }
    int n = 0;
    if (prepare_pair<SCALED, SWIGLU>() == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * 64, 1, 1);
        cfg.blockDim = dim3(kPairThreads, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<SCALED, SWIGLU>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
    }
    std::lock_guard<std::mutex> lk(mu);
    cache[dev] = n > 0 ? n : -1;
    return n;
}

int stages_pair(bool scaled, bool swiglu)
{
    return scaled ? (swiglu ? PairCfg<true, true>::STAGES : PairCfg<true, false>::STAGES)
                  : (swiglu ? PairCfg<false, true>::STAGES : PairCfg<false, false>::STAGES);
}

}  // namespace

int max_active_pairs(bool scaled, bool swiglu)
{
    return scaled ? (swiglu ? max_pairs_t<true, true>() : max_pairs_t<true, false>())
                  : (swiglu ? max_pairs_t<false, true>() : max_pairs_t<false, false>());
}

bool plan_pair(const GemmProblem& pb, int sms, int max_ctas, GemmPlan* plan)
{
    const bool swiglu = epi_swiglu(pb.epi);
    const bool scaled = pb.a_fmt == MX_A_E4M3_E8M0_1X32;
    const int nout = swiglu ? pb.N / 2 : pb.N;
    const int out_cols = swiglu ? 120 : 240;
    const int tiles = ((pb.M + 255) / 256) * ((nout + out_cols - 1) / out_cols);
    int pairs = max_active_pairs(scaled, swiglu);
    if (pairs <= 0) return false;
    pairs = std::min(pairs, sms / 2);
    if (max_ctas > 0) pairs = std::min(pairs, std::max(1, max_ctas / 2));
    pairs = std::min(pairs, tiles);
    *plan = GemmPlan();
    plan->kernel = 3;
    plan->block_n = 240;
    plan->a_rows = 128;
    plan->block_m = 256;
    plan->splits = 1;
    plan->units = tiles;
    plan->tiles = tiles;
    plan->acc_bufs = 2;
    plan->stages = stages_pair(scaled, swiglu);
    plan->grid_x = 2 * pairs;
    plan->grid_y = 1;
    plan->cluster = 2;
    plan->ws_bytes = kWorkspaceHeader;
    return true;
}

cudaError_t launch_pair(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st)
{
    const bool swiglu = epi_swiglu(pb.epi);
    const bool scaled = pb.a_fmt == MX_A_E4M3_E8M0_1X32;
    PairArgs a;
    memset(&a, 0, sizeof(a));
    if (!make_tmap_2d(&a.tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.a_codes, pb.K, pb.M, pb.K, 128, 128))
        return cudaErrorInvalidValue;
    const bool e2m1 = pb.b_fmt == MX_B_E2M1_E8M0_1X32;
    if (!make_tmap_2d(&a.tmB, e2m1 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                      pb.b_codes, pb.K, pb.N, e2m1 ? pb.K / 2 : pb.K, 128, 120))
        return cudaErrorInvalidValue;
    a.sa = scaled ? static_cast<const uint8_t*>(pb.a_scales) : nullptr;
    a.sb = scaled ? static_cast<const uint8_t*>(pb.b_scales) : nullptr;
    a.sxa = scaled ? nullptr : static_cast<const float*>(pb.a_scales);
    a.swb = scaled ? nullptr : static_cast<const float*>(pb.b_scales);
    a.bias = pb.bias;
    a.out = static_cast<__nv_bfloat16*>(pb.out);
    a.status = pb.status;
    a.prefetch_w = (launch_flags() & MX_LAUNCH_PDL) && (launch_flags() & MX_LAUNCH_PREFETCH_WEIGHTS) ? 1 : 0;
    a.M = pb.M;
    a.N = pb.N;
    a.K = pb.K;
    a.Nout = swiglu ? pb.N / 2 : pb.N;
    a.KB = pb.K / 32;
    a.num_kb = (pb.K + 127) / 128;
    a.tiles_m = (pb.M + 255) / 256;
    a.tiles = plan.units;
    a.b_fmt = pb.b_fmt;
    a.epi = pb.epi;
    a.n_half = pb.N / 2;
    // instruction descriptor: fp32 D, A e4m3, B e4m3 (0) or e2m1 (5), K-major
    // both, N = 240, M = 256; block-scaled: E8M0 scales (bit 23), the scale
    // IDs (bits 4-5 for B, 29-30 for A) are set per MMA
    const uint32_t b_code = e2m1 ? 5u : 0u;
    if (scaled)
        a.idesc = (b_code << 10) | ((240u >> 3) << 17) | (1u << 23) | ((256u >> 4) << 24);
    else
        a.idesc = (1u << 4) | ((240u >> 3) << 17) | ((256u >> 4) << 24);
    // transaction bytes count the global-side size: a 128-element e2m1 row is
    // 64 bytes although it lands as 128 bytes in shared memory
    const uint32_t b_row_bytes = e2m1 ? 64u : 128u;
    a.tx_bytes = 2u * (128u * 128u + 120u * b_row_bytes);
    int tl_ctas = 0;
    unsigned long long* tl = timeline_buffer(&tl_ctas);
    a.timeline = tl ? tl + static_cast<size_t>(tl_ctas) * kTimelineCtaSlots : nullptr;
    if (scaled) return swiglu ? launch_pair_t<true, true>(a, plan, st) : launch_pair_t<true, false>(a, plan, st);
    return swiglu ? launch_pair_t<false, true>(a, plan, st) : launch_pair_t<false, false>(a, plan, st);
}

}  // namespace mxg
