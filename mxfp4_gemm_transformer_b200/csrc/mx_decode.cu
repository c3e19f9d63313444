// mx_decode.cu -- the decode-shaped GEMM (M <= 64 tokens) for sm_100a.
//
//   out[m, n] = epilogue( sum_k x[m, k] w[n, k] )   with few tokens m
//
// With a handful of tokens the projection is a stream over the weights: every
// weight byte is read once and used M times, so the time is the weight bytes
// over HBM bandwidth.  The kernel is shaped for that:
//
//   * Weights are the MMA's A operand: 128 weight rows fill the 128 TMEM lanes
//     and the tokens are the MMA's N (16, 32 or 64 columns), so no tensor-core
//     work is spent on padding rows and the accumulator is small.
//   * The work is the list of (tile of 128 output columns, 128-wide K block)
//     units in tile-major order; CTA c takes the contiguous range
//     [c T / G, (c + 1) T / G) of the T units (stream-K), so every SM streams
//     the same number of weight bytes whatever the tile count.  A tile whose
//     K range is cut between CTAs is reduced through the caller's workspace:
//     each CTA adds its fp32 partial with atomic adds into the tile's
//     accumulator and counts its K blocks; the CTA that completes the count
//     runs the epilogue, then zeroes the accumulator and the count for the
//     next launch.  (The order of the fp32 additions is not fixed.)  With
//     whole-tile ranges (no workspace) a CTA only ever runs full tiles.
//   * A CTA uses at most ~110 KB of shared memory and 256 TMEM columns, so two
//     CTAs fit on an SM: under programmatic dependent launch the next GEMM's
//     CTAs start while this one drains, and (when weights may be prefetched)
//     already stream their first weight stages.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// MMA issuer (tcgen05.mma kind::mxf8f6f4 block-scaled, or kind::f8f6f4 for
// per-row fp32 scales), warp 2 scale-factor producer, warps 4-7 epilogue
// (thread = TMEM lane = weight row, columns = tokens).  For SwiGLU a tile holds
// 128 gate rows and the matching 128 up rows (two MMAs per K step sharing the
// token operand), so one thread holds both halves of its output column.
//
// Every wait is bounded (%globaltimer); a wait that runs out sets a bit in
// the workspace status word and the kernel tears down normally.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mx_internal.h"
#include "mx_kernel_common.cuh"
#include "mx_ptx.cuh"
#include "mx_quant_common.cuh"
#include "mx_decode_common.cuh"

namespace mxg {

// MT = tokens per MMA (N of the instruction); NSUB = 128-row weight sub-tiles
// per tile (2 for SwiGLU: gate, up); ONE_PER_SM = the whole SM's shared
// memory for one CTA (a deep weight ring for long-running problems) instead of
// at most 113 KB (two CTAs per SM, so the next launch's CTAs start beside
// this launch's).  Shared memory holds two rings: weight tiles with their
// scales (DW stages) and token tiles with theirs (DX stages).  Each has its
// own producer, so weights can run as far ahead of the tokens as the ring
// allows, and all of them before the previous kernel has finished.
template <int MT, int NSUB, bool SCALED, bool ONE_PER_SM>
struct DecCfg {
    static constexpr int BK = 128;                  // K elements per stage (128 bytes per row in smem)
    static constexpr int W_BYTES = NSUB * 128 * BK;  // e2m1 lands unpacked: one byte per element
    static constexpr int X_BYTES = MT * BK;
    static constexpr int SFA_BYTES = SCALED ? 512 * NSUB : 0;  // tcgen05.cp chunks: 128 rows x 4 K blocks
    static constexpr int SFB_BYTES = SCALED ? 512 : 0;
    static constexpr int BAR_BYTES = 512;
    // 228 KB of shared memory per SM with 1 KB reserved per CTA; 227 KB per CTA at most
    static constexpr int LIMIT = ONE_PER_SM ? 232448 : 115712;
    static constexpr int USABLE = LIMIT - 1024 - BAR_BYTES;
    // token stages: enough that a CTA's token tiles are requested in one or
    // two rounds; the rest of the budget goes to weight stages
    static constexpr int DX = ONE_PER_SM ? (MT <= 32 ? 8 : 4) : (MT <= 16 ? 5 : (MT <= 32 ? 6 : 3));
    static constexpr int DW_FIT = (USABLE - DX * (X_BYTES + SFB_BYTES)) / (W_BYTES + SFA_BYTES);
    static constexpr int DW = DW_FIT > 12 ? 12 : DW_FIT;
    static constexpr int OFF_X = DW * W_BYTES;
    static constexpr int OFF_SFA = OFF_X + DX * X_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + DW * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + DX * SFB_BYTES;
    static constexpr int SMEM_BYTES = 1024 + OFF_BAR + BAR_BYTES;
    static constexpr int SUB_COLS = MT < 32 ? 32 : MT;  // TMEM columns per sub-tile accumulator
    static constexpr int ACC_COLS = NSUB * SUB_COLS;
    static constexpr int SF_COLS = SCALED ? 4 * (NSUB + 1) : 0;
    static constexpr int ACC_BUFS = (2 * ACC_COLS + SF_COLS <= 256) ? 2 : 1;
    static constexpr int SF_BASE = ACC_BUFS * ACC_COLS;
    static constexpr int COLS = SF_BASE + SF_COLS;
    static constexpr int TMEM_COLS = COLS <= 32 ? 32 : COLS <= 64 ? 64 : COLS <= 128 ? 128 : 256;
    static_assert(DW >= 2, "shared memory too small for two weight stages");
    static_assert(COLS <= 256, "TMEM budget is half an SM");
    static_assert(SMEM_BYTES <= LIMIT, "over the shared-memory budget");
    static_assert(OFF_X % 1024 == 0 && OFF_SFA % 1024 == 0 && OFF_BAR % 16 == 0, "alignment");
    static_assert(DW * W_BYTES >= NSUB * MT * 128 * 4, "the weight ring holds a cluster partial");
};

// CL: the instance for cluster splits (a tile's K range over the CTAs of a
// thread-block cluster, partials reduced in distributed shared memory); the
// other instance runs whole tiles and stream-K.  Each carries only its own
// epilogue: on these microsecond launches the code on the critical path is
// fetched cold, so code that a launch never runs still costs time.
template <int MT, int NSUB, bool SCALED, bool ONE_PER_SM, bool CL>
__global__ void __launch_bounds__(kDecThreads, ONE_PER_SM ? 1 : 2) decode_kernel(const __grid_constant__ DecodeArgs p)
{
    using C = DecCfg<MT, NSUB, SCALED, ONE_PER_SM>;
    constexpr bool SWIGLU = NSUB == 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* wring = base;                 // [DW][W_BYTES]
    uint8_t* xring = base + C::OFF_X;      // [DX][X_BYTES]
    uint8_t* sfa_ring = base + C::OFF_SFA;  // [DW][SFA_BYTES]
    uint8_t* sfb_ring = base + C::OFF_SFB;  // [DX][SFB_BYTES]
    uint64_t* wfull = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
    uint64_t* wempty = wfull + C::DW;
    uint64_t* xfull = wempty + C::DW;
    uint64_t* xempty = xfull + C::DX;
    uint64_t* acc_full = xempty + C::DX;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* final_bar = acc_empty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_holder + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // the lane of each warp that issues single-thread operations (warp 1: the
    // tcgen05 MMAs, copies and commits, including the final commit)
    const bool leader = elect_one();

    // this CTA's units [g0, g1) (unit = tile * num_kb + K block)
    int g0, g1;
    const int S = CL ? p.cluster_s : 1;
    const int crank = S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
    if (S > 1) {
        // one tile per cluster; rank r takes K blocks [r nkb / S, (r + 1) nkb / S)
        const int tile = static_cast<int>(blockIdx.x) / S;
        g0 = tile * p.num_kb + crank * p.num_kb / S;
        g1 = tile * p.num_kb + (crank + 1) * p.num_kb / S;
    } else if (p.whole_tiles) {
        g0 = static_cast<int>(static_cast<long long>(blockIdx.x) * p.tiles / gridDim.x) * p.num_kb;
        g1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.tiles / gridDim.x) * p.num_kb;
    } else {
        g0 = static_cast<int>(static_cast<long long>(blockIdx.x) * p.total / gridDim.x);
        g1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.total / gridDim.x);
    }
    const int n_units = g1 - g0;

    if (threadIdx.x == 0) {
        dec_now(p, kDecStart);
        if (MXG_TRACE && p.timeline) {
            uint32_t sm;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
            dec_stamp(p, kDecSmid, sm);
            dec_stamp(p, kDecUnits, static_cast<unsigned long long>(n_units));
        }
        prefetch_tmap(&p.tmW);
        for (int s = 0; s < C::DW; ++s) {
            mbar_init(&wfull[s], SCALED ? 1 + 32 : 1);
            mbar_init(&wempty[s], 1);
        }
        // one arrival per lane of the token producer, or per quantising warp
        const uint32_t x_arrivals = (SCALED && p.x_bf16) ? static_cast<uint32_t>(p.xq_warps) : 32u;
        for (int s = 0; s < C::DX; ++s) {
            mbar_init(&xfull[s], x_arrivals);
            mbar_init(&xempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kDecEpiThreads / 32);
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
    // the next kernel in the stream may be scheduled now: it only reads what
    // this one writes after its own dependency wait
    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        dec_now(p, kDecReady);
    }

    if (warp == 0) {
        // ------------------------------------------------ weight-tile producer
        // With weight prefetch allowed the weights do not depend on the
        // previous kernel: the ring fills at once and keeps streaming.  Each
        // 128-row tile is requested as kWBoxes boxes of 128 / kWBoxes rows,
        // one per lane (measured: whole-tile launches with two CTAs per SM
        // stream about 1.45x faster this way than with one 128-row box).
        const uint64_t pol_w = policy_evict_first();
        uint32_t armed = 0, used = 0;  // per stage: parity of its last arming; armed at least once
        // Weight tiles that will not have a ring stage before the previous
        // kernel completes are prefetched into L2 now, so their loads hit
        // L2 on the critical path instead of waiting on HBM.  Only for
        // short unit ranges (at most one more ring's worth): a long range
        // streams through the ring anyway and would only flood L2.
        if (p.prefetch_w > 0 && n_units <= 2 * C::DW) {
            const int early = min(C::DW, p.prefetch_w);
            for (int i = early + lane; i < n_units; i += 32) {
                const int g = g0 + i;
                const int tile = g / p.num_kb, kb = g - tile * p.num_kb;
#pragma unroll
                for (int s = 0; s < NSUB; ++s)
                    for (int b = 0; b < kWBoxes; ++b)
                        tma_prefetch_l2_2d(&p.tmW, kb * C::BK,
                                           (s == 0 ? 0 : p.n_half) + tile * 128 + b * (128 / kWBoxes));
            }
        }
        uint32_t ws = 0, wph = 0;
        for (int i = 0; i < n_units; ++i) {
            const int g = g0 + i;
            const int tile = g / p.num_kb, kb = g - tile * p.num_kb;
            if (i == p.prefetch_w) pdl_wait();
            if (__any_sync(0xFFFFFFFFu, !wait_bar(&wempty[ws], wph ^ 1u, abort_flag, p.status))) break;
            if (lane == 0) mbar_arrive_expect_tx(&wfull[ws], p.w_tx);
            __syncwarp();
            if (lane < NSUB * kWBoxes) {
                const int s = lane / kWBoxes, b = lane % kWBoxes;
                const int row0 = (s == 0 ? 0 : p.n_half) + tile * 128 + b * (128 / kWBoxes);
                tma_load_2d(wring + ws * C::W_BYTES + s * 128 * C::BK + b * (128 / kWBoxes) * C::BK, &p.tmW,
                            &wfull[ws], kb * C::BK, row0, pol_w);
            }
            if (lane == 0) {
                if (i == 0) dec_now(p, kDecFirstTma);
                dec_detail(p, kDetW, i);
            }
            used |= 1u << ws;
            armed = (armed & ~(1u << ws)) | (wph << ws);
            if (++ws == C::DW) {
                ws = 0;
                wph ^= 1u;
            }
        }
        // before leaving, every load this warp started has landed (in a
        // normal run the MMA thread consumed them all already)
        if (lane == 0)
            for (int s = 0; s < C::DW; ++s)
                if (used & (1u << s)) wait_bar_final(&wfull[s], (armed >> s) & 1u, p.status);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // The whole warp runs the loop (barrier waits, descriptors); one
        // elected lane issues the tcgen05 operations.
        const uint32_t tmem_sfa = tmem + C::SF_BASE;      // 4 columns per weight sub-tile
        const uint32_t tmem_sfb = tmem_sfa + 4 * NSUB;  // 4 columns for the tokens
        const uint32_t w_s = smem_u32(wring), x_s = smem_u32(xring);
        const uint32_t sfa_s = smem_u32(sfa_ring), sfb_s = smem_u32(sfb_ring);
        uint32_t ws = 0, wph = 0, xs = 0, xph = 0, acc = 0, acc_phase = 0;
        int g = g0;
        while (g < g1) {
            const int tile = g / p.num_kb;
            const int seg_end = min(g1, (tile + 1) * p.num_kb);
            if (__any_sync(0xFFFFFFFFu, !wait_bar(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status))) break;
            tc_fence_after();
            const uint32_t d = tmem + acc * C::ACC_COLS;
            uint32_t accumulate = 0;
            bool ok = true;
            for (; g < seg_end; ++g) {
                const int kb = g - tile * p.num_kb;
                const bool wok = wait_bar(&wfull[ws], wph, abort_flag, p.status);
                if (leader) dec_detail(p, kDetWFull, g - g0);
                const bool xok = wok && wait_bar(&xfull[xs], xph, abort_flag, p.status);
                if (__any_sync(0xFFFFFFFFu, !xok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                fence_proxy_async_smem();  // token tiles and scales were written by cp.async
                if (leader) {
                    dec_detail(p, kDetXFull, g - g0);
                    if (g == g0) dec_now(p, kDecFirstFull);
                }
                const uint32_t sW = w_s + ws * C::W_BYTES;
                const uint32_t sX = x_s + xs * C::X_BYTES;
                if (leader) {
                    if (SCALED) {
#pragma unroll
                        for (int s = 0; s < NSUB; ++s)
                            tc_cp_32x128b_x4(tmem_sfa + 4 * s, sdesc_sf(sfa_s + ws * C::SFA_BYTES + 512 * s));
                        tc_cp_32x128b_x4(tmem_sfb, sdesc_sf(sfb_s + xs * C::SFB_BYTES));
                    }
                    const int krem = p.K - kb * C::BK;
                    if (krem >= C::BK) {
                        // the usual case: four K steps, fully unrolled
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t xd = sdesc_sw128(sX + kk * 32);
#pragma unroll
                            for (int s = 0; s < NSUB; ++s) {
                                const uint64_t wd = sdesc_sw128(sW + s * 128 * C::BK + kk * 32);
                                if (SCALED)
                                    mma_mx(d + s * C::SUB_COLS, wd, xd,
                                           p.idesc | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29),
                                           tmem_sfa + 4 * s, tmem_sfb, (kk > 0) ? 1u : accumulate);
                                else
                                    mma_f8(d + s * C::SUB_COLS, wd, xd, p.idesc, (kk > 0) ? 1u : accumulate);
                            }
                        }
                    } else {
                        // the last, partial K block
                        for (int kk = 0; kk < krem / 32; ++kk) {
                            const uint64_t xd = sdesc_sw128(sX + kk * 32);
#pragma unroll
                            for (int s = 0; s < NSUB; ++s) {
                                const uint64_t wd = sdesc_sw128(sW + s * 128 * C::BK + kk * 32);
                                if (SCALED)
                                    mma_mx(d + s * C::SUB_COLS, wd, xd,
                                           p.idesc | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29),
                                           tmem_sfa + 4 * s, tmem_sfb, (kk > 0) ? 1u : accumulate);
                                else
                                    mma_f8(d + s * C::SUB_COLS, wd, xd, p.idesc, (kk > 0) ? 1u : accumulate);
                            }
                        }
                    }
                    // release the stages only when a later unit of this CTA
                    // refills them (a commit is a tcgen05 instruction on the
                    // issue path; the tile's accumulator commit covers the rest)
                    if (g - g0 + C::DW < n_units) tc_commit(&wempty[ws]);
                    if (g - g0 + C::DX < n_units) tc_commit(&xempty[xs]);
                    dec_detail(p, kDetCommit, g - g0);
                }
                __syncwarp();
                accumulate = 1;
                if (++ws == C::DW) {
                    ws = 0;
                    wph ^= 1u;
                }
                if (++xs == C::DX) {
                    xs = 0;
                    xph ^= 1u;
                }
            }
            if (!ok) break;
            if (leader) {
                tc_commit(&acc_full[acc]);
                if (g == g1) dec_now(p, kDecLastCommit);
            }
            __syncwarp();
            if (C::ACC_BUFS == 2) {
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------ weight-scale producer
        // Each lane fills 16 bytes of every 128-row chunk with 4-byte
        // asynchronous copies: rows lane + 32 j, bytes j * 4 .. j * 4 + 3 =
        // the stage's four 32-wide K blocks (tcgen05.cp 32x128b layout, byte
        // (r % 32) * 16 + (r / 32) * 4 + kblock).  Rows past the end are
        // zero-filled.  Each lane's arrival on the stage's barrier fires when
        // its copies have landed.
        if (SCALED) {
            const int KB = p.KB;
            uint32_t ws = 0, wph = 0;
            for (int i = 0; i < n_units; ++i) {
                const int g = g0 + i;
                const int tile = g / p.num_kb, kb = g - tile * p.num_kb;
                if (i == p.prefetch_w) pdl_wait();
                if (!wait_bar(&wempty[ws], wph ^ 1u, abort_flag, p.status)) break;
                uint8_t* sf = sfa_ring + ws * C::SFA_BYTES;
#pragma unroll
                for (int s = 0; s < NSUB; ++s) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int n = (s == 0 ? 0 : p.n_half) + tile * 128 + lane + 32 * j;
                        const bool ok = n < p.N;
                        const int nn = ok ? n : 0;
                        const uint8_t* src = (p.b_fmt == MX_B_E4M3_E8M0_32X32)
                                                 ? p.sw8 + static_cast<size_t>(nn >> 5) * KB + kb * 4
                                                 : p.sw8 + static_cast<size_t>(nn) * KB + kb * 4;
                        cp_async_4(sf + 512 * s + lane * 16 + j * 4, src, ok ? 4u : 0u);
                    }
                }
                cp_async_arrive_noinc(&wfull[ws]);
                if (++ws == C::DW) {
                    ws = 0;
                    wph ^= 1u;
                }
            }
            cp_async_wait_all();  // nothing of ours in flight when the CTA leaves
        }
    } else if (warp == 3) {
        // ------------------------------------------------ token producer
        // The token tile (MT rows x 128 bytes) is written with 16-byte
        // asynchronous copies straight into the layout the 128-byte-swizzled
        // descriptor reads (16-byte chunk c of row r at r * 128 +
        // ((c ^ (r % 8)) * 16)), so these small, latency-critical loads never
        // queue behind the weight stream's tensor copies.  Only the M real
        // rows (and their scales) are copied: an MMA output column depends
        // on its own token row alone, and columns >= M are never stored, so
        // whatever the padding rows hold cannot reach a result.  Each lane
        // arrives once all its copies have landed.
        pdl_wait();
        if (SCALED && p.x_bf16) {
            dec_quant_tokens<C>(p, g0, n_units, xring, sfb_ring, xfull, xempty, abort_flag, lane, 32 * p.xq_warps);
        } else {
        uint32_t xs = 0, xph = 0;
        for (int i = 0; i < n_units; ++i) {
            const int g = g0 + i;
            const int kb = g % p.num_kb;
            if (!wait_bar(&xempty[xs], xph ^ 1u, abort_flag, p.status)) break;
            uint8_t* xt = xring + xs * C::X_BYTES;
            const uint8_t* src0 = p.x8 + static_cast<size_t>(kb) * C::BK;
            const int kleft = p.K - kb * C::BK;  // K elements of this block (a multiple of 16)
#pragma unroll
            for (int t = 0; t < MT * 8 / 32; ++t) {
                const int idx = lane + 32 * t;
                const int row = idx >> 3, c = idx & 7;
                if (row < p.M) {
                    const bool ok = c * 16 < kleft;  // past K (last block): zero-fill
                    cp_async_16(xt + row * 128 + ((c ^ (row & 7)) << 4),
                                src0 + static_cast<size_t>(row) * p.K + (ok ? c * 16 : 0), ok ? 16u : 0u);
                }
            }
            if (lane == 0) dec_detail(p, kDetX, i);
            if (SCALED) {
                uint8_t* sf = sfb_ring + xs * C::SFB_BYTES;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = lane + 32 * j;
                    if (m < p.M) cp_async_4(sf + lane * 16 + j * 4, p.sx8 + static_cast<size_t>(m) * p.KB + kb * 4, 4u);
                }
            }
            cp_async_arrive_noinc(&xfull[xs]);
            if (++xs == C::DX) {
                xs = 0;
                xph ^= 1u;
            }
        }
        cp_async_wait_all();  // nothing of ours in flight when the CTA leaves
        }
    } else {
        // ------------------------------------------------ epilogue (warps 4-7)
        const int q = warp & 3;       // TMEM lane quadrant this warp may read
        const int r = q * 32 + lane;  // weight row within a sub-tile = TMEM lane
        const int et = threadIdx.x - 128;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t acc = 0, acc_phase = 0;
        unsigned finals = 0;  // tiles whose epilogue this CTA ran after a reduction
        pdl_wait();
        // with a cluster split the CTA has one tile, whose accumulator is
        // ready only after every unit: until then these warps help quantise
        // the tokens
        if (SCALED && p.x_bf16 && p.xq_warps > 1)
            dec_quant_tokens<C>(p, g0, n_units, xring, sfb_ring, xfull, xempty, abort_flag, 32 + et,
                                32 * p.xq_warps);
        const int M = p.M;
        int g = g0;
        if (S > 1) {
            // park this CTA's fp32 partial in its own shared memory
            // ([NSUB][M][128], in the weight ring, whose reads by the MMAs have
            // all completed once the accumulator is ready); the cluster
            // reduces the partials after the role loops
            float* part = reinterpret_cast<float*>(wring);
            const bool ready = n_units == 0 || wait_bar(&acc_full[0], 0, abort_flag, p.status);
            if (!named_bar_or(1, kDecEpiThreads, !ready || *abort_flag)) {
                tc_fence_after();
                if (et == 0) dec_now(p, kDecFirstAcc);
#pragma unroll
                for (int s = 0; s < NSUB; ++s) {
                    for (int c = 0; c < M; c += 16) {
                        uint32_t v[16];
                        if (n_units > 0) {
                            tmem_ld16(lane_base + s * C::SUB_COLS + c, v);
                            tmem_ld_wait();
                        } else {
#pragma unroll
                            for (int t = 0; t < 16; ++t) v[t] = 0u;
                        }
#pragma unroll
                        for (int t = 0; t < 16; ++t)
                            if (c + t < M) part[(s * M + c + t) * 128 + r] = __uint_as_float(v[t]);
                    }
                }
                tc_fence_before();
                if (et == 0) dec_now(p, kDecRedAdded);
            }
            g = g1;  // no per-segment epilogue below
        }
        if constexpr (!CL)
        while (g < g1) {
            const int tile = g / p.num_kb;
            const int kb0 = g - tile * p.num_kb;
            const int seg_end = min(g1, (tile + 1) * p.num_kb);
            const int nkb = seg_end - g;
            g = seg_end;
            const bool ready = wait_bar(&acc_full[acc], acc_phase, abort_flag, p.status);
            // uniform exit decision for all epilogue warps (they meet at
            // further named barriers below)
            if (named_bar_or(1, kDecEpiThreads, !ready || *abort_flag)) break;
            tc_fence_after();
            if (et == 0 && g - nkb == g0) dec_now(p, kDecFirstAcc);
            const uint32_t abase = lane_base + acc * C::ACC_COLS;
            const int j = tile * 128 + r;  // output column of this thread
            const bool col_ok = j < p.Nout;
            float bg = 0.f, bu = 0.f, wg = 1.f, wu = 1.f;
            if (col_ok) {
                if (p.bias) {
                    bg = __ldg(p.bias + j);
                    if (SWIGLU) bu = __ldg(p.bias + j + p.n_half);
                }
                if (!SCALED) {
                    wg = __ldg(p.swf + j);
                    if (SWIGLU) wu = __ldg(p.swf + j + p.n_half);
                }
            }
            __nv_bfloat16* ocol = p.out + j;
            if (kb0 == 0 && nkb == p.num_kb) {
                // the whole K range is here: epilogue straight from TMEM
                for (int c = 0; c < M; c += 16) {
                    uint32_t gv[16], uv[16];
                    tmem_ld16(abase + c, gv);
                    if (SWIGLU) tmem_ld16(abase + C::SUB_COLS + c, uv);
                    tmem_ld_wait();
                    if (SWIGLU && p.q_codes) {
                        // output handed on as MX codes: every lane takes part
                        // (one 1 x 32 block per token per warp)
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int m = c + t;  // the same token in every lane
                            if (m < M) {
                                const float sx = (SCALED || !col_ok) ? 1.f : __ldg(p.sxf + m);
                                const float v = dec_epi<SWIGLU, !SCALED>(p.epi, __uint_as_float(gv[t]),
                                                                         __uint_as_float(uv[t]), sx, bg, bu, wg, wu);
                                dec_store_mxq(p, m, j, col_ok, lane, v);
                            }
                        }
                    } else if (col_ok) {
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int m = c + t;
                            if (m < M) {
                                const float sx = SCALED ? 1.f : __ldg(p.sxf + m);
                                const float v = dec_epi<SWIGLU, !SCALED>(p.epi, __uint_as_float(gv[t]),
                                                                         SWIGLU ? __uint_as_float(uv[t]) : 0.f, sx, bg,
                                                                         bu, wg, wu);
                                store_out(ocol + static_cast<size_t>(m) * p.Nout, p.epi, v);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[acc]);
            } else {
                // part of the K range: add the partial into the tile's fp32
                // accumulator ([NSUB][M][128], coalesced over the lanes)
                float* red = p.red + static_cast<size_t>(tile) * NSUB * M * 128 + r;
#pragma unroll
                for (int s = 0; s < NSUB; ++s) {
                    for (int c = 0; c < M; c += 16) {
                        uint32_t v[16];
                        tmem_ld16(abase + s * C::SUB_COLS + c, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 16; ++t)
                            if (c + t < M) atomicAdd(red + (static_cast<size_t>(s) * M + c + t) * 128, __uint_as_float(v[t]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[acc]);
                if (et == 0) dec_now(p, kDecRedAdded);
                // every epilogue thread's additions are ordered before one
                // thread's fence and count (fences are cumulative over what
                // the barrier ordered before them)
                named_bar_sync(1, kDecEpiThreads);
                if (et == 0) {
                    __threadfence();
                    const unsigned before = atomicAdd(p.counters + tile, static_cast<unsigned>(nkb));
                    const bool last = before + static_cast<unsigned>(nkb) == static_cast<unsigned>(p.num_kb);
                    if (last) {
                        p.counters[tile] = 0u;  // every K block of the tile is in: reset for the next launch
                        __threadfence();        // acquire: the other CTAs' additions before our reads
                    }
                    *last_flag = last ? 1 : 0;
                    dec_now(p, kDecCounted);
                }
                named_bar_sync(1, kDecEpiThreads);
                if (*last_flag) {
                    if (et == 0) ++finals;
                    // loads issued in batches (32 in flight), then clear and finish
                    constexpr int RB = SWIGLU ? 16 : 32;
                    for (int m0 = 0; m0 < M; m0 += RB) {
                        float gv[RB], uv[RB];
#pragma unroll
                        for (int t = 0; t < RB; ++t) {
                            if (m0 + t < M) {
                                gv[t] = __ldcg(red + static_cast<size_t>(m0 + t) * 128);
                                if (SWIGLU) uv[t] = __ldcg(red + static_cast<size_t>(M + m0 + t) * 128);
                            }
                        }
#pragma unroll
                        for (int t = 0; t < RB; ++t) {
                            const int m = m0 + t;
                            if (m < M) {
                                __stcg(red + static_cast<size_t>(m) * 128, 0.f);
                                if (SWIGLU) __stcg(red + static_cast<size_t>(M + m) * 128, 0.f);
                                if (SWIGLU && p.q_codes) {
                                    const float sx = (SCALED || !col_ok) ? 1.f : __ldg(p.sxf + m);
                                    dec_store_mxq(p, m, j, col_ok, lane,
                                                  dec_epi<SWIGLU, !SCALED>(p.epi, gv[t], uv[t], sx, bg, bu, wg, wu));
                                } else if (col_ok) {
                                    const float sx = SCALED ? 1.f : __ldg(p.sxf + m);
                                    const float v = dec_epi<SWIGLU, !SCALED>(p.epi, gv[t], SWIGLU ? uv[t] : 0.f, sx,
                                                                             bg, bu, wg, wu);
                                    store_out(ocol + static_cast<size_t>(m) * p.Nout, p.epi, v);
                                }
                            }
                        }
                    }
                    if (et == 0) dec_now(p, kDecFinalDone);
                }
            }
            if (C::ACC_BUFS == 2) {
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
        if (et == 0) {
            dec_now(p, kDecEpiDone);
            dec_stamp(p, kDecFinals, finals);
        }
    }
    __syncwarp();

    if (S > 1) {
        // ---------------------------------------------------- cluster reduction
        // every CTA of the cluster has parked its partial
        cluster_sync_all();
        if (threadIdx.x == 0) dec_now(p, kDecCounted);
        if (!*abort_flag) {
            // rank r finishes weight rows [r 128 / S, (r + 1) 128 / S) of the
            // tile: partials summed in rank order (deterministic), epilogue,
            // bf16 store
            const int tile = static_cast<int>(blockIdx.x) / S;
            const int row_lo = crank * 128 / S, nrows = (crank + 1) * 128 / S - row_lo;
            const int M = p.M;
            const uint32_t part_s = smem_u32(wring);
            if (SWIGLU && p.q_codes) {
                // output handed on as MX codes: rank r finishes whole 32-row
                // blocks b = r, r + S, ... of the tile's four (one 1 x 32
                // quantisation block per token), one warp per token at a time
                const int wid = static_cast<int>(threadIdx.x >> 5);
                for (int b = crank; b < 4; b += S) {
                    const int row = b * 32 + lane;
                    const int j = tile * 128 + row;
                    const bool col_ok = j < p.Nout;
                    float bgv = 0.f, buv = 0.f, wgv = 1.f, wuv = 1.f;
                    if (col_ok) {
                        if (p.bias) {
                            bgv = __ldg(p.bias + j);
                            buv = __ldg(p.bias + j + p.n_half);
                        }
                        if (!SCALED) {
                            wgv = __ldg(p.swf + j);
                            wuv = __ldg(p.swf + j + p.n_half);
                        }
                    }
                    for (int m = wid; m < M; m += kDecThreads / 32) {
                        float sg = 0.f, su = 0.f;
                        for (int q = 0; q < S; ++q) {  // rank order: deterministic
                            const uint32_t peer = map_peer_smem(part_s, static_cast<uint32_t>(q));
                            sg += ld_dsmem_f32(peer + static_cast<uint32_t>((m * 128 + row) * 4));
                            su += ld_dsmem_f32(peer + static_cast<uint32_t>(((M + m) * 128 + row) * 4));
                        }
                        const float sx = (SCALED || !col_ok) ? 1.f : __ldg(p.sxf + m);
                        dec_store_mxq(p, m, j, col_ok, lane,
                                      dec_epi<SWIGLU, !SCALED>(p.epi, sg, su, sx, bgv, buv, wgv, wuv));
                    }
                }
            }
            // one element per thread at a time: unrolling several (all their
            // remote loads first) measured slower, the larger code on this
            // short tail costing more than the round trips it saves
            constexpr int R = 1;
            const int total_e = (SWIGLU && p.q_codes) ? 0 : nrows * M;  // the MX-code output is done above
            for (int e0 = threadIdx.x; e0 < total_e; e0 += R * kDecThreads) {
                float vg[R][8], vu[R][8];
                float bg[R], bu[R], wg[R], wu[R], sx[R];
#pragma unroll
                for (int t = 0; t < R; ++t) {
                    const int e = e0 + t * kDecThreads;
                    bg[t] = 0.f;
                    bu[t] = 0.f;
                    wg[t] = 1.f;
                    wu[t] = 1.f;
                    sx[t] = 1.f;
                    if (e < total_e) {
                        const int row = row_lo + e % nrows, m = e / nrows;
                        const uint32_t off_g = static_cast<uint32_t>((m * 128 + row) * 4);
                        const uint32_t off_u = static_cast<uint32_t>(((M + m) * 128 + row) * 4);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (q < S) {
                                const uint32_t peer = map_peer_smem(part_s, static_cast<uint32_t>(q));
                                vg[t][q] = ld_dsmem_f32_batch(peer + off_g);
                                vu[t][q] = SWIGLU ? ld_dsmem_f32_batch(peer + off_u) : 0.f;
                            }
                        }
                        const int j = tile * 128 + row;
                        if (j < p.Nout) {
                            if (p.bias) {
                                bg[t] = __ldg(p.bias + j);
                                if (SWIGLU) bu[t] = __ldg(p.bias + j + p.n_half);
                            }
                            if (!SCALED) {
                                wg[t] = __ldg(p.swf + j);
                                if (SWIGLU) wu[t] = __ldg(p.swf + j + p.n_half);
                                sx[t] = __ldg(p.sxf + m);
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < R; ++t) {
                    const int e = e0 + t * kDecThreads;
                    if (e >= total_e) continue;
                    const int row = row_lo + e % nrows, m = e / nrows;
                    const int j = tile * 128 + row;
                    float sg = 0.f, su = 0.f;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (q < S) {
                            sg += vg[t][q];
                            if (SWIGLU) su += vu[t][q];
                        }
                    }
                    if (j < p.Nout)
                        store_out(p.out + static_cast<size_t>(m) * p.Nout + j, p.epi,
                                  dec_epi<SWIGLU, !SCALED>(p.epi, sg, su, sx[t], bg[t], bu[t], wg[t], wu[t]));
                }
            }
        }
        if (threadIdx.x == 0) dec_now(p, kDecFinalDone);
        // nobody leaves while a peer may still read its shared memory
        cluster_sync_all();
    }

    // ---------------------------------------------------- teardown
    __syncthreads();
    if (warp == 1) {
        if (leader) {
            // every MMA the issuing lane started has completed before TMEM is freed
            tc_commit(final_bar);
            wait_bar_final(final_bar, 0, p.status);
            dec_now(p, kDecEnd);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// host side

namespace {

template <int MT, int NSUB, bool SCALED, bool ONE, bool CL>
cudaError_t prepare_decode()
{
    using C = DecCfg<MT, NSUB, SCALED, ONE>;
    auto kern = decode_kernel<MT, NSUB, SCALED, ONE, CL>;
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && !done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        // all of the unified L1 / shared memory as shared memory (two CTAs per SM)
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

struct DecLaunch {
    const DecodeArgs* args;
    int grid;
    int cluster;
    cudaStream_t st;
    template <int MT, int NSUB, bool SCALED, bool ONE, bool CL>
    cudaError_t run() const
    {
        using C = DecCfg<MT, NSUB, SCALED, ONE>;
        cudaError_t e = prepare_decode<MT, NSUB, SCALED, ONE, CL>();
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid, 1, 1);
        cfg.blockDim = dim3(kDecThreads, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        int na = 0;
        if (cluster > 1) {
            attr[na].id = cudaLaunchAttributeClusterDimension;
            attr[na].val.clusterDim.x = cluster;
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
        return cudaLaunchKernelEx(&cfg, decode_kernel<MT, NSUB, SCALED, ONE, CL>, *args);
    }
    cudaError_t invalid() const { return cudaErrorInvalidValue; }
};

// How many clusters of `cluster` CTAs of a variant the device runs at once
// (cached per device, variant and size; 0 when the query fails).
struct DecClusters {
    int cluster;
    template <int MT, int NSUB, bool SCALED, bool ONE, bool CL>
    int run() const
    {
        using C = DecCfg<MT, NSUB, SCALED, ONE>;
        static std::mutex mu;
        static int cache[64][9] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64 || cluster < 1 || cluster > 8) return 0;
        {
            std::lock_guard<std::mutex> lk(mu);
            if (cache[dev][cluster]) return cache[dev][cluster] > 0 ? cache[dev][cluster] : 0;
        }
        if (prepare_decode<MT, NSUB, SCALED, ONE, CL>() != cudaSuccess) return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cluster * 16, 1, 1);
        cfg.blockDim = dim3(kDecThreads, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<MT, NSUB, SCALED, ONE, CL>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        std::lock_guard<std::mutex> lk(mu);
        cache[dev][cluster] = n > 0 ? n : -1;
        return n;
    }
    int invalid() const { return 0; }
};

struct DecStages {
    template <int MT, int NSUB, bool SCALED, bool ONE, bool CL>
    int run() const { return DecCfg<MT, NSUB, SCALED, ONE>::DW; }
    int invalid() const { return 0; }
};

struct DecAccBufs {
    template <int MT, int NSUB, bool SCALED, bool ONE, bool CL>
    int run() const { return DecCfg<MT, NSUB, SCALED, ONE>::ACC_BUFS; }
    int invalid() const { return 0; }
};

template <class Op>
auto dec_dispatch(int mt, bool swiglu, bool scaled, bool one, bool cl, const Op& op) -> decltype(op.invalid())
{
#define MXG_DEC(T, O, L)                                                                                          \
    if (mt == T && one == O && cl == L)                                                                           \
        return swiglu ? (scaled ? op.template run<T, 2, true, O, L>() : op.template run<T, 2, false, O, L>())     \
                      : (scaled ? op.template run<T, 1, true, O, L>() : op.template run<T, 1, false, O, L>());
    MXG_DEC(16, false, false)
    MXG_DEC(32, false, false)
    MXG_DEC(64, false, false)
    MXG_DEC(16, true, false)
    MXG_DEC(32, true, false)
    MXG_DEC(64, true, false)
    MXG_DEC(16, false, true)
    MXG_DEC(32, false, true)
    MXG_DEC(64, false, true)
    MXG_DEC(16, true, true)
    MXG_DEC(32, true, true)
    MXG_DEC(64, true, true)
#undef MXG_DEC
    return op.invalid();
}

}  // namespace

// Tokens per MMA (its N).  A short launch (fewer tiles than half the SMs) is
// latency-bound: there every M <= 32 takes the 32-column instance, so that
// consecutive decode GEMMs of different small M run the same code (switching
// instances between back-to-back launches measured ~0.4 us each).  A long
// launch streams: there M <= 16 keeps the 16-column tile, whose smaller token
// stages leave room for another weight stage.
int decode_tokens_tile(int M, bool short_launch)
{
    if (M > 32) return 64;
    return (M > 16 || short_launch) ? 32 : 16;
}

// Workspace of a decode plan: status block, per-tile counters, fp32 accumulators.
size_t decode_ws_bytes(int tiles, int nsub, int M)
{
    const size_t counters = (static_cast<size_t>(tiles) * 4 + 255) / 256 * 256;
    return kWorkspaceHeader + counters + static_cast<size_t>(tiles) * nsub * M * 128 * 4;
}

// Fills the decode fields of `plan`.  split: how a tile's K range is shared
// between CTAs -- kDecCluster (a cluster of `cluster` CTAs per tile, reduced
// in distributed shared memory), kDecStreamK (`grid` CTAs take equal unit
// ranges; cut tiles reduced with workspace atomics) or kDecWholeTiles (`grid`
// CTAs take whole tiles).  per_sm: 1 or 2 CTAs per SM (0 = choose: one with a
// deep weight ring when each CTA streams many more stages than the two-per-SM
// ring holds).  Returns false when the kernel cannot run the problem so.
bool plan_decode(const GemmProblem& pb, int split, int grid, int cluster, int per_sm, int sms, GemmPlan* plan)
{
    const bool swiglu = epi_swiglu(pb.epi);
    const bool scaled = a_fmt_e8m0(pb.a_fmt);
    if (pb.M < 1 || pb.M > 64) return false;
    if (scaled && (pb.K % 128) != 0) return false;  // 4-byte scale copies
    const int nout = swiglu ? pb.N / 2 : pb.N;
    const int tiles = (nout + 127) / 128;
    const int num_kb = (pb.K + 127) / 128;
    const long long total = static_cast<long long>(tiles) * num_kb;
    if (total > 0x7FFFFFFFLL) return false;
    const int nsub = swiglu ? 2 : 1;
    const int mt = decode_tokens_tile(pb.M, tiles * 2 <= sms);
    int g = 1, S = 1;
    bool cut = false;  // stream-K: some tile's K range is split between CTAs
    long long per_cta = 0;
    if (split == kDecCluster) {
        S = std::max(1, std::min(cluster, std::min(8, num_kb)));
        if (S < 2) return false;
        if (static_cast<long long>(tiles) * S > 0x7FFFFFFFLL) return false;
        g = tiles * S;
        per_cta = (num_kb + S - 1) / S;
    } else if (split == kDecWholeTiles) {
        g = std::max(1, std::min(grid, tiles));
        per_cta = static_cast<long long>((tiles + g - 1) / g) * num_kb;
    } else {
        g = static_cast<int>(std::max(1LL, std::min<long long>(grid, total)));
        for (int c = 1; c < g && !cut; ++c) cut = (static_cast<long long>(c) * total / g) % num_kb != 0;
        per_cta = (total + g - 1) / g;
    }
    bool one = per_sm == 1;
    if (per_sm == 0) one = per_cta > 3LL * dec_dispatch(mt, swiglu, scaled, false, false, DecStages{});
    if (S > 1 && dec_dispatch(mt, swiglu, scaled, one, true, DecClusters{S}) < 1) return false;
    plan->kernel = 1;
    plan->block_n = 128;
    plan->block_m = mt;
    plan->a_rows = mt;
    plan->tiles = tiles;
    plan->whole_tiles = split == kDecWholeTiles ? 1 : 0;
    plan->reduce = cut ? 1 : 0;
    plan->cluster = S;
    plan->one_per_sm = one ? 1 : 0;
    plan->grid_x = g;
    plan->grid_y = 1;
    plan->units = static_cast<int>(total);
    if (split == kDecCluster)
        plan->splits = S;
    else if (split == kDecWholeTiles)
        plan->splits = 1;
    else
        plan->splits = std::max(1, static_cast<int>((static_cast<long long>(g) * num_kb + total - 1) / total));
    plan->gsplit = 0;
    plan->part_rows = 0;
    plan->ws_bytes = cut ? decode_ws_bytes(tiles, nsub, pb.M) : kWorkspaceHeader;
    plan->acc_bufs = dec_dispatch(mt, swiglu, scaled, one, false, DecAccBufs{});
    plan->stages = dec_dispatch(mt, swiglu, scaled, one, false, DecStages{});
    return true;
}

cudaError_t launch_decode(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st)
{
    const bool swiglu = epi_swiglu(pb.epi);
    const bool scaled = a_fmt_e8m0(pb.a_fmt);
    const bool e2m1 = pb.b_fmt == MX_B_E2M1_E8M0_1X32;
    const int mt = plan.block_m;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    if (e2m1) {
        if (!make_tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, pb.b_codes, pb.K, pb.N, pb.K / 2, 128,
                          128 / kWBoxes))
            return cudaErrorInvalidValue;
    } else {
        if (!make_tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.b_codes, pb.K, pb.N, pb.K, 128, 128 / kWBoxes))
            return cudaErrorInvalidValue;
    }
    a.x_bf16 = pb.a_fmt == MX_A_BF16_E8M0_1X32 ? 1 : 0;
    a.x8 = a.x_bf16 ? nullptr : static_cast<const uint8_t*>(pb.a_codes);
    a.xb = a.x_bf16 ? static_cast<const __nv_bfloat16*>(pb.a_codes) : nullptr;
    a.sw8 = scaled ? static_cast<const uint8_t*>(pb.b_scales) : nullptr;
    a.sx8 = (scaled && !a.x_bf16) ? static_cast<const uint8_t*>(pb.a_scales) : nullptr;
    a.swf = scaled ? nullptr : static_cast<const float*>(pb.b_scales);
    a.sxf = scaled ? nullptr : static_cast<const float*>(pb.a_scales);
    a.bias = pb.bias;
    if (pb.epi == MX_EPI_SWIGLU_MXQ) {
        // codes [M, N/2], then the E8M0 scales [M, N/64]
        a.q_codes = static_cast<uint8_t*>(pb.out);
        a.q_scales = a.q_codes + static_cast<size_t>(pb.M) * (pb.N / 2);
    } else {
        a.out = static_cast<__nv_bfloat16*>(pb.out);
    }
    a.status = pb.status;
    if (plan.reduce) {
        uint8_t* ws = reinterpret_cast<uint8_t*>(pb.status);
        a.counters = reinterpret_cast<unsigned*>(ws + kWorkspaceHeader);
        a.red = reinterpret_cast<float*>(ws + kWorkspaceHeader +
                                         (static_cast<size_t>(plan.tiles) * 4 + 255) / 256 * 256);
    }
    // weight stages requested before the previous kernel has completed
    a.prefetch_w = 0;
    if ((launch_flags() & MX_LAUNCH_PDL) && (launch_flags() & MX_LAUNCH_PREFETCH_WEIGHTS))
        a.prefetch_w = decode_prefetch_stages() > 0 ? decode_prefetch_stages() : 0x7FFFFFFF;
    a.timeline = timeline_buffer(&a.timeline_ctas);
    a.whole_tiles = plan.whole_tiles;
    a.cluster_s = plan.cluster > 1 ? plan.cluster : 1;
    a.xq_warps = a.cluster_s > 1 ? 1 + kDecEpiThreads / 32 : 1;
    a.M = pb.M;
    a.N = pb.N;
    a.K = pb.K;
    a.Nout = swiglu ? pb.N / 2 : pb.N;
    a.KB = pb.K / 32;
    a.num_kb = (pb.K + 127) / 128;
    a.tiles = plan.tiles;
    a.n_half = pb.N / 2;
    a.total = plan.units;
    a.b_fmt = pb.b_fmt;
    a.epi = pb.epi;
    const uint32_t w_code = e2m1 ? 5u : 0u;  // A (weights): e2m1 or e4m3; B (tokens): e4m3
    if (scaled)
        a.idesc = (w_code << 7) | (0u << 10) | (static_cast<uint32_t>(mt >> 3) << 17) | (1u << 23) |
                  (static_cast<uint32_t>(128 >> 4) << 24);
    else
        a.idesc = (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(mt >> 3) << 17) |
                  (static_cast<uint32_t>(128 >> 4) << 24);
    // transaction bytes count the global-side size (a 128-element e2m1 row is
    // 64 bytes in memory, 128 in shared memory)
    const uint32_t w_row_bytes = e2m1 ? 64u : 128u;
    a.w_tx = static_cast<uint32_t>(swiglu ? 2 : 1) * 128u * w_row_bytes;
    return dec_dispatch(mt, swiglu, scaled, plan.one_per_sm != 0, a.cluster_s > 1,
                        DecLaunch{&a, plan.grid_x, a.cluster_s, st});
}

}  // namespace mxg
