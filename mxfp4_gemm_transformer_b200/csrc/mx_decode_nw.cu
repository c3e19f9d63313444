// mx_decode_nw.cu -- the decode-shaped GEMM (M <= 64 tokens) with the
// weights on the MMA's N side, for the E8M0 block-scaled formats.
//
//   out[m, n] = epilogue( sum_k x[m, k] w[n, k] )   with few tokens m
//
// A block-scaled tcgen05 MMA takes about the same issue time whatever its N
// (measured ~126 cycles for M = 128 from N = 16 to N = 256).  With the
// weights on the 128-row side (mx_decode.cu) one instruction moves 128
// weight rows x 32 K; here the weights are the instruction's N, 240 rows
// (SwiGLU: 120 gate rows and the matching 120 up rows), and the tokens its
// M side (128 TMEM lanes, only the first M real), so each instruction moves
// 1.9x the weight bytes.  240 rather than 256 keeps the accumulator
// (240 columns) and the scale factors (12 columns) inside 256 TMEM columns,
// so two CTAs still fit on an SM.
//
// Units are (tile of 240 weight rows, 128-wide K block).  A tile's K range is
// split over a thread-block cluster of up to 16 CTAs (partials reduced in
// distributed shared memory in rank order), or CTAs take whole tiles.
//
// Warp roles (256 threads): warp 0 weight TMA (boxes of 48 rows, or 40 rows
// per SwiGLU half), warp 1 MMA issue, warp 2 weight-scale copies, warp 3 token
// tiles (copied, or quantised from bf16), warps 4-7 epilogue (thread = TMEM
// lane = token row, columns = weight rows).  Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mx_decode_common.cuh"
#include "mx_internal.h"
#include "mx_kernel_common.cuh"
#include "mx_ptx.cuh"

namespace mxg {

constexpr int kNwRows = 240;  // weight rows per tile: the MMA's N

// MT = token rows held per stage (the MMA's M is 128; rows past MT read
// whatever follows in shared memory and land in output rows never stored);
// NSUB = 2 for SwiGLU (gate | up halves of the 240 rows); ONE_PER_SM = the
// whole SM's shared memory for one CTA instead of at most 113 KB.
template <int MT, int NSUB, bool ONE_PER_SM>
struct DecNwCfg {
    static constexpr int BK = 128;
    static constexpr int WROWS = kNwRows;
    static constexpr int OUT = NSUB == 2 ? WROWS / 2 : WROWS;  // output columns per tile
    static constexpr int W_BYTES = WROWS * BK;                 // e2m1 lands unpacked: a byte per element
    static constexpr int X_BYTES = MT * BK;
    static constexpr int SFA_BYTES = 1024;  // weight scales: two 128-row tcgen05.cp chunks
    static constexpr int SFB_BYTES = 512;   // token scales: one chunk
    static constexpr int BAR_BYTES = 512;
    static constexpr int LIMIT = ONE_PER_SM ? 232448 : 115712;
    static constexpr int USABLE = LIMIT - 1024 - BAR_BYTES;
    static constexpr int DX = ONE_PER_SM ? (MT <= 32 ? 8 : 4) : (MT <= 32 ? 4 : 2);
    // token ring first: the MMA reads 128 token rows per stage, and rows past
    // MT then run into later stages or the weight ring, inside the CTA
    static constexpr int OFF_X = 0;
    static constexpr int OFF_W = ((DX * X_BYTES + 1023) / 1024) * 1024;
    static constexpr int DW_FIT = (USABLE - OFF_W - DX * SFB_BYTES) / (W_BYTES + SFA_BYTES);
    static constexpr int DW = DW_FIT > 8 ? 8 : DW_FIT;
    static constexpr int OFF_SFA = OFF_W + DW * W_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + DW * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + DX * SFB_BYTES;
    static constexpr int SMEM_BYTES = 1024 + OFF_BAR + BAR_BYTES;
    // TMEM: accumulator [128 lanes][240 columns], then 8 columns of weight
    // scales (4 per 128-row chunk) and 4 of token scales
    static constexpr int ACC_COLS = WROWS;
    static constexpr int SF_W = ACC_COLS;
    static constexpr int SF_X = SF_W + 8;
    static constexpr int TMEM_COLS = 256;
    // cluster partial: [MT][PSTRIDE] fp32 in the weight ring (odd stride:
    // the 32 token rows of a warp write a column into 32 different banks)
    static constexpr int PSTRIDE = WROWS + 1;
    static_assert(DW >= 2, "shared memory too small for two weight stages");
    static_assert(SF_X + 4 <= TMEM_COLS, "TMEM budget is half an SM");
    static_assert(SMEM_BYTES <= LIMIT, "over the shared-memory budget");
    static_assert(OFF_W % 1024 == 0 && OFF_SFA % 1024 == 0 && OFF_BAR % 16 == 0, "alignment");
    static_assert((DX - 1) * X_BYTES + 128 * BK <= OFF_SFA, "token rows read past MT stay in shared memory");
    static_assert(DW * W_BYTES >= MT * PSTRIDE * 4, "the weight ring holds a cluster partial");
    static_assert(OUT % 8 == 0 && (NSUB == 1 ? WROWS % 48 == 0 : OUT % 40 == 0), "box split");
};

template <int MT, int NSUB, bool ONE_PER_SM>
__global__ void __launch_bounds__(kDecThreads, ONE_PER_SM ? 1 : 2)
    decode_nw_kernel(const __grid_constant__ DecodeArgs p)
{
    using C = DecNwCfg<MT, NSUB, ONE_PER_SM>;
    constexpr bool SWIGLU = NSUB == 2;
    constexpr int NBOX = SWIGLU ? 6 : 5;          // weight boxes per unit
    constexpr int BOX_ROWS = SWIGLU ? 40 : 48;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* xring = base + C::OFF_X;       // [DX][X_BYTES]
    uint8_t* wring = base + C::OFF_W;       // [DW][W_BYTES]
    uint8_t* sfa_ring = base + C::OFF_SFA;  // [DW][SFA_BYTES] weight scales
    uint8_t* sfb_ring = base + C::OFF_SFB;  // [DX][SFB_BYTES] token scales
    uint64_t* wfull = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
    uint64_t* wempty = wfull + C::DW;
    uint64_t* xfull = wempty + C::DW;
    uint64_t* xempty = xfull + C::DX;
    uint64_t* acc_full = xempty + C::DX;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* final_bar = acc_empty + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool leader = elect_one();

    // this CTA's units [g0, g1) (unit = tile * num_kb + K block)
    int g0, g1;
    const int S = p.cluster_s;
    const int crank = S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
    if (S > 1) {
        const int tile = static_cast<int>(blockIdx.x) / S;
        g0 = tile * p.num_kb + crank * p.num_kb / S;
        g1 = tile * p.num_kb + (crank + 1) * p.num_kb / S;
    } else {
        g0 = static_cast<int>(static_cast<long long>(blockIdx.x) * p.tiles / gridDim.x) * p.num_kb;
        g1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.tiles / gridDim.x) * p.num_kb;
    }
    const int n_units = g1 - g0;

    if (threadIdx.x == 0) {
        dec_now(p, kDecStart);
        prefetch_tmap(&p.tmW);
        for (int s = 0; s < C::DW; ++s) {
            mbar_init(&wfull[s], 1 + 32);  // the tensor copies' transaction bytes + 32 scale-copy lanes
            mbar_init(&wempty[s], 1);
        }
        const uint32_t x_arrivals = p.x_bf16 ? 32u * static_cast<uint32_t>(p.xq_warps) : 32u;
        for (int s = 0; s < C::DX; ++s) {
            mbar_init(&xfull[s], x_arrivals);
            mbar_init(&xempty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kDecEpiThreads / 32);
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
    if (threadIdx.x == 0) {
        pdl_launch_dependents();
        dec_now(p, kDecReady);
    }

    if (warp == 0) {
        // ------------------------------------------------ weight-tile producer
        // Weights do not depend on the previous kernel: with weight prefetch
        // allowed the ring fills before the dependency wait.  A unit's 240
        // rows are requested as NBOX boxes, one per lane.
        const uint64_t pol_w = policy_evict_first();
        uint32_t armed = 0, used = 0;
        uint32_t ws = 0, wph = 0;
        for (int i = 0; i < n_units; ++i) {
            const int g = g0 + i;
            const int tile = g / p.num_kb, kb = g - tile * p.num_kb;
            if (i == p.prefetch_w) pdl_wait();
            if (__any_sync(0xFFFFFFFFu, !wait_bar(&wempty[ws], wph ^ 1u, abort_flag, p.status))) break;
            if (lane == 0) mbar_arrive_expect_tx(&wfull[ws], p.w_tx);
            __syncwarp();
            if (lane < NBOX) {
                int row0, srow;
                if (SWIGLU) {
                    const int h = lane / 3, j = lane % 3;
                    row0 = (h ? p.n_half : 0) + tile * C::OUT + j * BOX_ROWS;
                    srow = h * C::OUT + j * BOX_ROWS;
                } else {
                    row0 = tile * C::WROWS + lane * BOX_ROWS;
                    srow = lane * BOX_ROWS;
                }
                tma_load_2d(wring + ws * C::W_BYTES + srow * C::BK, &p.tmW, &wfull[ws], kb * C::BK, row0, pol_w);
            }
            if (lane == 0 && i == 0) dec_now(p, kDecFirstTma);
            used |= 1u << ws;
            armed = (armed & ~(1u << ws)) | (wph << ws);
            if (++ws == C::DW) {
                ws = 0;
                wph ^= 1u;
            }
        }
        if (lane == 0)
            for (int s = 0; s < C::DW; ++s)
                if (used & (1u << s)) wait_bar_final(&wfull[s], (armed >> s) & 1u, p.status);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // D[token][weight row] += X (A, 128 rows) x W (B, 240 rows) per K step
        const uint32_t sfw = tmem + C::SF_W, sfx = tmem + C::SF_X;
        const uint32_t w_s = smem_u32(wring), x_s = smem_u32(xring);
        const uint32_t sfa_s = smem_u32(sfa_ring), sfb_s = smem_u32(sfb_ring);
        uint32_t ws = 0, wph = 0, xs = 0, xph = 0, acc_phase = 0;
        int g = g0;
        while (g < g1) {
            const int tile = g / p.num_kb;
            const int seg_end = min(g1, (tile + 1) * p.num_kb);
            if (__any_sync(0xFFFFFFFFu, !wait_bar(acc_empty, acc_phase ^ 1u, abort_flag, p.status))) break;
            tc_fence_after();
            uint32_t accumulate = 0;
            bool ok = true;
            for (; g < seg_end; ++g) {
                const bool wok = wait_bar(&wfull[ws], wph, abort_flag, p.status);
                const bool xok = wok && wait_bar(&xfull[xs], xph, abort_flag, p.status);
                if (__any_sync(0xFFFFFFFFu, !xok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                fence_proxy_async_smem();  // token tiles and scales were written by cp.async or st.shared
                if (leader) {
                    if (g == g0) dec_now(p, kDecFirstFull);
                    const uint32_t sW = w_s + ws * C::W_BYTES;
                    const uint32_t sX = x_s + xs * C::X_BYTES;
                    tc_cp_32x128b_x4(sfw, sdesc_sf(sfa_s + ws * C::SFA_BYTES));
                    tc_cp_32x128b_x4(sfw + 4, sdesc_sf(sfa_s + ws * C::SFA_BYTES + 512));
                    tc_cp_32x128b_x4(sfx, sdesc_sf(sfb_s + xs * C::SFB_BYTES));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_mx(tmem, sdesc_sw128(sX + kk * 32), sdesc_sw128(sW + kk * 32),
                               p.idesc | (static_cast<uint32_t>(kk) << 4) | (static_cast<uint32_t>(kk) << 29), sfx,
                               sfw, (kk > 0) ? 1u : accumulate);
                    // release a stage only when a later unit refills it
                    if (g - g0 + C::DW < n_units) tc_commit(&wempty[ws]);
                    if (g - g0 + C::DX < n_units) tc_commit(&xempty[xs]);
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
                tc_commit(acc_full);
                if (g == g1) dec_now(p, kDecLastCommit);
            }
            __syncwarp();
            acc_phase ^= 1u;
        }
    } else if (warp == 2) {
        // ------------------------------------------------ weight-scale producer
        // 240 weight rows in two 128-row tcgen05.cp chunks (rows 240-255
        // zero): row r of the unit -> byte (r / 128) * 512 + (r % 32) * 16 +
        // ((r % 128) / 32) * 4 + K block, with 4-byte asynchronous copies.
        const int KB = p.KB;
        const bool blk32 = p.b_fmt == MX_B_E4M3_E8M0_32X32;
        uint32_t ws = 0, wph = 0;
        for (int i = 0; i < n_units; ++i) {
            const int g = g0 + i;
            const int tile = g / p.num_kb, kb = g - tile * p.num_kb;
            if (i == p.prefetch_w) pdl_wait();
            if (!wait_bar(&wempty[ws], wph ^ 1u, abort_flag, p.status)) break;
            uint8_t* sf = sfa_ring + ws * C::SFA_BYTES;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = lane + 32 * j;
                int n;
                if (SWIGLU)
                    n = r < C::OUT ? tile * C::OUT + r : p.n_half + tile * C::OUT + (r - C::OUT);
                else
                    n = tile * C::WROWS + r;
                const bool ok = r < C::WROWS && n < p.N;
                const int nn = ok ? n : 0;
                const uint8_t* src = p.sw8 + static_cast<size_t>(blk32 ? (nn >> 5) : nn) * KB + kb * 4;
                cp_async_4(sf + (r >> 7) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4, src, ok ? 4u : 0u);
            }
            cp_async_arrive_noinc(&wfull[ws]);
            if (++ws == C::DW) {
                ws = 0;
                wph ^= 1u;
            }
        }
        cp_async_wait_all();
    } else if (warp == 3) {
        // ------------------------------------------------ token producer
        // Token rows (and their scales) into the swizzled token stage, only
        // the M real rows; or quantised from bf16 (see dec_quant_tokens).
        pdl_wait();
        if (p.x_bf16) {
            dec_quant_tokens<C>(p, g0, n_units, xring, sfb_ring, xfull, xempty, abort_flag, lane, 32 * p.xq_warps);
        } else {
            uint32_t xs = 0, xph = 0;
            for (int i = 0; i < n_units; ++i) {
                const int kb = (g0 + i) % p.num_kb;
                if (!wait_bar(&xempty[xs], xph ^ 1u, abort_flag, p.status)) break;
                uint8_t* xt = xring + xs * C::X_BYTES;
                const uint8_t* src0 = p.x8 + static_cast<size_t>(kb) * C::BK;
#pragma unroll
                for (int t = 0; t < MT * 8 / 32; ++t) {
                    const int idx = lane + 32 * t;
                    const int row = idx >> 3, c = idx & 7;
                    if (row < p.M)
                        cp_async_16(xt + row * 128 + ((c ^ (row & 7)) << 4), src0 + static_cast<size_t>(row) * p.K + c * 16,
                                    16u);
                }
                uint8_t* sf = sfb_ring + xs * C::SFB_BYTES;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = lane + 32 * j;
                    if (m < p.M) cp_async_4(sf + lane * 16 + j * 4, p.sx8 + static_cast<size_t>(m) * p.KB + kb * 4, 4u);
                }
                cp_async_arrive_noinc(&xfull[xs]);
                if (++xs == C::DX) {
                    xs = 0;
                    xph ^= 1u;
                }
            }
            cp_async_wait_all();
        }
    } else {
        // ------------------------------------------------ epilogue (warps 4-7)
        // warp q reads TMEM lanes 32q..32q+31 = token rows; a warp whose rows
        // are all >= M skips the TMEM reads (they are warp-wide instructions)
        const int q = warp & 3;
        const int et = threadIdx.x - 128;
        const int m = q * 32 + lane;  // this thread's token row
        const int M = p.M;
        const bool warp_rows = q * 32 < M;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
        pdl_wait();
        if (p.x_bf16 && p.xq_warps > 1)
            dec_quant_tokens<C>(p, g0, n_units, xring, sfb_ring, xfull, xempty, abort_flag, 32 + et, 32 * p.xq_warps);
        if (S > 1) {
            // one tile: park this CTA's partial [M][PSTRIDE] in its weight
            // ring (its MMAs, the last readers of the ring, have completed);
            // the cluster reduces the partials after the role loops
            const bool ready = n_units == 0 || wait_bar(acc_full, 0, abort_flag, p.status);
            if (!named_bar_or(1, kDecEpiThreads, !ready || *abort_flag)) {
                tc_fence_after();
                if (et == 0) dec_now(p, kDecFirstAcc);
                float* part = reinterpret_cast<float*>(wring);
                if (warp_rows) {
#pragma unroll 1
                    for (int c0 = 0; c0 < C::WROWS; c0 += 16) {
                        uint32_t v[16];
                        if (n_units > 0) {
                            tmem_ld16(lane_base + c0, v);
                            tmem_ld_wait();
                        } else {
#pragma unroll
                            for (int t = 0; t < 16; ++t) v[t] = 0u;
                        }
                        if (m < M)
#pragma unroll
                            for (int t = 0; t < 16; ++t) part[m * C::PSTRIDE + c0 + t] = __uint_as_float(v[t]);
                    }
                }
                tc_fence_before();
            }
        } else {
            // whole tiles: epilogue straight from TMEM
            uint32_t acc_phase = 0;
            for (int g = g0; g < g1; g += p.num_kb) {
                const int tile = g / p.num_kb;
                const bool ready = wait_bar(acc_full, acc_phase, abort_flag, p.status);
                // uniform exit decision for all epilogue warps
                if (named_bar_or(1, kDecEpiThreads, !ready || *abort_flag)) break;
                tc_fence_after();
                if (et == 0 && g == g0) dec_now(p, kDecFirstAcc);
                if (warp_rows) {
                    __nv_bfloat16* orow = p.out + static_cast<size_t>(m < M ? m : 0) * p.Nout;
                    if (SWIGLU) {
#pragma unroll 1
                        for (int c0 = 0; c0 < C::OUT; c0 += 8) {
                            uint32_t gv[8], uv[8];
                            tmem_ld8(lane_base + c0, gv);
                            tmem_ld8(lane_base + C::OUT + c0, uv);
                            tmem_ld_wait();
                            if (m < M) {
#pragma unroll
                                for (int t = 0; t < 8; ++t) {
                                    const int j = tile * C::OUT + c0 + t;
                                    if (j < p.Nout) {
                                        const float bg = p.bias ? __ldg(p.bias + j) : 0.f;
                                        const float bu = p.bias ? __ldg(p.bias + j + p.n_half) : 0.f;
                                        store_out(orow + j, p.epi, dec_epi<true, false>(
                                            p.epi, __uint_as_float(gv[t]), __uint_as_float(uv[t]), 1.f, bg, bu, 1.f,
                                            1.f));
                                    }
                                }
                            }
                        }
                    } else {
#pragma unroll 1
                        for (int c0 = 0; c0 < C::WROWS; c0 += 16) {
                            uint32_t v[16];
                            tmem_ld16(lane_base + c0, v);
                            tmem_ld_wait();
                            if (m < M) {
#pragma unroll
                                for (int t = 0; t < 16; ++t) {
                                    const int j = tile * C::WROWS + c0 + t;
                                    if (j < p.Nout) {
                                        const float bg = p.bias ? __ldg(p.bias + j) : 0.f;
                                        store_out(orow + j, p.epi, dec_epi<false, false>(
                                            p.epi, __uint_as_float(v[t]), 0.f, 1.f, bg, 0.f, 1.f, 1.f));
                                    }
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                acc_phase ^= 1u;
            }
        }
        if (et == 0) dec_now(p, kDecEpiDone);
    }
    __syncwarp();

    if (S > 1) {
        // ---------------------------------------------------- cluster reduction
        cluster_sync_all();
        if (threadIdx.x == 0) dec_now(p, kDecCounted);
        if (!*abort_flag) {
            // rank r finishes output columns [r OUT / S, (r + 1) OUT / S) of
            // the tile for every token: partials summed in rank order
            // (deterministic), epilogue, bf16 store
            const int tile = static_cast<int>(blockIdx.x) / S;
            const int c_lo = crank * C::OUT / S, ncols = (crank + 1) * C::OUT / S - c_lo;
            const int M = p.M;
            const uint32_t part_s = smem_u32(wring);
            const int total_e = ncols * M;
            for (int e = threadIdx.x; e < total_e; e += kDecThreads) {
                const int m = e / ncols, c = c_lo + e % ncols;
                const uint32_t off_g = static_cast<uint32_t>((m * C::PSTRIDE + c) * 4);
                const uint32_t off_u = static_cast<uint32_t>((m * C::PSTRIDE + C::OUT + c) * 4);
                float vg[16], vu[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if (r < S) {
                        const uint32_t peer = map_peer_smem(part_s, static_cast<uint32_t>(r));
                        vg[r] = ld_dsmem_f32_batch(peer + off_g);
                        vu[r] = SWIGLU ? ld_dsmem_f32_batch(peer + off_u) : 0.f;
                    }
                }
                float sg = 0.f, su = 0.f;
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    if (r < S) {
                        sg += vg[r];
                        if (SWIGLU) su += vu[r];
                    }
                }
                const int j = tile * C::OUT + c;
                if (j < p.Nout) {
                    const float bg = p.bias ? __ldg(p.bias + j) : 0.f;
                    const float bu = (SWIGLU && p.bias) ? __ldg(p.bias + j + p.n_half) : 0.f;
                    store_out(p.out + static_cast<size_t>(m) * p.Nout + j, p.epi,
                              dec_epi<SWIGLU, false>(p.epi, sg, su, 1.f, bg, bu, 1.f, 1.f));
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

template <int MT, int NSUB, bool ONE>
cudaError_t prepare_decode_nw()
{
    using C = DecNwCfg<MT, NSUB, ONE>;
    auto kern = decode_nw_kernel<MT, NSUB, ONE>;
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && !done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        // clusters of up to 16 CTAs (beyond the portable 8)
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

struct NwLaunch {
    const DecodeArgs* args;
    int grid;
    int cluster;
    cudaStream_t st;
    template <int MT, int NSUB, bool ONE>
    cudaError_t run() const
    {
        using C = DecNwCfg<MT, NSUB, ONE>;
        cudaError_t e = prepare_decode_nw<MT, NSUB, ONE>();
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
        return cudaLaunchKernelEx(&cfg, decode_nw_kernel<MT, NSUB, ONE>, *args);
    }
    cudaError_t invalid() const { return cudaErrorInvalidValue; }
};

// Clusters of `cluster` CTAs the device runs at once (cached; 0 = cannot).
struct NwClusters {
    int cluster;
    template <int MT, int NSUB, bool ONE>
    int run() const
    {
        using C = DecNwCfg<MT, NSUB, ONE>;
        static std::mutex mu;
        static int cache[64][17] = {};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64 || cluster < 1 || cluster > 16) return 0;
        {
            std::lock_guard<std::mutex> lk(mu);
            if (cache[dev][cluster]) return cache[dev][cluster] > 0 ? cache[dev][cluster] : 0;
        }
        if (prepare_decode_nw<MT, NSUB, ONE>() != cudaSuccess) return 0;
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
        if (cudaOccupancyMaxActiveClusters(&n, decode_nw_kernel<MT, NSUB, ONE>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        std::lock_guard<std::mutex> lk(mu);
        cache[dev][cluster] = n > 0 ? n : -1;
        return n;
    }
    int invalid() const { return 0; }
};

struct NwStages {
    template <int MT, int NSUB, bool ONE>
    int run() const { return DecNwCfg<MT, NSUB, ONE>::DW; }
    int invalid() const { return 0; }
};

template <class Op>
auto nw_dispatch(int mt, bool swiglu, bool one, const Op& op) -> decltype(op.invalid())
{
#define MXG_NW(T, O) \
    if (mt == T && one == O) return swiglu ? op.template run<T, 2, O>() : op.template run<T, 1, O>();
    MXG_NW(32, false)
    MXG_NW(64, false)
    MXG_NW(32, true)
    MXG_NW(64, true)
#undef MXG_NW
    return op.invalid();
}

}  // namespace

// Fills `plan` for the weights-on-N decode kernel.  split: kDecCluster (a
// cluster of `cluster` CTAs per tile, up to 16) or kDecWholeTiles (`grid`
// CTAs take whole tiles).  per_sm: 1 or 2 CTAs per SM (0 = choose).  Only the
// E8M0 formats; K % 128 == 0 (4-byte scale copies).
bool plan_decode_nw(const GemmProblem& pb, int split, int grid, int cluster, int per_sm, GemmPlan* plan)
{
    const bool swiglu = epi_swiglu(pb.epi);
    if (!a_fmt_e8m0(pb.a_fmt) || pb.b_fmt == MX_B_E4M3_F32_ROW) return false;
    if (pb.M < 1 || pb.M > 64 || (pb.K % 128) != 0) return false;
    const int out_cols = swiglu ? kNwRows / 2 : kNwRows;
    const int nout = swiglu ? pb.N / 2 : pb.N;
    const int tiles = (nout + out_cols - 1) / out_cols;
    const int num_kb = pb.K / 128;
    const long long total = static_cast<long long>(tiles) * num_kb;
    if (total > 0x7FFFFFFFLL) return false;
    const int mt = pb.M <= 32 ? 32 : 64;
    int g = 1, S = 1;
    long long per_cta = 0;
    if (split == kDecCluster) {
        S = std::max(1, std::min(cluster, std::min(16, num_kb)));
        if (S < 2 || static_cast<long long>(tiles) * S > 0x7FFFFFFFLL) return false;
        g = tiles * S;
        per_cta = (num_kb + S - 1) / S;
    } else if (split == kDecWholeTiles) {
        g = std::max(1, std::min(grid, tiles));
        per_cta = static_cast<long long>((tiles + g - 1) / g) * num_kb;
    } else {
        return false;
    }
    bool one = per_sm == 1;
    if (per_sm == 0) one = per_cta > 3LL * nw_dispatch(mt, swiglu, false, NwStages{});
    if (S > 1 && nw_dispatch(mt, swiglu, one, NwClusters{S}) < 1) return false;
    plan->kernel = 2;
    plan->block_n = kNwRows;
    plan->block_m = mt;
    plan->a_rows = mt;
    plan->tiles = tiles;
    plan->whole_tiles = split == kDecWholeTiles ? 1 : 0;
    plan->reduce = 0;
    plan->cluster = S;
    plan->one_per_sm = one ? 1 : 0;
    plan->grid_x = g;
    plan->grid_y = 1;
    plan->units = static_cast<int>(total);
    plan->splits = split == kDecCluster ? S : 1;
    plan->gsplit = 0;
    plan->part_rows = 0;
    plan->ws_bytes = kWorkspaceHeader;
    plan->acc_bufs = 1;
    plan->stages = nw_dispatch(mt, swiglu, one, NwStages{});
    return true;
}

cudaError_t launch_decode_nw(const GemmProblem& pb, const GemmPlan& plan, cudaStream_t st)
{
    const bool swiglu = epi_swiglu(pb.epi);
    const bool e2m1 = pb.b_fmt == MX_B_E2M1_E8M0_1X32;
    DecodeArgs a;
    memset(&a, 0, sizeof(a));
    const uint32_t box_rows = swiglu ? 40u : 48u;
    if (e2m1) {
        if (!make_tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, pb.b_codes, pb.K, pb.N, pb.K / 2, 128,
                          box_rows))
            return cudaErrorInvalidValue;
    } else {
        if (!make_tmap_2d(&a.tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, pb.b_codes, pb.K, pb.N, pb.K, 128, box_rows))
            return cudaErrorInvalidValue;
    }
    a.x_bf16 = pb.a_fmt == MX_A_BF16_E8M0_1X32 ? 1 : 0;
    a.x8 = a.x_bf16 ? nullptr : static_cast<const uint8_t*>(pb.a_codes);
    a.xb = a.x_bf16 ? static_cast<const __nv_bfloat16*>(pb.a_codes) : nullptr;
    a.sw8 = static_cast<const uint8_t*>(pb.b_scales);
    a.sx8 = a.x_bf16 ? nullptr : static_cast<const uint8_t*>(pb.a_scales);
    a.bias = pb.bias;
    a.out = static_cast<__nv_bfloat16*>(pb.out);
    a.status = pb.status;
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
    a.num_kb = pb.K / 128;
    a.tiles = plan.tiles;
    a.n_half = pb.N / 2;
    a.total = plan.units;
    a.b_fmt = pb.b_fmt;
    a.epi = pb.epi;
    // A (tokens) e4m3; B (weights) e4m3 or e2m1; M = 128, N = 240, E8M0 scales
    const uint32_t w_code = e2m1 ? 5u : 0u;
    a.idesc = (0u << 7) | (w_code << 10) | (static_cast<uint32_t>(kNwRows >> 3) << 17) | (1u << 23) |
              (static_cast<uint32_t>(128 >> 4) << 24);
    // transaction bytes count the global-side size (e2m1 rows are 64 bytes)
    a.w_tx = static_cast<uint32_t>(kNwRows) * (e2m1 ? 64u : 128u);
    return nw_dispatch(plan.block_m, swiglu, plan.one_per_sm != 0, NwLaunch{&a, plan.grid_x, a.cluster_s, st});
}

}  // namespace mxg
