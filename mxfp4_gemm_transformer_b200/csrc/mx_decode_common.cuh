// mx_decode_common.cuh -- parts of the decode kernel (mx_decode.cu): the
// launch arguments, the trace stamps, the epilogue value of one output and the
// fused quantisation of bf16 tokens into the token ring.
#pragma once
#include <cuda_bf16.h>

#include "mx_internal.h"
#include "mx_kernel_common.cuh"
#include "mx_ptx.cuh"
#include "mx_quant_common.cuh"

namespace mxg {

struct DecodeArgs {
    CUtensorMap tmW;     // weight codes [N, K]: box {128 elements, 128 rows}
    const uint8_t* x8;   // activation (token) codes [M, K]
    const __nv_bfloat16* xb;  // bf16 activations [M, K] quantised here (x_bf16), else null
    const uint8_t* sw8;  // weight E8M0 scales [N/32, K/32] (32 x 32) or [N, K/32] (1 x 32)
    const uint8_t* sx8;  // activation E8M0 scales [M, K/32]
    const float* swf;    // per-channel fp32 weight scales [N]
    const float* sxf;    // per-token fp32 activation scales [M]
    const float* bias;   // fp32 [N] or null
    __nv_bfloat16* out;  // [M, Nout] (null under MX_EPI_SWIGLU_MXQ)
    uint8_t* q_codes;    // MX_EPI_SWIGLU_MXQ: e4m3 codes [M, Nout]
    uint8_t* q_scales;   // MX_EPI_SWIGLU_MXQ: E8M0 scales [M, Nout / 32]
    unsigned* status;    // workspace status word
    unsigned* counters;  // [tiles] K blocks accumulated so far (zero between launches)
    float* red;          // [tiles][NSUB][M][128] fp32 accumulators (zero between launches)
    unsigned long long* timeline;  // optional per-CTA %globaltimer stamps (null = off)
    int timeline_ctas;
    int prefetch_w;      // weight stages that may be read before the previous kernel completes
    int whole_tiles;     // CTAs take whole tiles: no cross-CTA reduction
    int cluster_s;       // > 1: the K range of one tile split over a cluster of this many CTAs
    int x_bf16;          // tokens arrive as bf16 and are quantised (1 x 32, E8M0) into the token ring
    int xq_warps;        // warps that quantise tokens: the token warp, plus the epilogue warps with a cluster
    int M, N, K, Nout, KB, num_kb, tiles, n_half;
    int total;  // tiles * num_kb units
    int b_fmt, epi;
    uint32_t idesc;
    uint32_t w_tx;  // transaction bytes of one weight stage
};

// Per-CTA trace slots (mx_debug_set_timeline), in %globaltimer ns unless noted:
// start, set-up done, first weight load issued, first unit landed (MMA side),
// last MMA committed, first accumulator ready (epilogue side), epilogue done,
// end; for the last split tile: partial added, count returned, epilogue of the
// reduced tile done; then SM id, units, reduced tiles finished here.
enum DecStamp {
    kDecStart = 0, kDecReady, kDecFirstTma, kDecFirstFull, kDecLastCommit, kDecFirstAcc, kDecEpiDone, kDecEnd,
    kDecRedAdded = 8, kDecCounted = 9, kDecFinalDone = 10, kDecSmid = 11, kDecUnits = 12, kDecFinals = 13,
    kDecSlots = 16
};

__device__ __forceinline__ void dec_stamp(const DecodeArgs& p, int slot, unsigned long long v)
{
    if (MXG_TRACE && p.timeline && static_cast<int>(blockIdx.x) < p.timeline_ctas) p.timeline[blockIdx.x * kDecSlots + slot] = v;
}

// Stamp the current %globaltimer (the timer is read only when tracing is on).
__device__ __forceinline__ void dec_now(const DecodeArgs& p, int slot)
{
    if (MXG_TRACE && p.timeline && static_cast<int>(blockIdx.x) < p.timeline_ctas)
        p.timeline[blockIdx.x * kDecSlots + slot] = globaltimer_ns();
}

// Per-unit detail of CTA 0 (its first 48 units), in the 256 slots after the
// per-CTA records: rows of 48 -- weight load issued, token load issued,
// weights landed (MMA side), tokens landed (MMA side), MMAs committed.
enum DecDetail { kDetW = 0, kDetX, kDetWFull, kDetXFull, kDetCommit, kDetRow = 48 };

__device__ __forceinline__ void dec_detail(const DecodeArgs& p, int row, int i)
{
    if (MXG_TRACE && p.timeline && blockIdx.x == 0 && i < kDetRow)
        p.timeline[static_cast<size_t>(p.timeline_ctas) * kDecSlots + row * kDetRow + i] = globaltimer_ns();
}

constexpr int kDecThreads = 256;
constexpr int kDecEpiThreads = 128;
constexpr int kWBoxes = 4;  // tensor-copy boxes per 128-row weight tile (issued by separate lanes)

// Value of one output from its fp32 accumulators (g: gate or plain, u: up).
template <bool SWIGLU, bool F32ROW>
__device__ __forceinline__ float dec_epi(int epi, float g, float u, float sx, float bg, float bu, float wg, float wu)
{
    if (F32ROW) {
        g *= sx * wg;
        if (SWIGLU) u *= sx * wu;
    }
    if (SWIGLU) {
        g += bg;
        u += bu;
        return sigmoid_mul(g, g) * u;
    }
    if (epi == MX_EPI_NONE) return g;
    g += bg;
    return epi == MX_EPI_BIAS_GELU_TANH ? gelu_tanh(g) : g;
}

// MX_EPI_SWIGLU_MXQ: output value v of column j, token m, handed on as the
// next GEMM's MX operand.  The 32 lanes of the calling warp hold 32
// consecutive output columns of the same token -- one 1 x 32 block -- so the
// block amax is a warp reduction; every lane of the warp must call this
// (lanes outside the output pass col_ok = false and v = 0).  The value is
// rounded to bf16 first, as the unfused chain stores it.
__device__ __forceinline__ void dec_store_mxq(const DecodeArgs& p, int m, int j, bool col_ok, int lane, float v)
{
    const float vb = __bfloat162float(__float2bfloat16_rn(col_ok ? v : 0.f));
    float amax = fabsf(vb);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, s));
    const int e = e8m0_exponent(amax, 8, 0x600000u);
    const uint8_t code = static_cast<uint8_t>(to_e4m3x2(vb * pow2_neg(e), 0.f) & 0xFFu);
    if (col_ok) {
        p.q_codes[static_cast<size_t>(m) * p.Nout + j] = code;
        if (lane == 0) p.q_scales[static_cast<size_t>(m) * (p.Nout / 32) + j / 32] = static_cast<uint8_t>(e);
    }
}

// Fused activation quantisation: the token tile of each unit (M rows x 128 K)
// is quantised from bf16 straight into the token ring, in the layout the
// 128-byte-swizzled descriptor reads (16-byte chunk c of row r at
// r * 128 + ((c ^ (r % 8)) * 16)), and each 32-wide block's E8M0 exponent into
// the scale tile (byte (r % 32) * 16 + (r / 32) * 4 + block, the layout the
// scale copy expects).  The CTA's units hold n_units x M x 4 blocks of 32
// elements, numbered unit-major; `nthreads` threads own every nthreads-th
// block starting at `qid`, so that with few tokens the blocks of different
// units belong to different threads and their loads are in flight together.
// Each thread keeps its next two blocks loaded ahead of their conversion and
// walks the units in order: it waits until the unit's ring stage is free,
// writes its blocks of that unit and fences them to the tensor core's (async)
// proxy; then its warp arrives once on the stage's barrier (every warp
// arrives for every unit, which also keeps each thread within one phase of
// every stage's barriers).  All 32 lanes of each quantising warp call this.  Rows >= M are not written: an MMA output column depends on its
// own token row alone and columns >= M are never stored.
template <class C>
__device__ __forceinline__ void dec_load_block(const DecodeArgs& p, int g0, int b, uint4 (&v)[4])
{
    const int per_unit = p.M * 4;
    const int i = b / per_unit, r4 = b - i * per_unit;
    const int row = r4 >> 2, q = r4 & 3;
    const int kb = (g0 + i) % p.num_kb;
    const uint4* src = reinterpret_cast<const uint4*>(p.xb + static_cast<size_t>(row) * p.K + kb * C::BK + q * 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = __ldcg(src + j);
}

template <class C>
__device__ __forceinline__ void dec_store_block(const DecodeArgs& p, int b, const uint4 (&v)[4], uint8_t* xt,
                                                uint8_t* sf)
{
    const int r4 = b % (p.M * 4);
    const int row = r4 >> 2, q = r4 & 3;
    float f[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float g[8];
        bf16x8_to_f32(v[j], g);
#pragma unroll
        for (int t = 0; t < 8; ++t) f[8 * j + t] = g[t];
    }
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(f[t]));
    const int e = e8m0_exponent(amax, 8, 0x600000u);
    const float inv = pow2_neg(e);
    uint32_t w[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
        w[t] = static_cast<uint32_t>(to_e4m3x2(f[4 * t] * inv, f[4 * t + 1] * inv)) |
               (static_cast<uint32_t>(to_e4m3x2(f[4 * t + 2] * inv, f[4 * t + 3] * inv)) << 16);
    *reinterpret_cast<uint4*>(xt + row * 128 + (((2 * q) ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(xt + row * 128 + (((2 * q + 1) ^ (row & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
    sf[(row & 31) * 16 + (row >> 5) * 4 + q] = static_cast<uint8_t>(e);
}

template <class C>
__device__ __forceinline__ void dec_quant_tokens(const DecodeArgs& p, int g0, int n_units, uint8_t* xring,
                                                 uint8_t* sfb_ring, uint64_t* xfull, uint64_t* xempty,
                                                 volatile int* abort_flag, int qid, int nthreads)
{
    const int per_unit = p.M * 4;
    const int total = n_units * per_unit;
    int nb = qid;              // next owned block to load
    int b0 = total, b1 = total;  // loaded blocks, oldest first (total = none)
    uint4 v0[4], v1[4];
    if (nb < total) {
        dec_load_block<C>(p, g0, nb, v0);
        b0 = nb;
        nb += nthreads;
    }
    if (nb < total) {
        dec_load_block<C>(p, g0, nb, v1);
        b1 = nb;
        nb += nthreads;
    }
    uint32_t xs = 0, xph = 0;
    for (int i = 0; i < n_units; ++i) {
        if (__any_sync(0xFFFFFFFFu, !wait_bar(&xempty[xs], xph ^ 1u, abort_flag, p.status))) break;
        uint8_t* xt = xring + xs * C::X_BYTES;
        uint8_t* sf = sfb_ring + xs * C::SFB_BYTES;
        while (b0 < total && b0 / per_unit == i) {
            dec_store_block<C>(p, b0, v0, xt, sf);
#pragma unroll
            for (int j = 0; j < 4; ++j) v0[j] = v1[j];
            b0 = b1;
            b1 = total;
            if (nb < total) {
                dec_load_block<C>(p, g0, nb, v1);
                b1 = nb;
                nb += nthreads;
            }
        }
        // every lane's writes to the async proxy, then one arrival per warp
        // (one per lane serialised on the barrier measured ~1 us per launch)
        fence_proxy_async_smem();
        __syncwarp();
        if ((qid & 31) == 0) mbar_arrive(&xfull[xs]);
        if (++xs == C::DX) {
            xs = 0;
            xph ^= 1u;
        }
    }
}

}  // namespace mxg
