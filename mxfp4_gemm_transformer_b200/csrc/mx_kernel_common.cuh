// mx_kernel_common.cuh -- device helpers shared by the GEMM kernels: the
// bounded mbarrier wait and the fp32 epilogue math.
#pragma once
#include <cuda_bf16.h>

#include "mx_internal.h"
#include "mx_ptx.cuh"

namespace mxg {

// ---------------------------------------------------------------------------
// bounded wait

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned* status)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > MXG_WATCHDOG_NS) {
            *abort_flag = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag, for teardown: a CTA must not
// leave (or free TMEM) while its own asynchronous operations are in flight.
__device__ __forceinline__ bool wait_bar_final(uint64_t* bar, uint32_t parity, unsigned* status)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > MXG_WATCHDOG_NS) {
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// epilogue math (fp32)

__device__ __forceinline__ float sigmoid_mul(float v, float t)
{
    // v * sigmoid(t) with z = e^-|t| in (0, 1]: v / (1 + z) for t >= 0 and
    // v z / (1 + z) for t < 0, so nothing overflows and the divisor stays in
    // [1, 2].  z = 2^(-|t| log2 e) keeps subnormal values, so the far negative
    // tail (t < -87, where e^t is below fp32's normal range) still gives v e^t.
    const float z = ex2_approx(-fabsf(t) * 1.4426950408889634f);
    return __fdividef(t >= 0.0f ? v : v * z, 1.0f + z);
}

// 0.5 v (1 + tanh(u)) == v * sigmoid(2u), u = sqrt(2/pi) (v + 0.044715 v^3)
__device__ __forceinline__ float gelu_tanh(float v)
{
    const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
    return sigmoid_mul(v, 2.0f * u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Number of epilogue warps of the tile kernels: two per TMEM lane quadrant,
// each taking every other 32-column chunk of the tile.
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;

// One 32-column chunk of one accumulator row: fp32 scales, bias, activation,
// rounded to bf16 pairs.  colp holds the tile's per-column parameters in
// shared memory (bias of gate/plain and up columns, weight scales of both),
// 256 floats each; every lane reads the same address, so the reads are
// broadcasts.
template <int EPI, bool SWIGLU, bool F32ROW>
__device__ __forceinline__ void epi_chunk(const uint32_t (&g)[32], const uint32_t (&h)[32], float sx,
                                          const float* __restrict__ colp, int c, uint32_t (&packed)[16])
{
#pragma unroll
    for (int j2 = 0; j2 < 16; ++j2) {
        float v[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int j = 2 * j2 + t;
            float a = __uint_as_float(g[j]);
            if (F32ROW) a *= sx * colp[512 + c + j];
            if (SWIGLU) {
                float b = __uint_as_float(h[j]);
                if (F32ROW) b *= sx * colp[768 + c + j];
                a += colp[c + j];
                b += colp[256 + c + j];
                v[t] = sigmoid_mul(a, a) * b;
            } else {
                if (EPI != MX_EPI_NONE) a += colp[c + j];
                v[t] = (EPI == MX_EPI_BIAS_GELU_TANH) ? gelu_tanh(a) : a;
            }
        }
        packed[j2] = pack_bf16x2(v[0], v[1]);
    }
}


// The in-place residual epilogue of one 32-column chunk: acc (x row/column
// fp32 scales) + bias (0 without one) + the residual already in out, rounded
// once to bf16 pairs.
template <bool F32ROW>
__device__ __forceinline__ void epi_chunk_residual(const uint32_t (&g)[32], float sx, const float* __restrict__ colp,
                                                   int c, const float (&res)[32], uint32_t (&packed)[16])
{
#pragma unroll
    for (int j2 = 0; j2 < 16; ++j2) {
        float v[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const int j = 2 * j2 + t;
            float a = __uint_as_float(g[j]);
            if (F32ROW) a *= sx * colp[512 + c + j];
            v[t] = (a + colp[c + j]) + res[j];
        }
        packed[j2] = pack_bf16x2(v[0], v[1]);
    }
}

// out[m, col0 .. col0 + 31] as fp32, the residual the in-place epilogue adds
// (zeros past the `lim` valid columns, or for rows >= M).
__device__ __forceinline__ void load_row32_bf16(const __nv_bfloat16* out, int Nout, int M, int m, int col0, int lim,
                                                float (&r)[32])
{
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = 0.f;
    if (m >= M || lim <= 0) return;
    const __nv_bfloat16* src = out + static_cast<size_t>(m) * Nout + col0;
    if (lim >= 32 && (Nout & 7) == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src) + q);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                r[8 * q + 2 * t] = __uint_as_float(w[t] << 16);
                r[8 * q + 2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < lim) r[j] = __bfloat162float(src[j]);
    }
}

// Final store of one output element; the in-place residual epilogue first
// adds the value already there.
__device__ __forceinline__ void store_out(__nv_bfloat16* o, int epi, float v)
{
    if (epi == MX_EPI_RESIDUAL) v += __bfloat162float(*o);
    *o = __float2bfloat16_rn(v);
}

// Stores one warp's 32 x 32 chunk of bf16 results (row = lane, 16 packed
// pairs per lane) through `buf`, 2 KB of the warp's own shared memory.  Each
// lane parks its row's 64 bytes there, 16-byte pieces XOR-swizzled by row
// pair (no bank conflicts on either side), then four lanes write one row's 64
// contiguous bytes, eight rows a pass, so every global store covers whole
// 32-byte sectors.  row0 = output row of lane 0, col0 = output column of the
// chunk's first column, lim = valid columns (<= 32); rows >= M are skipped.
__device__ __forceinline__ void store_chunk_staged(uint8_t* buf, const uint32_t (&pk)[16], int lane,
                                                   __nv_bfloat16* out, int Nout, int M, int row0, int col0, int lim)
{
    __syncwarp();  // the previous chunk's reads of buf are done
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) * 16)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    __syncwarp();
    const int sub = lane & 3, col8 = sub * 8;
    const bool vec_ok = (Nout & 7) == 0;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
        const int rr = pass * 8 + (lane >> 2);
        const int mr = row0 + rr;
        if (mr >= M || col8 >= lim) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(buf + rr * 64 + ((sub ^ ((rr >> 1) & 3)) * 16));
        __nv_bfloat16* o = out + static_cast<size_t>(mr) * Nout + col0 + col8;
        if (vec_ok && col8 + 8 <= lim) {
            *reinterpret_cast<uint4*>(o) = v;
        } else {
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
            for (int j = 0; j < 8 && col8 + j < lim; ++j)
                reinterpret_cast<uint16_t*>(o)[j] =
                    static_cast<uint16_t>((j & 1) ? (vv[j >> 1] >> 16) : (vv[j >> 1] & 0xFFFFu));
        }
    }
}

}  // namespace mxg
