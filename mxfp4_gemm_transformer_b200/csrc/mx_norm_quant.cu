// mx_norm_quant.cu -- residual add + RMSNorm + 1x32 E8M0 quantisation
// of each row, the producer that hands the next GEMM its MX operand
// (sly-radiance README, radiance_fused_norm.py row: add_rms_quant returning
// (q_fp8, scale) for the W4A8 linear; RMSNorm with a plain weight as the DiT
// page's dit.rs rms_norm defines it: x * rsqrt(mean x^2 + eps) * w).
//
// One CTA per row, 256 threads; thread t owns the 8-element vectors t,
// t + 256, ... of the row and keeps the rounded sums r = bf16(x + residual)
// in registers between the two passes:
//   pass 1  r, written back to residual; sum of r^2 (fp32, thread partials,
//           then warp shuffles and one shared-memory step);
//   pass 2  y = bf16(r * rsqrt(mean + eps) * w), optionally stored; each
//           32-wide block (four consecutive threads) takes its E8M0 exponent
//           from the block amax and its e4m3 codes exactly as the 1x32
//           activation quantisation does.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mx_internal.h"
#include "mx_ptx.cuh"
#include "mx_quant_common.cuh"

namespace mxg {
namespace {

template <int VPT>
__global__ void __launch_bounds__(256) add_rms_quant_kernel(const uint4* __restrict__ x, uint4* __restrict__ res,
                                                            const uint4* __restrict__ w, float eps, int K,
                                                            uint4* __restrict__ y_out, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales)
{
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float part[8];
    const int n8 = K / 8;
    const size_t base = static_cast<size_t>(blockIdx.x) * n8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint4 rv[VPT];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int t = threadIdx.x + i * 256;
        rv[i] = make_uint4(0u, 0u, 0u, 0u);
        if (t < n8) {
            float a[8], b[8];
            bf16x8_to_f32(__ldcg(x + base + t), a);
            bf16x8_to_f32(__ldcg(res + base + t), b);
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * j] + b[2 * j], a[2 * j + 1] + b[2 * j + 1]);
                o[j] = *reinterpret_cast<const uint32_t*>(&h);
                const float lo = __low2float(h), hi = __high2float(h);
                ss = fmaf(lo, lo, ss);
                ss = fmaf(hi, hi, ss);
            }
            rv[i] = make_uint4(o[0], o[1], o[2], o[3]);
            res[base + t] = rv[i];
        }
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, s);
    if (lane == 0) part[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) tot += part[i];  // every thread sums the 8 warps in the same order
    const float inv = rsqrtf(tot / static_cast<float>(K) + eps);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int t = threadIdx.x + i * 256;
        const bool live = t < n8;  // n8 % 4 == 0: a block's four threads are live together
        float r[8], wv[8], y[8];
        bf16x8_to_f32(rv[i], r);
        bf16x8_to_f32(live ? __ldg(w + t) : make_uint4(0u, 0u, 0u, 0u), wv);
        uint32_t yb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(r[2 * j] * inv * wv[2 * j], r[2 * j + 1] * inv * wv[2 * j + 1]);
            yb[j] = *reinterpret_cast<const uint32_t*>(&h);
            y[2 * j] = __low2float(h);
            y[2 * j + 1] = __high2float(h);
        }
        float amax = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(y[j]));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        const int e = e8m0_exponent(amax, 8, 0x600000u);
        const float s = pow2_neg(e);
        if (!live) continue;
        if (y_out) y_out[base + t] = make_uint4(yb[0], yb[1], yb[2], yb[3]);
        uint2 q;
        q.x = static_cast<uint32_t>(to_e4m3x2(y[0] * s, y[1] * s)) | (static_cast<uint32_t>(to_e4m3x2(y[2] * s, y[3] * s)) << 16);
        q.y = static_cast<uint32_t>(to_e4m3x2(y[4] * s, y[5] * s)) | (static_cast<uint32_t>(to_e4m3x2(y[6] * s, y[7] * s)) << 16);
        reinterpret_cast<uint2*>(codes)[base + t] = q;
        if ((t & 3) == 0) scales[(base + t) >> 2] = static_cast<uint8_t>(e);
    }
}

template <int VPT>
cudaError_t launch_t(const void* x, void* res, const void* w, float eps, int M, int K, void* y_out, void* codes,
                     void* scales, cudaStream_t st)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(M, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    int na = 0;
    if (launch_flags() & MX_LAUNCH_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, add_rms_quant_kernel<VPT>, static_cast<const uint4*>(x), static_cast<uint4*>(res),
                              static_cast<const uint4*>(w), eps, K, static_cast<uint4*>(y_out),
                              static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
}

}  // namespace

// K % 32 == 0, K <= 16384 (validated by the caller).
cudaError_t launch_add_rms_quant(const void* x, void* res, const void* w, float eps, int M, int K, void* y_out,
                                 void* codes, void* scales, cudaStream_t st)
{
    const int vpt = (K / 8 + 255) / 256;
    if (vpt <= 1) return launch_t<1>(x, res, w, eps, M, K, y_out, codes, scales, st);
    if (vpt <= 2) return launch_t<2>(x, res, w, eps, M, K, y_out, codes, scales, st);
    if (vpt <= 4) return launch_t<4>(x, res, w, eps, M, K, y_out, codes, scales, st);
    return launch_t<8>(x, res, w, eps, M, K, y_out, codes, scales, st);
}

}  // namespace mxg
