// mx_api.cu -- the extern "C" boundary of libmxgemm.so: argument validation,
// device checks, and dispatch to the quantisation and GEMM launchers.
// Validation happens before any CUDA call, so bad arguments are reported
// (and nothing is launched) even on a machine without a GPU.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <algorithm>

#include "mx_internal.h"

namespace mxg {

namespace {
constexpr size_t kWorkspaceBytes = 256;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

mx_status arch_ok(DeviceInfo* info)
{
    if (current_device(info) != cudaSuccess) return MX_ERR_CUDA;
    if (info->major != 10 || info->minor != 0) return MX_ERR_ARCH;
    return MX_OK;
}

mx_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MX_OK : MX_ERR_CUDA; }
}  // namespace

cudaError_t current_device(DeviceInfo* out)
{
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev].device != dev) {
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess) return e;
        cache[dev].device = dev;
        cache[dev].sms = prop.multiProcessorCount;
        cache[dev].major = prop.major;
        cache[dev].minor = prop.minor;
        cache[dev].smem_optin = prop.sharedMemPerBlockOptin;
    }
    *out = cache[dev];
    return cudaSuccess;
}

mx_status validate_gemm(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                               const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out, int M,
                               int N, int K)
{
    const bool a_bf16 = a_fmt == MX_A_BF16_E8M0_1X32;  // a_scales unused
    if (!a_codes || (!a_scales && !a_bf16) || !b_codes || !b_scales || !out) return MX_ERR_NULL;
    if (epi != MX_EPI_NONE && epi != MX_EPI_BIAS && epi != MX_EPI_BIAS_GELU_TANH && epi != MX_EPI_SWIGLU &&
        epi != MX_EPI_RESIDUAL && epi != MX_EPI_SWIGLU_MXQ)
        return MX_ERR_FORMAT;
    const bool pair_ok = ((a_fmt == MX_A_E4M3_E8M0_1X32 || a_bf16) &&
                          (b_fmt == MX_B_E4M3_E8M0_32X32 || b_fmt == MX_B_E2M1_E8M0_1X32)) ||
                         (a_fmt == MX_A_E4M3_F32_ROW && b_fmt == MX_B_E4M3_F32_ROW) ||
                         (a_fmt == MX_A_E2M1_E8M0_1X32 && b_fmt == MX_B_E2M1_E8M0_1X32);
    if (!pair_ok) return MX_ERR_FORMAT;
    if ((epi == MX_EPI_BIAS || epi == MX_EPI_BIAS_GELU_TANH) && !bias) return MX_ERR_NULL;
    if (epi == MX_EPI_NONE && bias) return MX_ERR_FORMAT;
    if (M < 1 || N < 1 || K < 32 || (K % 32) != 0) return MX_ERR_SHAPE;
    if (b_fmt == MX_B_E4M3_E8M0_32X32 && (N % 32) != 0) return MX_ERR_SHAPE;
    if (b_fmt == MX_B_E2M1_E8M0_1X32 && (K % 128) != 0) return MX_ERR_SHAPE;
    if (epi_swiglu(epi) && (N % 64) != 0) return MX_ERR_SHAPE;
    if (!aligned(a_codes, 16) || !aligned(b_codes, b_fmt == MX_B_E2M1_E8M0_1X32 ? 32 : 16) || !aligned(out, 16))
        return MX_ERR_ALIGN;
    const uintptr_t sal = (a_fmt == MX_A_E4M3_F32_ROW) ? 4 : 1;
    if ((!a_bf16 && !aligned(a_scales, sal)) || !aligned(b_scales, sal) || (bias && !aligned(bias, 4)))
        return MX_ERR_ALIGN;
    return MX_OK;
}

}  // namespace mxg

using namespace mxg;

extern "C" {

const char* mx_status_string(mx_status s)
{
    switch (s) {
    case MX_OK: return "MX_OK";
    case MX_ERR_NULL: return "MX_ERR_NULL: a required pointer is NULL";
    case MX_ERR_SHAPE: return "MX_ERR_SHAPE: size out of range or not a required multiple";
    case MX_ERR_ALIGN: return "MX_ERR_ALIGN: pointer not aligned as required";
    case MX_ERR_FORMAT: return "MX_ERR_FORMAT: unknown or invalid format / epilogue combination";
    case MX_ERR_WORKSPACE: return "MX_ERR_WORKSPACE: workspace missing or too small";
    case MX_ERR_ARCH: return "MX_ERR_ARCH: current device is not sm_100";
    case MX_ERR_CUDA: return "MX_ERR_CUDA: a CUDA call or kernel launch failed";
    case MX_ERR_TIMEOUT: return "MX_ERR_TIMEOUT: a kernel gave up on a bounded wait";
    }
    return "unknown mx_status";
}

mx_status mx_gemm_grouped(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                          const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out, int groups,
                          const int* offsets, int N, int K, void* workspace, size_t ws_bytes, void* stream)
{
    if (!offsets) return MX_ERR_NULL;
    if (groups < 1 || groups > kMaxGroups || offsets[0] != 0) return MX_ERR_SHAPE;
    for (int g = 0; g < groups; ++g)
        if (offsets[g + 1] < offsets[g]) return MX_ERR_SHAPE;
    const int M = offsets[groups];
    if (a_fmt != MX_A_E4M3_E8M0_1X32 && a_fmt != MX_A_E2M1_E8M0_1X32) return MX_ERR_FORMAT;
    if (epi == MX_EPI_SWIGLU_MXQ) return MX_ERR_FORMAT;
    // shapes and formats as mx_gemm (one row stands in when every group is empty)
    mx_status s = validate_gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M > 0 ? M : 1, N,
                                K);
    if (s != MX_OK) return s;
    if (static_cast<long long>(groups) * N > (1LL << 31) - 1) return MX_ERR_SHAPE;
    if (!workspace || ws_bytes < kWorkspaceBytes) return MX_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return MX_ERR_ALIGN;
    DeviceInfo dev;
    s = arch_ok(&dev);
    if (s != MX_OK) return s;
    if (M == 0) return MX_OK;  // no rows in any group: nothing to compute
    GemmProblem pb{a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K,
                   static_cast<unsigned*>(workspace), groups, offsets};
    GemmPlan plan;
    if (plan_gemm_grouped(pb, dev, &plan) != cudaSuccess) return MX_ERR_CUDA;
    return from_cuda(launch_gemm(pb, plan, static_cast<cudaStream_t>(stream)));
}

mx_status mx_quant_act(const void* x, int M, int K, void* codes, void* scales, mx_a_fmt fmt, void* stream)
{
    if (!x || !codes || !scales) return MX_ERR_NULL;
    if (fmt != MX_A_E4M3_E8M0_1X32 && fmt != MX_A_E4M3_F32_ROW && fmt != MX_A_E2M1_E8M0_1X32) return MX_ERR_FORMAT;
    if (M < 1 || K < 32 || (K % 32) != 0) return MX_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, fmt == MX_A_E4M3_F32_ROW ? 4 : 1))
        return MX_ERR_ALIGN;
    DeviceInfo dev;
    mx_status s = arch_ok(&dev);
    if (s != MX_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fmt == MX_A_E4M3_E8M0_1X32)
        return from_cuda(launch_quant_e8m0_1x32(x, M, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), st));
    if (fmt == MX_A_E2M1_E8M0_1X32)  // the 1 x 32 e2m1 rule of the weights, on rows of activations
        return from_cuda(launch_quant_w_e2m1_1x32(x, M, K, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), st));
    return from_cuda(launch_quant_f32_row(x, M, K, static_cast<uint8_t*>(codes), static_cast<float*>(scales), st));
}

mx_status mx_add_rms_quant(const void* x, void* residual, const void* w, float eps, int M, int K, void* y_out,
                           void* codes, void* scales, void* stream)
{
    if (!x || !residual || !w || !codes || !scales) return MX_ERR_NULL;
    if (M < 1 || K < 32 || (K % 32) != 0 || K > 16384 || !(eps >= 0.f)) return MX_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(residual, 16) || !aligned(w, 16) || !aligned(codes, 16) ||
        (y_out && !aligned(y_out, 16)))
        return MX_ERR_ALIGN;
    DeviceInfo dev;
    mx_status s = arch_ok(&dev);
    if (s != MX_OK) return s;
    return from_cuda(launch_add_rms_quant(x, residual, w, eps, M, K, y_out, codes, scales,
                                          static_cast<cudaStream_t>(stream)));
}

mx_status mx_quant_weight(const void* w, int N, int K, void* codes, void* scales, mx_b_fmt fmt, void* stream)
{
    if (!w || !codes || !scales) return MX_ERR_NULL;
    if (fmt != MX_B_E4M3_E8M0_32X32 && fmt != MX_B_E2M1_E8M0_1X32 && fmt != MX_B_E4M3_F32_ROW)
        return MX_ERR_FORMAT;
    if (N < 1 || K < 32 || (K % 32) != 0) return MX_ERR_SHAPE;
    if (fmt == MX_B_E4M3_E8M0_32X32 && (N % 32) != 0) return MX_ERR_SHAPE;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, fmt == MX_B_E4M3_F32_ROW ? 4 : 1))
        return MX_ERR_ALIGN;
    DeviceInfo dev;
    mx_status s = arch_ok(&dev);
    if (s != MX_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* c8 = static_cast<uint8_t*>(codes);
    switch (fmt) {
    case MX_B_E4M3_E8M0_32X32:
        return from_cuda(launch_quant_w_e4m3_32x32(w, N, K, c8, static_cast<uint8_t*>(scales), st));
    case MX_B_E2M1_E8M0_1X32:
        return from_cuda(launch_quant_w_e2m1_1x32(w, N, K, c8, static_cast<uint8_t*>(scales), st));
    default:
        return from_cuda(launch_quant_f32_row(w, N, K, c8, static_cast<float*>(scales), st));
    }
}

size_t mx_gemm_workspace_size(int M, int N, int K, mx_a_fmt a_fmt, mx_b_fmt b_fmt, mx_epi epi)
{
    if (M < 1 || N < 1 || K < 32) return kWorkspaceBytes;
    DeviceInfo dev;
    if (current_device(&dev) != cudaSuccess || dev.major != 10 || dev.minor != 0) {
        cudaGetLastError();
        return kWorkspaceBytes;  // no usable device: the minimum (plans are per device)
    }
    GemmProblem pb{};
    pb.a_fmt = a_fmt;
    pb.b_fmt = b_fmt;
    pb.epi = epi;
    pb.M = M;
    pb.N = N;
    pb.K = K;
    GemmPlan plan;
    if (plan_gemm(pb, dev, static_cast<size_t>(-1), &plan) != cudaSuccess) return kWorkspaceBytes;
    return std::max(plan.ws_bytes, kWorkspaceBytes);
}

mx_status mx_gemm(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                  const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out, int M, int N,
                  int K, void* workspace, size_t ws_bytes, void* stream)
{
    mx_status s = validate_gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K);
    if (s != MX_OK) return s;
    if (!workspace || ws_bytes < kWorkspaceBytes) return MX_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return MX_ERR_ALIGN;
    DeviceInfo dev;
    s = arch_ok(&dev);
    if (s != MX_OK) return s;
    GemmProblem pb{a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K,
                   static_cast<unsigned*>(workspace)};
    GemmPlan plan;
    if (plan_gemm(pb, dev, ws_bytes, &plan) != cudaSuccess) return MX_ERR_CUDA;
    if (plan.ws_bytes > ws_bytes) return MX_ERR_WORKSPACE;  // bf16 activations quantised ahead: no room
    return from_cuda(launch_gemm(pb, plan, static_cast<cudaStream_t>(stream)));
}

mx_status mx_gemm_plan(int M, int N, int K, mx_a_fmt a_fmt, mx_b_fmt b_fmt, mx_epi epi, int* block_n, int* splits,
                       int* grid, int* acc_bufs)
{
    if (!block_n || !splits || !grid || !acc_bufs) return MX_ERR_NULL;
    if (M < 1 || N < 1 || K < 32 || (K % 32) != 0) return MX_ERR_SHAPE;
    (void)b_fmt;
    DeviceInfo dev;
    mx_status s = arch_ok(&dev);
    if (s != MX_OK) return s;
    GemmProblem pb{};
    pb.a_fmt = a_fmt;
    pb.b_fmt = b_fmt;
    pb.epi = epi;
    pb.M = M;
    pb.N = N;
    pb.K = K;
    GemmPlan plan;
    if (plan_gemm(pb, dev, static_cast<size_t>(-1), &plan) != cudaSuccess) return MX_ERR_CUDA;
    *block_n = plan.block_n;
    *splits = plan.splits;
    *grid = plan.grid_x * plan.grid_y;
    *acc_bufs = plan.acc_bufs;
    return MX_OK;
}

void mx_set_tuning(int block_n, int splits, int max_ctas, int block_m)
{
    set_tuning(block_n, splits, max_ctas, block_m);
}

void mx_debug_set_timeline(void* buffer, size_t bytes) { set_timeline(buffer, bytes); }

void mx_set_launch_flags(unsigned flags)
{
    set_launch_flags(flags & (MX_LAUNCH_PDL | MX_LAUNCH_PREFETCH_WEIGHTS | MX_LAUNCH_DETERMINISTIC));
}

void mx_set_decode_tuning(int mode, int ctas, int ctas_per_sm, int prefetch_stages, int split, int cluster_size)
{
    set_decode_tuning(mode < 0 ? -1 : (mode > 0 ? 1 : 0), ctas < 0 ? 0 : ctas,
                      (ctas_per_sm == 1 || ctas_per_sm == 2) ? ctas_per_sm : 0,
                      prefetch_stages < 0 ? 0 : prefetch_stages, (split >= 0 && split <= 3) ? split : 0,
                      (cluster_size >= 2 && cluster_size <= 8) ? cluster_size : 0);
}

mx_status mx_gemm_plan_info(int M, int N, int K, mx_a_fmt a_fmt, mx_b_fmt b_fmt, mx_epi epi, size_t ws_bytes,
                            mx_plan_info* info)
{
    if (!info) return MX_ERR_NULL;
    if (M < 1 || N < 1 || K < 32 || (K % 32) != 0) return MX_ERR_SHAPE;
    DeviceInfo dev;
    mx_status s = arch_ok(&dev);
    if (s != MX_OK) return s;
    GemmProblem pb{};
    pb.a_fmt = a_fmt;
    pb.b_fmt = b_fmt;
    pb.epi = epi;
    pb.M = M;
    pb.N = N;
    pb.K = K;
    GemmPlan plan;
    if (plan_gemm(pb, dev, ws_bytes, &plan) != cudaSuccess) return MX_ERR_CUDA;
    memset(info, 0, sizeof(*info));
    info->kernel = plan.kernel;
    info->block_m = plan.block_m;
    info->block_n = plan.block_n;
    info->splits = plan.splits;
    if (plan.kernel == 1)
        info->k_reduction = plan.reduce ? 3 : (plan.cluster > 1 ? 1 : 0);
    else
        info->k_reduction = plan.splits > 1 ? (plan.gsplit ? 2 : 1) : 0;
    info->grid = plan.grid_x * plan.grid_y;
    info->acc_bufs = plan.acc_bufs;
    info->stages = plan.stages;
    info->tiles = plan.kernel != 0 ? plan.tiles : plan.units / std::max(1, plan.splits);
    info->ws_bytes = std::max(plan.ws_bytes, kWorkspaceBytes);
    info->ctas_per_sm = plan.kernel == 1 ? (plan.one_per_sm ? 1 : 2) : 1;
    info->act_quant = plan.act_quant;
    return MX_OK;
}

mx_status mx_workspace_status(void* workspace, void* stream)
{
    if (!workspace) return MX_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MX_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MX_ERR_CUDA;
    if (word == 0) return MX_OK;
    const unsigned zero = 0;
    if (cudaMemcpyAsync(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice, st) != cudaSuccess) return MX_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MX_ERR_CUDA;
    return MX_ERR_TIMEOUT;
}

mx_status mx_debug_watchdog(void* workspace, size_t ws_bytes, unsigned timeout_us, void* stream)
{
    if (!workspace) return MX_ERR_NULL;
    if (ws_bytes < kWorkspaceBytes) return MX_ERR_WORKSPACE;
    if (timeout_us == 0 || timeout_us > 10000000u) return MX_ERR_SHAPE;
    DeviceInfo dev;
    mx_status s = arch_ok(&dev);
    if (s != MX_OK) return s;
    return from_cuda(launch_watchdog_probe(static_cast<unsigned*>(workspace), timeout_us, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
