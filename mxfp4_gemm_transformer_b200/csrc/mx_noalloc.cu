// mx_noalloc.cu -- mx_gemm for callers that cannot allocate device memory.
//
// mx_gemm needs a small caller-owned workspace (the status word its bounded
// waits report into).  Some callers have no way to provide one: runtimes that
// hand kernels a fixed memory arena and forbid hidden allocations, and plain-C
// plugin hosts that expose no device allocator at all.  mx_gemm_noalloc serves them: it takes the same
// inputs and outputs and uses a scratch array that lives in the library
// itself, so the call allocates nothing.
#include <cuda.h>

#include <cstdint>
#include <mutex>

#include "mx_internal.h"

namespace mxg {
namespace {

// The scratch every mx_gemm_noalloc call on a device shares.  Every GPU that
// loads the library holds these bytes until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MX_NOALLOC_SCRATCH_BYTES];

// Identity of the current context: its unique id where the driver has
// cuCtxGetId (a destroyed and recreated context gets a new one, even at the
// same address), else the context handle; 0 when neither can be read.
unsigned long long context_identity()
{
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (get_id && get_id(ctx, &id) == CUDA_SUCCESS) return id;
    return static_cast<unsigned long long>(reinterpret_cast<uintptr_t>(ctx));
}

// Device address of g_noalloc_scratch, resolved with the device current (in
// host code the symbol's name is only a host-side stand-in, never a device
// address) and cached per device together with the context it belongs to: a
// device reset, or a new primary context, loads the module again and may move
// the array, so a changed context is looked up afresh.
cudaError_t scratch_address(void** out)
{
    static std::mutex mu;
    static void* addr[64] = {};
    static unsigned long long owner[64] = {};
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const unsigned long long ctx = context_identity();
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev] || ctx == 0 || owner[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
        owner[dev] = ctx;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace mxg

using namespace mxg;

extern "C" mx_status mx_gemm_noalloc(const void* a_codes, const void* a_scales, mx_a_fmt a_fmt, const void* b_codes,
                                     const void* b_scales, mx_b_fmt b_fmt, const float* bias, mx_epi epi, void* out,
                                     int M, int N, int K, void* stream)
{
    mx_status s = validate_gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K);
    if (s != MX_OK) return s;
    DeviceInfo dev;
    if (current_device(&dev) != cudaSuccess) return MX_ERR_CUDA;
    if (dev.major != 10 || dev.minor != 0) return MX_ERR_ARCH;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MX_ERR_CUDA;
    GemmProblem pb{a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K,
                   static_cast<unsigned*>(scratch)};
    GemmPlan plan;
    // The scratch is shared by every call on the device, whatever the stream,
    // so only its status word is used: plans that keep split-K partials and
    // arrival counters in the workspace are excluded (they would collide
    // between concurrent calls); K splits go through a cluster instead.
    if (plan_gemm(pb, dev, kWorkspaceHeader, &plan) != cudaSuccess) return MX_ERR_CUDA;
    // bf16 activations outside the decode kernel would be quantised into the
    // shared scratch, which concurrent calls would overwrite
    if (plan.ws_bytes > MX_NOALLOC_SCRATCH_BYTES || plan.act_quant == 2) return MX_ERR_WORKSPACE;
    return launch_gemm(pb, plan, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}
