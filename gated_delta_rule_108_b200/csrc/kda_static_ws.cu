// kda_static_ws.cu -- kda_chunk_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin whose host framework owns all
// device memory through its own pool and forbids other allocations, a
// latency-critical loop that cannot afford cudaMalloc's implicit device-wide
// synchronisation, or a tool that runs within a fixed, pre-reserved memory
// budget.  For them, kda_chunk_fwd_static takes the scratch space that
// kda_chunk_fwd needs from a fixed array that lives in this library's device
// image, so nothing is allocated per call.
//
// The array is KDA_STATIC_WORKSPACE_BYTES long; every GPU that loads the
// library holds it until the process exits.  In host code the name
// g_static_workspace is only a stand-in for the device array, never a device
// address, so the address is looked up with cudaGetSymbolAddress on the first
// call on each device (with that device current) and cached together with the
// CUDA context it belongs to.  If that context has been torn down since (e.g.
// cudaDeviceReset), the module is loaded again at another address, so a call
// that finds a different current context repeats the look-up.  All calls share
// the array; kda_chunk_fwd rewrites every part of it that it reads (its status
// word and chunk table are set by its first kernel, its per-chunk records are
// written before they are read), so stale contents from an earlier call do
// not matter -- but calls that overlap on the GPU (different streams or
// devices' threads racing on one device) race on it.
#include <cuda.h>

#include <mutex>

#include "../../include/kda.h"
#include "kda_launch.h"

namespace {

static __device__ __align__(256) unsigned char g_static_workspace[KDA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_dev_ptr[kMaxDevices] = {};
CUcontext g_dev_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, reached through the runtime (the library links
// only the CUDA runtime).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of g_static_workspace on the current device: set up on the
// first call per device (with that device current), again if the device's
// context has changed since.
cudaError_t static_workspace_ptr(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return cudaErrorUnknown;
    // null until this host thread's first runtime call that binds the context
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ptr[dev] || !ctx || g_dev_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);   // binds the device's context
        if (e != cudaSuccess) return e;
        if (get(&ctx) != CUDA_SUCCESS) return cudaErrorUnknown;
        g_dev_ptr[dev] = p;
        g_dev_ctx[dev] = ctx;
    }
    *out = g_dev_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_static(const void* q, const void* k, const void* v,
                                           const float* log_alpha, const float* beta,
                                           const float* initial_state, const int32_t* cu_seqlens,
                                           int B, int T, int H, int dk, int dv, int num_seqs,
                                           kda_dtype dtype, void* o, float* final_state,
                                           void* stream) {
    const size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, num_seqs,
                                                     cu_seqlens != nullptr, dtype);
    if (need > (size_t)KDA_STATIC_WORKSPACE_BYTES)
        return (kda_status)kda::set_error(KDA_ERR_WORKSPACE,
                              "kda_chunk_fwd_static: these sizes need %zu bytes of workspace but the "
                              "static workspace holds %zu; call kda_chunk_fwd with a caller-owned "
                              "workspace instead", need, (size_t)KDA_STATIC_WORKSPACE_BYTES);
    void* ws = nullptr;
    const cudaError_t e = static_workspace_ptr(&ws);
    if (e != cudaSuccess)
        return (kda_status)kda::set_error(KDA_ERR_CUDA, "kda_chunk_fwd_static: cudaGetSymbolAddress failed: %s",
                              cudaGetErrorString(e));
    return kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state, cu_seqlens, B, T, H, dk, dv,
                         num_seqs, dtype, o, final_state, ws, KDA_STATIC_WORKSPACE_BYTES, stream);
}
