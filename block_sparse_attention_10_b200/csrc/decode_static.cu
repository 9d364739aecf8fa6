// decode_static.cu — msa_decode_static: the decode step with its scratch in a
// fixed device array that the library owns, for callers that cannot allocate.
//
// msa_decode needs caller scratch for the pooled block scores and the
// selected block ids between its kernels.  Some callers cannot provide it: a
// plugin inside a host framework whose allocator owns all device memory and
// that is handed only its inputs and outputs, or a latency-critical loop that
// must not call cudaMalloc (which can synchronise the whole device).  For
// them the scratch lives in g_msa_static_scratch below, a file-scope device
// array of MSA_STATIC_SCRATCH_BYTES that every GPU loading the library holds
// until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// is only a stand-in symbol), so the address is looked up once per device with
// cudaGetSymbolAddress, with that device current, and cached.  The lookup
// happens in the first call on each device; with lazy module loading (the CUDA
// default) that first call is also when the driver loads this file's module and
// places the array in device memory, so it is the warm-up call and belongs
// before any stream capture.  The cache is keyed by the context's unique id:
// after cudaDeviceReset the next call sees a new context and looks the address
// up again instead of reusing one from the destroyed context.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace msa {
namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_msa_static_scratch[MSA_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

// Unique id (never reused within the process) of the calling thread's current context, or 0.
unsigned long long current_context_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_msa_static_scratch on the current device, looked up once per
// device (again after a device reset, which gives the device a new context).
int static_scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return MSA_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    const unsigned long long ctx = current_context_id();
    if (g_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_msa_static_scratch) != cudaSuccess || ptr == nullptr) return MSA_ECUDA;
        g_scratch_addr[dev] = ptr;
        // the lookup made the device's context current if it was not yet
        g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
    }
    *out = g_scratch_addr[dev];
    return MSA_OK;
}

}  // namespace
}  // namespace msa

extern "C" int msa_decode_static(const msa_params_t* p, void* out, float* lse, int32_t* sel_out,
                                 cudaStream_t stream) {
    // Argument checks of msa_decode: with no workspace it validates everything else
    // and returns MSA_EWORKSPACE without enqueueing any work.
    const int r = msa_decode(p, nullptr, 0, out, lse, sel_out, stream);
    if (r != MSA_EWORKSPACE) return r;
    const size_t need = msa_workspace_size(p);
    if (need == 0 || need > MSA_STATIC_SCRATCH_BYTES) return MSA_EWORKSPACE;
    void* scratch = nullptr;
    if (const int e = msa::static_scratch_address(&scratch)) return e;
    // The kernels overwrite every scratch entry they read (all block scores and
    // all 16 selection slots per query), so nothing has to be cleared first.
    return msa_decode(p, scratch, MSA_STATIC_SCRATCH_BYTES, out, lse, sel_out, stream);
}
