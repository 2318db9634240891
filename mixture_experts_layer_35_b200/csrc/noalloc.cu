// noalloc.cu -- moe_fused_forward_noalloc: the fused forward for callers that cannot
// allocate device memory.
//
// Its scratch (what moe_fused_forward keeps in the caller's workspace: router logits,
// routing, permutation tables, h, the FP32 accumulator) lives in one file-scope
// device array of MOE_NOALLOC_SCRATCH_BYTES.  The array is part of this library's
// module, so every GPU that loads the library holds it until the process exits.
//
// Host code cannot use the array's name as a device address (in host code it names a
// host-side stand-in).  The first call on each device, with that device current, looks
// up the real device address with cudaGetSymbolAddress, clears the error word, and keeps
// the address for that device and CUDA context; later calls reuse it.  That first call
// should therefore happen before any stream capture starts.  A new primary context on
// the device (after cudaDeviceReset) reloads the module, so the address is looked up
// again when the current context changes.
//
// Every call on a device shares the one array, and it keeps the previous call's
// contents.  Nothing in it needs to start at zero on a call: the many-token path clears
// its own counters, and everything else is fully overwritten before it is read.  The
// device error word is the exception: it collects the MOE_DEVERR_* flags of every call
// until moe_noalloc_get_error reads and clears it, as moe_get_error does for a caller's
// workspace.  Calls whose work overlaps on the GPU (other streams, concurrent graphs)
// race on the array.
#include <mutex>

#include "kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};

// The current CUDA context (driver entry point resolved once through the runtime), used
// only as a key: a different value means the module, and with it the array, was reloaded.
typedef int (*CtxGetCurrentFn)(void**);
void* current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    void* ctx = nullptr;
    if (fn && fn(&ctx) != 0) ctx = nullptr;
    return ctx;
}

// Device address of the scratch array on the current device (set up once per device and
// context; the set-up clears the error word on `stream`).
cudaError_t scratch_address(void** out, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    void* ctx = current_context();
    if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(p, 0, moe::kHeaderBytes, stream);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_fused_forward_noalloc(const moe_layer_desc* d, const void* x, void* out,
                                                  float* topk_w_out, int32_t* topk_ids_out, float* logits_out,
                                                  void* stream) {
    const size_t need = moe_workspace_size(d);
    if (need == 0 || d->T == 0)  // invalid description (its status) or nothing to do
        return moe_fused_forward(d, x, out, topk_w_out, topk_ids_out, logits_out, nullptr, 0, stream);
    if (need > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
    void* ws = nullptr;
    if (scratch_address(&ws, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    return moe_fused_forward(d, x, out, topk_w_out, topk_ids_out, logits_out, ws, MOE_NOALLOC_SCRATCH_BYTES,
                             stream);
}

extern "C" moe_status_t moe_noalloc_get_error(int* code, void* stream) {
    if (!code) return MOE_ERR_INVALID_ARG;
    void* ws = nullptr;
    if (scratch_address(&ws, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    return moe_get_error(ws, code, stream);
}
