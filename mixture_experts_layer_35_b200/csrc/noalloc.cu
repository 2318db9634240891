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
// up the real device address with cudaGetSymbolAddress and keeps it for that device;
// later calls reuse it.  That first call should therefore happen before any stream
// capture starts.
//
// Every call on a device shares the one array, and it keeps the previous call's
// contents.  The entry point clears the part that must start at zero (the error word)
// at the start of every call; everything else is fully overwritten before it is read.
// Calls whose work overlaps on the GPU (other streams, concurrent graphs) race on the
// array.
#include <mutex>

#include "kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
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
    if (scratch_address(&ws) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, moe::kHeaderBytes, (cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
    return moe_fused_forward(d, x, out, topk_w_out, topk_ids_out, logits_out, ws, MOE_NOALLOC_SCRATCH_BYTES,
                             stream);
}
