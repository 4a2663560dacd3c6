// static_scratch.cu -- lcx_attn_fwd_split_static: split-KV attention whose
// partial results live in a static device array of the library, so the call
// allocates nothing and needs no caller workspace.
//
// The array is one __device__ object per device (created when the library's
// module is loaded into that device's context).  Its address is resolved once
// per device with cudaGetSymbolAddress and cached.  Nothing in it has to start
// at zero: every partial row the merge kernel reads is written by the
// attention kernel of the same call (a key split without tiles writes the
// empty result), so the array is never cleared.
#include <cuda_runtime.h>

#include <mutex>

#include "lcx_internal.h"

namespace lcx {
namespace {

constexpr int64_t kStaticScratchBytes = int64_t(LCX_STATIC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_split_scratch[LCX_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// The calling thread's current device's copy of the scratch array.
lcx_status scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(LCX_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return fail(LCX_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_split_scratch);
        if (e != cudaSuccess || !p)
            return fail(LCX_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s",
                        cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LCX_OK;
}

}  // namespace
}  // namespace lcx

extern "C" lcx_status lcx_attn_fwd_split_static(const lcx_attn_args *a, int32_t num_splits,
                                                void *stream) {
    using namespace lcx;
    clear_error();
    if (!a) return fail(LCX_ERR_INVALID_ARG, "args is NULL");
    if (num_splits == 1) return lcx_attn_fwd_split(a, 1, nullptr, 0, stream);
    const int64_t dv = a->Dv > 0 ? a->Dv : a->D;   // the partial outputs' head dim
    const int64_t need = lcx_attn_split_workspace_bytes(a->B, a->Hq, a->L, dv, num_splits);
    if (need < 0)
        return fail(LCX_ERR_INVALID_ARG, "invalid sizes or num_splits for split-KV attention");
    if (need > kStaticScratchBytes)
        return fail(LCX_ERR_UNSUPPORTED,
                    "split-KV needs %lld bytes of scratch; the static array holds %lld",
                    (long long)need, (long long)kStaticScratchBytes);
    if (need == 0) return lcx_attn_fwd_split(a, num_splits, nullptr, 0, stream);
    void *scratch = nullptr;
    lcx_status st = scratch_for_current_device(&scratch);
    if (st != LCX_OK) return st;
    return lcx_attn_fwd_split(a, num_splits, scratch, kStaticScratchBytes, stream);
}
