// static_scratch.cu -- lcx_attn_fwd_split_static: split-KV attention whose
// partial results live in a static device array of the library, so the call
// allocates nothing and needs no caller workspace.
//
// The array is one __device__ object per CUDA context (created when the
// library's module is loaded into that context).  Host code cannot use the
// array's name as a device address, so every call asks the runtime for the
// current context's copy with cudaGetSymbolAddress (checked).  That lookup
// allocates nothing once the module is loaded; resolving it on every call
// rather than caching it means a context that was destroyed and created
// again (cudaDeviceReset, a released and re-retained primary context) gets
// its own array's address, never a stale one.  Nothing in the array has to
// start at zero: every partial row the merge kernel reads is written by the
// attention kernel of the same call (a key split without tiles writes the
// empty result), so the array is never cleared.
#include <cuda_runtime.h>

#include "lcx_internal.h"

namespace lcx {
namespace {

constexpr int64_t kStaticScratchBytes = int64_t(LCX_STATIC_SCRATCH_BYTES);

__device__ __align__(256) unsigned char g_split_scratch[LCX_STATIC_SCRATCH_BYTES];

// The current context's copy of the scratch array.
lcx_status scratch_for_current_context(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_split_scratch);
    if (e != cudaSuccess || !p)
        return fail(LCX_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s",
                    cudaGetErrorString(e));
    *out = p;
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
    lcx_status st = scratch_for_current_context(&scratch);
    if (st != LCX_OK) return st;
    return lcx_attn_fwd_split(a, num_splits, scratch, kStaticScratchBytes, stream);
}
