// lcx_internal.h -- declarations shared by the library's translation units
// (host validation helpers and the per-thread last-error string).
#pragma once
#include <cstdint>
#include <cstdio>
#include <string>

#include <cuda_runtime.h>

#include "../../include/lcx.h"

namespace lcx {

// Record `msg` as the calling thread's last error and return `st`.
lcx_status fail(lcx_status st, const char *fmt, ...);

// Clear the calling thread's last error.
void clear_error();

// Validate RoPE parameters (shared by every entry point).
lcx_status check_rope_params(const lcx_rope_params *p);

// Fill theta'_i (fp32, head_dim/2 entries) and mscale for validated params;
// seq_len is the actual context length the length-dependent modes use.
void rope_table_unchecked(const lcx_rope_params *p, int64_t seq_len, float *inv_freq,
                          float *mscale);

// The context length a call uses for the length-dependent modes.
inline int64_t effective_seq_len(const lcx_rope_params *p, int64_t call_len) {
    return p->seq_len > 0 ? p->seq_len : call_len;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The rotate pass of lcx_apply_rope (argument checks included).  With y_x8
// (bf16 x only, NULL = none) it writes the split-QK^T key parts instead: y the
// fp16 parts h = f16(y'), and y_x8, a row of 2 D bytes per (b, h, l) starting at
// twice y's element offset, the e5m2 bytes of y' - h then those of h.
lcx_status apply_rope_impl(const lcx_rope_params *params, const void *x, void *y, void *y_x8,
                           int32_t dtype, int64_t B, int64_t H, int64_t L,
                           const int64_t *x_strides, const int64_t *y_strides, int64_t pos_offset,
                           cudaStream_t stream);

// Contiguous fp16 copy of a bf16 [B, H, L, D] tensor (element strides, the last
// one 1), values converted exactly where fp16 holds them (the split mode's V).
lcx_status bf16_to_f16_impl(const void *x, const int64_t *x_strides, void *y, int64_t B,
                            int64_t H, int64_t L, int64_t D, cudaStream_t stream);

// Enqueue the merge of n_parts partial results ([n_parts, B, Hq, L, D] fp32 o,
// [n_parts, B, Hq, L] fp32 lse) into o (dtype, strides) and optionally lse.
// Arguments are assumed valid.
lcx_status launch_merge(const float *o_parts, const float *lse_parts, int n_parts, int64_t B,
                        int64_t Hq, int64_t L, int64_t D, void *o, int32_t dtype,
                        const int64_t *o_strides, float *lse_out, cudaStream_t stream);

}  // namespace lcx
