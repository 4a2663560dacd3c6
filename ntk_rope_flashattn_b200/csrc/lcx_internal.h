// lcx_internal.h -- declarations shared by the library's translation units
// (host validation helpers and the per-thread last-error string).
#pragma once
#include <cstdint>
#include <cstdio>
#include <string>

#include "../../include/lcx.h"

namespace lcx {

// Record `msg` as the calling thread's last error and return `st`.
lcx_status fail(lcx_status st, const char *fmt, ...);

// Clear the calling thread's last error.
void clear_error();

// Validate RoPE parameters (shared by every entry point).
lcx_status check_rope_params(const lcx_rope_params *p);

// Fill theta'_i (fp32, head_dim/2 entries) and mscale for validated params.
void rope_table_unchecked(const lcx_rope_params *p, float *inv_freq, float *mscale);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace lcx
