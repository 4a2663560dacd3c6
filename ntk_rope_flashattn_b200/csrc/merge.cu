// merge.cu -- combine partial attention results over disjoint key sets
// (lcx_attn_merge; the second pass of split-KV attention).
//
// "8.3 长上下文技术", sections 8.3.4 (online softmax: partial sums are rescaled
// by their running maxima) and 8.3.5 (Ring Attention, step 3: each KV block's
// partial output is folded in by the online-softmax rescaling).  Part s of a
// query row holds o_s (normalised over its own keys) and lse_s = ln Z_s; with
// m = max_s lse_s and w_s = e^(lse_s - m):
//   o = sum_s w_s o_s / sum_s w_s,   lse = m + ln sum_s w_s.
// Empty parts (lse_s = -inf) weigh nothing; a row with only empty parts gets
// o = 0, lse = -inf.
//
// HBM-bound: one warp per query row reads the n parts' D fp32 values (each
// lane a 16- or 8-byte slice, so a warp reads whole 512/256-byte rows) and the
// n part LSEs (one broadcast load each), and writes D output values once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "lcx_internal.h"

namespace lcx {
namespace {

constexpr int kMergeWarps = 8;  // rows per 256-thread block

template <int D, bool kF32>
__global__ void __launch_bounds__(kMergeWarps * 32)
    merge_kernel(const float *__restrict__ o_parts, const float *__restrict__ lse_parts,
                 int n_parts, long long rows, int Hq, int L, void *o, long long os0,
                 long long os1, long long os2, float *lse_out) {
    // Launched as a programmatic dependent of the attention kernel that writes
    // the parts: wait here until that grid has completed and its writes are
    // visible (a plain launch passes straight through).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    constexpr int V = D / 32;  // values per lane: 4 (D=128) or 2 (D=64)
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    float m = -INFINITY;
    for (int s = lane; s < n_parts; s += 32) m = fmaxf(m, lse_parts[(long long)s * rows + row]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    float z = 0.f;  // this lane's parts' weights
    if (m != -INFINITY) {
        // 32 parts at a time: lane u computes the weight of part s0 + u (0 for
        // an empty part), the warp takes it by shuffle; the parts' rows have no
        // dependence on one another, so eight of them are loaded at once.
        for (int s0 = 0; s0 < n_parts; s0 += 32) {
            const int s = s0 + lane;
            const float l = s < n_parts ? lse_parts[(long long)s * rows + row] : -INFINITY;
            const float wl = l == -INFINITY ? 0.f : expf(l - m);
            z += wl;
            const int nu = min(32, n_parts - s0);
#pragma unroll 8
            for (int u = 0; u < nu; ++u) {
                const float w = __shfl_sync(0xffffffffu, wl, u);
                const float *src = o_parts + ((long long)(s0 + u) * rows + row) * D + lane * V;
                if constexpr (V == 4) {
                    float4 x = __ldcs(reinterpret_cast<const float4 *>(src));
                    if (w == 0.f) x = make_float4(0.f, 0.f, 0.f, 0.f);
                    acc[0] += w * x.x;
                    acc[1] += w * x.y;
                    acc[2] += w * x.z;
                    acc[3] += w * x.w;
                } else {
                    float2 x = __ldcs(reinterpret_cast<const float2 *>(src));
                    if (w == 0.f) x = make_float2(0.f, 0.f);
                    acc[0] += w * x.x;
                    acc[1] += w * x.y;
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    const long long h_all = row / L;                  // b * Hq + h
    const long long b = h_all / Hq, h = h_all % Hq, i = row % L;
    const long long ob = b * os0 + h * os1 + i * os2 + lane * V;
    if constexpr (kF32) {
        float *dst = reinterpret_cast<float *>(o) + ob;
#pragma unroll
        for (int e = 0; e < V; ++e) dst[e] = acc[e] * inv;
    } else {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(o) + ob;
#pragma unroll
        for (int e = 0; e < V; e += 2)
            *reinterpret_cast<__nv_bfloat162 *>(dst + e) =
                __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
    }
    if (lse_out && lane == 0) lse_out[row] = z > 0.f ? m + logf(z) : -INFINITY;
}

}  // namespace

lcx_status launch_merge(const float *o_parts, const float *lse_parts, int n_parts, int64_t B,
                        int64_t Hq, int64_t L, int64_t D, void *o, int32_t dtype,
                        const int64_t *o_strides, float *lse_out, cudaStream_t stream) {
    const long long rows = (long long)B * Hq * L;
    if (rows == 0) return LCX_OK;
    const long long blocks = (rows + kMergeWarps - 1) / kMergeWarps;
    if (blocks > 0x7fffffffLL) return fail(LCX_ERR_UNSUPPORTED, "too many rows to merge");
    // A programmatic dependent launch: the grid may be scheduled while the
    // attention kernel that writes the parts finishes (the kernel waits for
    // it), which hides this launch's latency behind that kernel's tail.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(blocks));
    cfg.blockDim = dim3(unsigned(kMergeWarps * 32));
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const bool f32 = dtype == LCX_F32;
    const long long s0 = o_strides[0], s1 = o_strides[1], s2 = o_strides[2];
    const int hq = int(Hq), l = int(L);
    cudaError_t le;
    if (D == 128)
        le = f32 ? cudaLaunchKernelEx(&cfg, merge_kernel<128, true>, o_parts, lse_parts, n_parts,
                                      rows, hq, l, o, s0, s1, s2, lse_out)
                 : cudaLaunchKernelEx(&cfg, merge_kernel<128, false>, o_parts, lse_parts, n_parts,
                                      rows, hq, l, o, s0, s1, s2, lse_out);
    else
        le = f32 ? cudaLaunchKernelEx(&cfg, merge_kernel<64, true>, o_parts, lse_parts, n_parts,
                                      rows, hq, l, o, s0, s1, s2, lse_out)
                 : cudaLaunchKernelEx(&cfg, merge_kernel<64, false>, o_parts, lse_parts, n_parts,
                                      rows, hq, l, o, s0, s1, s2, lse_out);
    if (le != cudaSuccess)
        return fail(LCX_ERR_CUDA, "merge launch failed: %s", cudaGetErrorString(le));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "merge launch failed: %s", cudaGetErrorString(e));
    return LCX_OK;
}

}  // namespace lcx

extern "C" lcx_status lcx_attn_merge(const float *o_parts, const float *lse_parts,
                                     int32_t n_parts, int64_t B, int64_t Hq, int64_t L,
                                     int64_t D, void *o, int32_t dtype,
                                     const int64_t *o_strides, float *lse, void *stream) {
    using namespace lcx;
    clear_error();
    if (n_parts < 1 || n_parts > 4096) return fail(LCX_ERR_INVALID_ARG, "n_parts must be in [1, 4096]");
    if (B < 0 || Hq <= 0 || L < 0) return fail(LCX_ERR_INVALID_ARG, "bad sizes");
    if (dtype != LCX_BF16 && dtype != LCX_F32) return fail(LCX_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (D != 64 && D != 128) return fail(LCX_ERR_UNSUPPORTED, "head_dim %lld: only 64 and 128", (long long)D);
    if (!o_strides) return fail(LCX_ERR_INVALID_ARG, "o_strides is NULL");
    if (B == 0 || L == 0) return LCX_OK;
    if (L > (int64_t(1) << 30) || Hq > 65536 || B * Hq * L > (int64_t(1) << 40))
        return fail(LCX_ERR_UNSUPPORTED, "sizes too large");
    if (!o_parts || !lse_parts || !o) return fail(LCX_ERR_INVALID_ARG, "NULL buffer");
    if (!aligned16(o_parts)) return fail(LCX_ERR_UNSUPPORTED, "o_parts must be 16-byte aligned");
    if (!aligned16(o)) return fail(LCX_ERR_UNSUPPORTED, "o must be 16-byte aligned");
    const int es = dtype == LCX_BF16 ? 2 : 4;
    if (o_strides[3] != 1) return fail(LCX_ERR_UNSUPPORTED, "o: head_dim stride must be 1");
    for (int d = 0; d < 3; ++d)
        if (o_strides[d] < 0 || (o_strides[d] * es) % 16 != 0)
            return fail(LCX_ERR_UNSUPPORTED, "o: strides must be non-negative multiples of 16 bytes");
    return launch_merge(o_parts, lse_parts, n_parts, B, Hq, L, D, o, dtype, o_strides, lse,
                        static_cast<cudaStream_t>(stream));
}
