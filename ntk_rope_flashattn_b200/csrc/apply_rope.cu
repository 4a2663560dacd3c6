// apply_rope.cu -- the memory-bound rotate-pairs pass (lcx_apply_rope).
//
// y_p = ms (x_p cos phi - x_q sin phi), y_q = ms (x_p sin phi + x_q cos phi),
// phi = m theta'_i, m = pos_offset + l ("Long Context: RoPE / YaRN / NTK /
// MLA", sections 2.2 and 2.4 apply_rope; 6.4 for ms folded into cos/sin).
//
// Layout of the work: a CTA owns a run of positions of one batch entry and
// walks every head of that run.  Each thread owns one 16-byte vector of pairs
// at one position: it evaluates the cos/sin of its pairs once (fp64 angle +
// range reduction + libm sincosf) and reuses them across all H heads, so the
// trigonometry costs 1/H of a pass and the kernel streams HBM with 128-bit
// loads and stores.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "lcx_internal.h"
#include "rope_angle.cuh"

namespace lcx {
namespace {

constexpr int kMaxHalf = 256;  // head_dim <= 512

struct RopeArgs {
    const char *x;
    char *y;
    char *y_x8;                  // bf16 x only, or NULL: y then receives the fp16 parts
                                 // h = f16(y') and y_x8 the 8-bit cross parts (below)
    long long xs_b, xs_h, xs_l;  // element strides
    long long ys_b, ys_h, ys_l;
    int H, L;
    long long pos_offset;
    int D;                // head_dim
    int jobs_per_row;     // 16-byte jobs per (position, head)
    int rows_per_cta;     // positions per CTA
    float ms;
    float theta[kMaxHalf];
};

template <typename T>
struct Vec;  // 16 bytes of T as 32-bit words
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;  // elements per 16 bytes
};
template <>
struct Vec<float> {
    static constexpr int N = 4;
};

__device__ __forceinline__ void unpack(const uint4 &v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        x[2 * k] = __uint_as_float(w[k] << 16);
        x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void unpack(const uint4 &v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ uint32_t pk(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint4 pack(const float (&y)[8]) {
    return make_uint4(pk(y[0], y[1]), pk(y[2], y[3]), pk(y[4], y[5]), pk(y[6], y[7]));
}
__device__ __forceinline__ uint4 pack(const float (&y)[4]) {
    return make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                      __float_as_uint(y[3]));
}

__device__ __forceinline__ uint32_t pk16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float2 unpk16(uint32_t v) {
    float lo, hi;
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(v));
    return make_float2(lo, hi);
}
__device__ __forceinline__ uint32_t pk8x4(float x0, float x1, float x2, float x3) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
    return uint32_t(lo) | (uint32_t(hi) << 16);
}

// Split-QK^T keys: the 8 rotated values y of the vector at element e of a row
// are stored as fp16 parts h = f16(y) (16 bytes at y's place, which is fp16
// here) and, in the 8-bit cross row of 2 D bytes, the e5m2 bytes of the
// residual y - h at bytes e .. e + 7 and of h at bytes D + e .. D + e + 7 (the
// key order [r8 | h8] the attention kernel's cross product expects).  The
// cross row of (b, h, l) starts at twice the element offset of y's row.
__device__ __forceinline__ void store_split(const RopeArgs &a, int b, int l, int h, int e,
                                            const float (&y)[8]) {
    const long long row = b * a.ys_b + l * a.ys_l + (long long)h * a.ys_h;
    const uint4 hv = make_uint4(pk16(y[0], y[1]), pk16(y[2], y[3]), pk16(y[4], y[5]),
                                pk16(y[6], y[7]));
    __stcs(reinterpret_cast<uint4 *>(a.y + 2 * (row + e)), hv);
    const uint32_t w[4] = {hv.x, hv.y, hv.z, hv.w};
    float hf[8], r[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = unpk16(w[k]);
        hf[2 * k] = f.x;
        hf[2 * k + 1] = f.y;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) r[k] = y[k] - hf[k];   // exact in fp32
    char *x8 = a.y_x8 + 2 * row;
    __stcs(reinterpret_cast<uint2 *>(x8 + e),
           make_uint2(pk8x4(r[0], r[1], r[2], r[3]), pk8x4(r[4], r[5], r[6], r[7])));
    __stcs(reinterpret_cast<uint2 *>(x8 + a.D + e),
           make_uint2(pk8x4(hf[0], hf[1], hf[2], hf[3]), pk8x4(hf[4], hf[5], hf[6], hf[7])));
}

// HALF pairing: a job covers N consecutive pairs i0..i0+N-1, i.e. the vector
// at element i0 and the vector at element i0 + D/2.  kX8: write the split
// mode's fp16 and 8-bit cross parts instead of y in x's type (bf16 x only).
template <typename T, bool kHalf, bool kX8>
__global__ void __launch_bounds__(256) apply_rope_kernel(const __grid_constant__ RopeArgs a) {
    constexpr int N = Vec<T>::N;
    constexpr int P = kHalf ? N : N / 2;  // pairs per job
    const int job = threadIdx.x % a.jobs_per_row;
    const int slot = threadIdx.x / a.jobs_per_row;
    const int l = blockIdx.x * a.rows_per_cta + slot;
    const int b = blockIdx.y;
    if (slot >= a.rows_per_cta || l >= a.L) return;

    const int i0 = job * P;                         // first pair of the job
    const long long m = a.pos_offset + l;
    float c[P], s[P];
#pragma unroll
    for (int e = 0; e < P; ++e) {
        rope_sincos(m, a.theta[i0 + e], &c[e], &s[e]);
        c[e] *= a.ms;
        s[e] *= a.ms;
    }
    // element offsets of the job's vectors within a row
    const int half_d = a.jobs_per_row * (kHalf ? N : N / 2);  // D/2
    const int e1 = kHalf ? i0 : 2 * i0;
    const int e2 = kHalf ? i0 + half_d : 0;

    const char *xb = a.x + sizeof(T) * (b * a.xs_b + l * a.xs_l);
    char *yb = a.y + sizeof(T) * (b * a.ys_b + l * a.ys_l);

    // Heads are processed in batches of kHB: every load of a batch is issued
    // before any store, so a thread keeps 2 kHB 16-byte loads in flight (the
    // in-place case forbids the compiler from doing this reordering itself).
    constexpr int kHB = 4;
    for (int h0 = 0; h0 < a.H; h0 += kHB) {
        uint4 va[kHB], vb[kHB];
#pragma unroll
        for (int u = 0; u < kHB; ++u) {
            if (h0 + u < a.H) {
                const T *xr = reinterpret_cast<const T *>(xb + sizeof(T) * ((h0 + u) * a.xs_h));
                va[u] = __ldcs(reinterpret_cast<const uint4 *>(xr + e1));
                if (kHalf) vb[u] = __ldcs(reinterpret_cast<const uint4 *>(xr + e2));
            }
        }
#pragma unroll
        for (int u = 0; u < kHB; ++u) {
            if (h0 + u >= a.H) break;
            T *yr = reinterpret_cast<T *>(yb + sizeof(T) * ((h0 + u) * a.ys_h));
            if (kHalf) {
                float x1[N], x2[N], y1[N], y2[N];
                unpack(va[u], x1);
                unpack(vb[u], x2);
#pragma unroll
                for (int e = 0; e < N; ++e) {
                    y1[e] = fmaf(x1[e], c[e], -x2[e] * s[e]);
                    y2[e] = fmaf(x1[e], s[e], x2[e] * c[e]);
                }
                if constexpr (sizeof(T) == 2 && kX8) {
                    store_split(a, b, l, h0 + u, e1, y1);
                    store_split(a, b, l, h0 + u, e2, y2);
                } else {
                    __stcs(reinterpret_cast<uint4 *>(yr + e1), pack(y1));
                    __stcs(reinterpret_cast<uint4 *>(yr + e2), pack(y2));
                }
            } else {
                float x[N], y[N];
                unpack(va[u], x);
#pragma unroll
                for (int e = 0; e < P; ++e) {
                    y[2 * e] = fmaf(x[2 * e], c[e], -x[2 * e + 1] * s[e]);
                    y[2 * e + 1] = fmaf(x[2 * e], s[e], x[2 * e + 1] * c[e]);
                }
                if constexpr (sizeof(T) == 2 && kX8) {
                    float y8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y8[e] = y[e];
                    store_split(a, b, l, h0 + u, e1, y8);
                } else {
                    __stcs(reinterpret_cast<uint4 *>(yr + e1), pack(y));
                }
            }
        }
    }
}

// bf16 [B, H, L, D] (element strides, last one 1) -> contiguous fp16 copy:
// one 16-byte vector (8 values) per thread and step, grid-stride over the rows.
__global__ void __launch_bounds__(256) bf16_to_f16_kernel(const __nv_bfloat16 *x,
                                                          long long xs_b, long long xs_h,
                                                          long long xs_l, uint16_t *y, int H,
                                                          int L, int vpr, long long n) {
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n; i += (long long)gridDim.x * 256) {
        const long long row = i / vpr;
        const int c = int(i % vpr);
        const int l = int(row % L);
        const long long bh = row / L;
        const int h = int(bh % H), b = int(bh / H);
        const uint4 v = __ldcs(reinterpret_cast<const uint4 *>(x + b * xs_b + h * xs_h + l * xs_l) + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            o[k] = pk16(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u));
        __stcs(reinterpret_cast<uint4 *>(y) + i, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

}  // namespace

lcx_status bf16_to_f16_impl(const void *x, const int64_t *x_strides, void *y, int64_t B,
                            int64_t H, int64_t L, int64_t D, cudaStream_t s) {
    if (D % 8 != 0) return fail(LCX_ERR_UNSUPPORTED, "head dim must be a multiple of 8");
    const long long n = (long long)B * H * L * (D / 8);
    if (n == 0) return LCX_OK;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long blocks = std::min<long long>((n + 255) / 256, (long long)sms * 8);
    bf16_to_f16_kernel<<<unsigned(blocks), 256, 0, s>>>(
        static_cast<const __nv_bfloat16 *>(x), x_strides[0], x_strides[1], x_strides[2],
        static_cast<uint16_t *>(y), int(H), int(L), int(D / 8), n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "bf16 -> fp16 launch failed: %s", cudaGetErrorString(e));
    return LCX_OK;
}

lcx_status apply_rope_impl(const lcx_rope_params *params, const void *x, void *y, void *y_x8,
                           int32_t dtype, int64_t B, int64_t H, int64_t L,
                           const int64_t *x_strides, const int64_t *y_strides, int64_t pos_offset,
                           cudaStream_t s) {
    lcx_status st = check_rope_params(params);
    if (st != LCX_OK) return st;
    if (dtype != LCX_BF16 && dtype != LCX_F32)
        return fail(LCX_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    if (B < 0 || H < 0 || L < 0) return fail(LCX_ERR_INVALID_ARG, "negative size");
    if (!x_strides) return fail(LCX_ERR_INVALID_ARG, "x_strides is NULL");
    if (pos_offset < 0) return fail(LCX_ERR_INVALID_ARG, "pos_offset must be >= 0");
    if (B == 0 || H == 0 || L == 0) return LCX_OK;
    if (!x || !y) return fail(LCX_ERR_INVALID_ARG, "x or y is NULL");
    const int64_t *ys = y_strides ? y_strides : x_strides;
    const int D = params->head_dim;
    if (x_strides[3] != 1 || ys[3] != 1)
        return fail(LCX_ERR_UNSUPPORTED, "the head_dim stride must be 1");
    if (D % 16 != 0) return fail(LCX_ERR_UNSUPPORTED, "head_dim %d must be a multiple of 16", D);
    if (B > 65535) return fail(LCX_ERR_UNSUPPORTED, "batch %lld exceeds 65535", (long long)B);
    if (L > (int64_t(1) << 31) - 1 || H > (int64_t(1) << 31) - 1)
        return fail(LCX_ERR_UNSUPPORTED, "L or H exceeds 2^31 - 1");
    if (pos_offset + L > (int64_t(1) << 31))
        return fail(LCX_ERR_UNSUPPORTED, "positions must stay below 2^31");
    const int es = dtype == LCX_BF16 ? 2 : 4;
    const int vec = 16 / es;
    for (int d = 0; d < 3; ++d) {
        if (x_strides[d] < 0 || ys[d] < 0)
            return fail(LCX_ERR_UNSUPPORTED, "negative strides are not supported");
        if (x_strides[d] % vec != 0 || ys[d] % vec != 0)
            return fail(LCX_ERR_UNSUPPORTED, "strides must be multiples of 16 bytes");
    }
    if (!aligned16(x) || !aligned16(y) || !aligned16(y_x8))
        return fail(LCX_ERR_UNSUPPORTED, "x and y must be 16-byte aligned");
    if (y_x8 && (dtype != LCX_BF16 || x == y))
        return fail(LCX_ERR_UNSUPPORTED, "split parts need bf16 x and a separate y");
    if (x == y) {
        for (int d = 0; d < 3; ++d)
            if (x_strides[d] != ys[d])
                return fail(LCX_ERR_INVALID_ARG, "in-place rotation needs identical strides");
    }

    RopeArgs a;
    a.x = static_cast<const char *>(x);
    a.y = static_cast<char *>(y);
    a.y_x8 = static_cast<char *>(y_x8);
    a.D = D;
    a.xs_b = x_strides[0];
    a.xs_h = x_strides[1];
    a.xs_l = x_strides[2];
    a.ys_b = ys[0];
    a.ys_h = ys[1];
    a.ys_l = ys[2];
    a.H = int(H);
    a.L = int(L);
    a.pos_offset = pos_offset;
    rope_table_unchecked(params, effective_seq_len(params, pos_offset + L), a.theta, &a.ms);
    const bool half = params->pairing == LCX_PAIR_HALF;
    a.jobs_per_row = half ? (D / 2) / vec : D / vec;
    a.rows_per_cta = 256 / a.jobs_per_row;
    if (a.rows_per_cta < 1) a.rows_per_cta = 1;
    const int threads = a.rows_per_cta * a.jobs_per_row;
    dim3 grid(unsigned((L + a.rows_per_cta - 1) / a.rows_per_cta), unsigned(B));
    if (dtype == LCX_BF16) {
        if (y_x8)
            half ? apply_rope_kernel<__nv_bfloat16, true, true><<<grid, threads, 0, s>>>(a)
                 : apply_rope_kernel<__nv_bfloat16, false, true><<<grid, threads, 0, s>>>(a);
        else
            half ? apply_rope_kernel<__nv_bfloat16, true, false><<<grid, threads, 0, s>>>(a)
                 : apply_rope_kernel<__nv_bfloat16, false, false><<<grid, threads, 0, s>>>(a);
    } else {
        if (half)
            apply_rope_kernel<float, true, false><<<grid, threads, 0, s>>>(a);
        else
            apply_rope_kernel<float, false, false><<<grid, threads, 0, s>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(LCX_ERR_CUDA, "apply_rope launch failed: %s", cudaGetErrorString(e));
    return LCX_OK;
}

}  // namespace lcx

extern "C" lcx_status lcx_apply_rope(const lcx_rope_params *params, const void *x, void *y,
                                     int32_t dtype, int64_t B, int64_t H, int64_t L,
                                     const int64_t *x_strides, const int64_t *y_strides,
                                     int64_t pos_offset, void *stream) {
    lcx::clear_error();
    return lcx::apply_rope_impl(params, x, y, nullptr, dtype, B, H, L, x_strides, y_strides,
                                pos_offset, static_cast<cudaStream_t>(stream));
}
