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
    char *y_lo;                  // bf16 only, or NULL: y_lo = bf16(y' - bf16(y'))
    long long xs_b, xs_h, xs_l;  // element strides
    long long ys_b, ys_h, ys_l;
    int H, L;
    long long pos_offset;
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

// The residual of the bf16 rounding, y - bf16(y), rounded to bf16 again: the
// "lo" half of a hi/lo pair (hi + lo carries y to ~16 significant bits).  Same
// layout as y; e2 < 0 means only the vector at e1 exists.
template <int N>
__device__ __forceinline__ void store_lo(const RopeArgs &a, int b, int l, int h, int e1, int e2,
                                         const float (&y1)[N], const float (&y2)[N],
                                         const uint4 &h1, const uint4 &h2) {
    __nv_bfloat16 *lr = reinterpret_cast<__nv_bfloat16 *>(
        a.y_lo + 2 * (b * a.ys_b + l * a.ys_l + (long long)h * a.ys_h));
    float r1[8], r2[8], f[8];
    unpack(h1, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) r1[e] = y1[e] - f[e];
    __stcs(reinterpret_cast<uint4 *>(lr + e1), pack(r1));
    if (e2 >= 0) {
        unpack(h2, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) r2[e] = y2[e] - f[e];
        __stcs(reinterpret_cast<uint4 *>(lr + e2), pack(r2));
    }
}

// HALF pairing: a job covers N consecutive pairs i0..i0+N-1, i.e. the vector
// at element i0 and the vector at element i0 + D/2.  kLo: also write the lo
// parts (bf16 only).
template <typename T, bool kHalf, bool kLo>
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
                const uint4 h1 = pack(y1), h2 = pack(y2);
                __stcs(reinterpret_cast<uint4 *>(yr + e1), h1);
                __stcs(reinterpret_cast<uint4 *>(yr + e2), h2);
                if constexpr (sizeof(T) == 2 && kLo)
                    store_lo(a, b, l, h0 + u, e1, e2, y1, y2, h1, h2);
            } else {
                float x[N], y[N];
                unpack(va[u], x);
#pragma unroll
                for (int e = 0; e < P; ++e) {
                    y[2 * e] = fmaf(x[2 * e], c[e], -x[2 * e + 1] * s[e]);
                    y[2 * e + 1] = fmaf(x[2 * e], s[e], x[2 * e + 1] * c[e]);
                }
                const uint4 h = pack(y);
                __stcs(reinterpret_cast<uint4 *>(yr + e1), h);
                if constexpr (sizeof(T) == 2 && kLo)
                    store_lo(a, b, l, h0 + u, e1, -1, y, y, h, h);
            }
        }
    }
}

}  // namespace

lcx_status apply_rope_impl(const lcx_rope_params *params, const void *x, void *y, void *y_lo,
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
    if (!aligned16(x) || !aligned16(y) || !aligned16(y_lo))
        return fail(LCX_ERR_UNSUPPORTED, "x and y must be 16-byte aligned");
    if (y_lo && dtype != LCX_BF16) return fail(LCX_ERR_UNSUPPORTED, "a lo part needs bf16");
    if (x == y) {
        for (int d = 0; d < 3; ++d)
            if (x_strides[d] != ys[d])
                return fail(LCX_ERR_INVALID_ARG, "in-place rotation needs identical strides");
    }

    RopeArgs a;
    a.x = static_cast<const char *>(x);
    a.y = static_cast<char *>(y);
    a.y_lo = static_cast<char *>(y_lo);
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
        if (y_lo)
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
