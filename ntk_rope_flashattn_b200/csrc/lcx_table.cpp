// lcx_table.cpp -- the RoPE frequency table per scaling mode (host, fp64 math,
// one rounding to fp32), argument checks and error reporting for the C ABI.
//
// Frequencies ("Long Context: RoPE / YaRN / NTK / MLA", sections 2.4, 4.2, 5.2,
// 6.2, 6.3; "8.3 长上下文技术", sections 8.3.1-8.3.3):
//   theta_i  = 1 / b^(2i/D)
//   PI       : theta_i / s
//   NTK      : 1 / (b s^(D/(D-2)))^(2i/D)
//   YARN     : theta_i * (ramp_i + (1 - ramp_i) / s),
//              ramp_i = clamp((L_train theta_i / 2pi - alpha) / (beta - alpha), 0, 1)
//   DYNAMIC  : NTK with s = seq_len / L_train when seq_len > L_train, else plain
//              ("AI Day 9: 长上下文技术", Dynamic NTK)
//   FACTORS  : theta_i / lambda_i, the short table while seq_len <= L_train
//              (Long Context 7.3-7.4, LongRoPE)
//   mscale   : 1 + 0.1 ln s for YARN with s > 1, otherwise 1.
#include <cmath>
#include <cstdarg>
#include <cstring>

#include "lcx_internal.h"

namespace lcx {

namespace {
thread_local char g_last_error[512] = {0};
}

lcx_status fail(lcx_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

void clear_error() { g_last_error[0] = 0; }

lcx_status check_rope_params(const lcx_rope_params *p) {
    if (!p) return fail(LCX_ERR_INVALID_ARG, "rope params pointer is NULL");
    if (p->mode < LCX_ROPE_NONE || p->mode > LCX_ROPE_FACTORS)
        return fail(LCX_ERR_INVALID_ARG, "unknown rope mode %d", p->mode);
    if (p->head_dim < 2 || p->head_dim > 512 || (p->head_dim & 1))
        return fail(LCX_ERR_INVALID_ARG, "head_dim %d must be even and in [2, 512]", p->head_dim);
    if (p->pairing != LCX_PAIR_HALF && p->pairing != LCX_PAIR_INTERLEAVED)
        return fail(LCX_ERR_INVALID_ARG, "unknown pairing %d", p->pairing);
    if (p->reserved != 0) return fail(LCX_ERR_INVALID_ARG, "reserved field must be 0");
    if (p->mode != LCX_ROPE_NONE && !(p->base > 1.0 && std::isfinite(p->base)))
        return fail(LCX_ERR_INVALID_ARG, "base %g must be finite and > 1", p->base);
    if ((p->mode == LCX_ROPE_PI || p->mode == LCX_ROPE_NTK || p->mode == LCX_ROPE_YARN) &&
        !(p->scale > 0.0 && std::isfinite(p->scale)))
        return fail(LCX_ERR_INVALID_ARG, "scale %g must be finite and > 0", p->scale);
    if ((p->mode == LCX_ROPE_NTK || p->mode == LCX_ROPE_DYNAMIC_NTK) && p->head_dim < 4)
        return fail(LCX_ERR_INVALID_ARG, "NTK scaling needs head_dim >= 4");
    if (p->seq_len < 0) return fail(LCX_ERR_INVALID_ARG, "seq_len must be >= 0");
    if (p->mode == LCX_ROPE_DYNAMIC_NTK && p->original_max_pos <= 0)
        return fail(LCX_ERR_INVALID_ARG, "original_max_pos must be > 0 for dynamic NTK");
    if (p->mode == LCX_ROPE_FACTORS) {
        if (!p->factors) return fail(LCX_ERR_INVALID_ARG, "factor table is NULL");
        for (int i = 0; i < p->head_dim / 2; ++i) {
            if (!(p->factors[i] > 0.0) || !std::isfinite(p->factors[i]))
                return fail(LCX_ERR_INVALID_ARG, "factor %d must be finite and > 0", i);
            if (p->factors_short &&
                (!(p->factors_short[i] > 0.0) || !std::isfinite(p->factors_short[i])))
                return fail(LCX_ERR_INVALID_ARG, "short factor %d must be finite and > 0", i);
        }
    }
    if (p->mode == LCX_ROPE_YARN) {
        if (p->original_max_pos <= 0)
            return fail(LCX_ERR_INVALID_ARG, "original_max_pos must be > 0 for YaRN");
        if (!(p->beta > p->alpha) || !std::isfinite(p->alpha) || !std::isfinite(p->beta))
            return fail(LCX_ERR_INVALID_ARG, "YaRN needs finite alpha < beta (got %g, %g)",
                        p->alpha, p->beta);
    }
    return LCX_OK;
}

void rope_table_unchecked(const lcx_rope_params *p, int64_t seq_len, float *inv_freq,
                          float *mscale) {
    const int D = p->head_dim;
    const double two_pi = 6.283185307179586476925286766559;
    int mode = p->mode;
    double s_ntk = p->scale;
    if (mode == LCX_ROPE_DYNAMIC_NTK) {
        if (seq_len > p->original_max_pos) {
            mode = LCX_ROPE_NTK;
            s_ntk = double(seq_len) / double(p->original_max_pos);
        } else {
            mode = LCX_ROPE_PLAIN;
        }
    }
    const double *lam = nullptr;
    if (mode == LCX_ROPE_FACTORS)
        lam = (p->factors_short && seq_len <= p->original_max_pos) ? p->factors_short : p->factors;
    const double ntk_base =
        (mode == LCX_ROPE_NTK) ? p->base * std::pow(s_ntk, double(D) / double(D - 2)) : 0.0;
    for (int i = 0; i < D / 2; ++i) {
        const double expo = (2.0 * i) / double(D);
        double f = 0.0;
        switch (mode) {
            case LCX_ROPE_NONE:
                f = 0.0;
                break;
            case LCX_ROPE_PLAIN:
                f = 1.0 / std::pow(p->base, expo);
                break;
            case LCX_ROPE_PI:
                f = 1.0 / (std::pow(p->base, expo) * p->scale);
                break;
            case LCX_ROPE_NTK:
                f = 1.0 / std::pow(ntk_base, expo);
                break;
            case LCX_ROPE_YARN: {
                const double theta = 1.0 / std::pow(p->base, expo);
                const double turns = double(p->original_max_pos) * theta / two_pi;
                double ramp = (turns - p->alpha) / (p->beta - p->alpha);
                ramp = ramp < 0.0 ? 0.0 : (ramp > 1.0 ? 1.0 : ramp);
                f = theta * (ramp + (1.0 - ramp) / p->scale);
                break;
            }
            case LCX_ROPE_FACTORS:
                f = 1.0 / (std::pow(p->base, expo) * lam[i]);
                break;
        }
        inv_freq[i] = static_cast<float>(f);
    }
    const double ms =
        (mode == LCX_ROPE_YARN && p->scale > 1.0) ? 1.0 + 0.1 * std::log(p->scale) : 1.0;
    *mscale = static_cast<float>(ms);
}

}  // namespace lcx

extern "C" {

lcx_status lcx_rope_table(const lcx_rope_params *params, float *inv_freq, float *mscale) {
    lcx::clear_error();
    lcx_status st = lcx::check_rope_params(params);
    if (st != LCX_OK) return st;
    if (!inv_freq || !mscale)
        return lcx::fail(LCX_ERR_INVALID_ARG, "inv_freq and mscale must be non-NULL");
    if ((params->mode == LCX_ROPE_DYNAMIC_NTK || params->mode == LCX_ROPE_FACTORS) &&
        params->seq_len <= 0)
        return lcx::fail(LCX_ERR_INVALID_ARG, "this mode needs seq_len > 0");
    lcx::rope_table_unchecked(params, params->seq_len, inv_freq, mscale);
    return LCX_OK;
}

const char *lcx_status_string(lcx_status status) {
    switch (status) {
        case LCX_OK: return "ok";
        case LCX_ERR_INVALID_ARG: return "invalid argument";
        case LCX_ERR_UNSUPPORTED: return "unsupported argument combination";
        case LCX_ERR_CUDA: return "CUDA error";
        case LCX_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char *lcx_last_error(void) { return lcx::g_last_error; }

int32_t lcx_version(void) { return LCX_VERSION; }

}  // extern "C"
