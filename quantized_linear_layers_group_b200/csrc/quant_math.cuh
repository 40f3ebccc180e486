// quant_math.cuh -- the per-element arithmetic of dynamic quantisation,
// shared by the stand-alone quantisers and the GEMM that quantises its own
// activation tiles, so that both produce the same codes and scales bit for bit.
//
//   scale = amax / Qmax          IEEE binary32 division (__fdiv_rn)
//   v     = x / scale            correctly rounded quotient (see quotient())
//   INT8: q = clamp(rint_half_even(v), -127, 127)
//   FP8 : q = e4m3_rn_satfinite(clamp(v, -448, 448))
//   amax == 0 -> scale = 0, q = 0.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qlin.h"

namespace qlin {
namespace qm {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// 8 bf16 in a uint4 -> 8 floats (exact widening)
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        f[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

__device__ __forceinline__ float absmax8(const uint4& v) {
    float f[8];
    unpack8(v, f);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// The quotient x / s, correctly rounded (IEEE binary32 division) for every x
// whose code can be non-zero.  One scale serves a whole row (or group), so its
// reciprocal r = RN(1/s) is formed once and each element takes Markstein's
// correction step (P. Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// q0 = RN(x r) within an ulp of x/s, the residual x - q0 s is exact as an fma
// and RN(q0 + residual * r) is the correctly rounded quotient, barring
// underflow or overflow.  For s in [2^-68, 2^92] neither can touch a quotient
// of magnitude >= 2^-33, and anything smaller than that quantises to a zero
// code under either rounding; copysign keeps the sign of a zero x.  Other
// scales use the IEEE division itself.
struct Divisor {
    float s, r;
    bool fast;
};

__device__ __forceinline__ Divisor make_divisor(float s) {
    Divisor d;
    d.s = s;
    d.fast = (s >= 0x1p-68f && s <= 0x1p92f);
    d.r = d.fast ? __frcp_rn(s) : 0.f;
    return d;
}

// FAST_ONLY: the caller has checked d.fast, so no IEEE division is compiled
// in (and no registers need to survive a call to it).
template <bool FAST_ONLY = false>
__device__ __forceinline__ float quotient(float x, const Divisor& d) {
    if (FAST_ONLY || d.fast) {
        const float q0 = __fmul_rn(x, d.r);
        const float rem = __fmaf_rn(-q0, d.s, x);
        return copysignf(__fmaf_rn(rem, d.r, q0), x);
    }
    return __fdiv_rn(x, d.s);
}

template <bool FAST_ONLY = false>
__device__ __forceinline__ uint32_t quant_int8_x4(const float* f, const Divisor& d) {
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int r = 0;
        if (d.s != 0.f) {
            r = __float2int_rn(quotient<FAST_ONLY>(f[i], d));
            r = max(-127, min(127, r));
        }
        out |= (uint32_t)(r & 0xFF) << (8 * i);
    }
    return out;
}

template <bool FAST_ONLY = false>
__device__ __forceinline__ uint32_t quant_e4m3_x4(const float* f, const Divisor& d) {
    if (d.s == 0.f) return 0u;
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = fminf(fmaxf(quotient<FAST_ONLY>(f[i], d), -448.f), 448.f);
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[0], v[1]), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v[2], v[3]), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

template <int FMT, bool FAST_ONLY = false>
__device__ __forceinline__ uint2 quant8(const uint4& v, const Divisor& d) {
    float f[8];
    unpack8(v, f);
    uint2 r;
    if constexpr (FMT == QLIN_FMT_INT8) {
        r.x = quant_int8_x4<FAST_ONLY>(f, d);
        r.y = quant_int8_x4<FAST_ONLY>(f + 4, d);
    } else {
        r.x = quant_e4m3_x4<FAST_ONLY>(f, d);
        r.y = quant_e4m3_x4<FAST_ONLY>(f + 4, d);
    }
    return r;
}

}  // namespace qm
}  // namespace qlin
