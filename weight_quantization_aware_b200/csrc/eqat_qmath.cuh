// Element arithmetic of the EfficientQAT quantizer, in IEEE fp32 with explicit
// rounding intrinsics so that no step is contracted into an FMA or replaced by a
// reciprocal.  Eq. 1 and Eq. 2 of the zhaoyang97 ACL2025 notes ("Block-AP"):
//   W_int = clamp(round(W/s) + z, 0, 2^b - 1),   W-hat = (W_int - z) * s,
// with z rounded in every forward (modelfoundations note, "Paper vs. code":
// round_ste on the zero point) and round() half-to-even.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace eqat {

constexpr float kStepMin = 1e-5f;  // floor of s for constant groups (EQAT_S_MIN)

struct QuantElem {
    float u;      // W / s, correctly rounded
    float c;      // clamped code, integer-valued
    bool inside;  // 0 <= round(u) + zr <= Q
};

__device__ __forceinline__ QuantElem quant_elem(float w, float s, float zr, float Q) {
    QuantElem e;
    e.u = __fdiv_rn(w, s);
    const float q = __fadd_rn(rintf(e.u), zr);
    e.inside = (q >= 0.0f) && (q <= Q);
    e.c = fminf(fmaxf(q, 0.0f), Q);
    return e;
}

__device__ __forceinline__ float dequant_elem(float c, float zr, float s) {
    return __fmul_rn(__fsub_rn(c, zr), s);
}

// Min-max init of one group (modelfoundations note, Phase 1).
__device__ __forceinline__ void minmax_step_zero(float xmin, float xmax, float Q, float &s,
                                                 float &z) {
    float sc = __fdiv_rn(__fsub_rn(xmax, xmin), Q);
    if (!(sc >= kStepMin)) sc = kStepMin;
    s = sc;
    z = rintf(__fdiv_rn(-xmin, sc));
}

// ---------------------------------------------------------------- bf16 helpers

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
    return *reinterpret_cast<uint32_t *>(&h);
}

// Loads 8 consecutive elements (16 bytes of bf16, 32 bytes of fp32) as floats.
template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 r = __ldg(reinterpret_cast<const uint4 *>(p));
    v[0] = bf16_lo(r.x); v[1] = bf16_hi(r.x);
    v[2] = bf16_lo(r.y); v[3] = bf16_hi(r.y);
    v[4] = bf16_lo(r.z); v[5] = bf16_hi(r.z);
    v[6] = bf16_lo(r.w); v[7] = bf16_hi(r.w);
}

template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void store8(T *p, const float (&v)[8]);

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 r;
    r.x = pack_bf16x2(v[0], v[1]);
    r.y = pack_bf16x2(v[2], v[3]);
    r.z = pack_bf16x2(v[4], v[5]);
    r.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(p) = r;
}

template <>
__device__ __forceinline__ void store8<float>(float *p, const float (&v)[8]) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

}  // namespace eqat
