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
    float u;      // W / s (see round_quotient for its accuracy)
    float c;      // clamped code, integer-valued
    bool inside;  // 0 <= round(W/s) + zr <= Q
};

// round(RN(W/s)) without a division per weight.  With rcp = RN(1/s),
// q = RN(W * rcp) satisfies |q - RN(W/s)| < |W/s| 2^-22 (two roundings of the
// quotient against one), so round(q) can differ from round(RN(W/s)) only if q
// lies within |q| 2^-21 of a half-integer, a rounding boundary of round().
// There the IEEE division decides; elsewhere the product does.  The returned
// integer is therefore always round(RN(W/s)); u is RN(W/s) on the exact path
// and q (within 2^-22 relative) otherwise.
__device__ __forceinline__ float round_quotient(float w, float s, float rcp, float &u) {
    const float q = __fmul_rn(w, rcp);
    const float r = rintf(q);
    const float to_half = __fsub_rn(0.5f, fabsf(__fsub_rn(q, r)));  // distance to nearest half-integer
    if (to_half <= fabsf(q) * 0x1p-21f) {
        u = __fdiv_rn(w, s);
        return rintf(u);
    }
    u = q;
    return r;
}

// Round-half-to-even with two full-rate additions: for |x| < 2^22,
// RN(RN(x + 1.5 * 2^23) - 1.5 * 2^23) == rint(x), because x + 1.5 * 2^23 lies in
// [2^23, 2^24) where the spacing of fp32 is 1.  (For larger |x| the callers'
// near-boundary test always fires and the exact path decides.)  Unlike rintf this
// keeps the work off the quarter-rate conversion pipe.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float rint_small(float x) { return __fsub_rn(__fadd_rn(x, kRoundMagic), kRoundMagic); }

// round_quotient for N weights of one group with a single branch: the fast
// decisions for all N first, then, only if one of them lies within the bound of a
// rounding boundary, the IEEE division for those.  r[j] = round(RN(w[j]/s)); u[j]
// as in round_quotient.
template <int N>
__device__ __forceinline__ void round_quotients(const float (&w)[N], float s, float rcp, float (&r)[N],
                                                float (&u)[N]) {
    bool near = false;
#pragma unroll
    for (int j = 0; j < N; ++j) {
        u[j] = __fmul_rn(w[j], rcp);
        r[j] = rint_small(u[j]);
        // near a half-integer: |u - r| >= 1/2 - |u| 2^-21 (one rounding of the
        // threshold, far inside the factor-2 margin of the bound)
        near |= fabsf(__fsub_rn(u[j], r[j])) >= __fmaf_rn(fabsf(u[j]), -0x1p-21f, 0.5f);
    }
    if (near) {
#pragma unroll
        for (int j = 0; j < N; ++j) {
            if (fabsf(__fsub_rn(u[j], r[j])) >= __fmaf_rn(fabsf(u[j]), -0x1p-21f, 0.5f)) {
                u[j] = __fdiv_rn(w[j], s);
                r[j] = rintf(u[j]);
            }
        }
    }
}

// Eq. 1 and the straight-through mask for one weight; rcp = __frcp_rn(s).
__device__ __forceinline__ QuantElem quant_elem(float w, float s, float rcp, float zr, float Q) {
    QuantElem e;
    const float q = __fadd_rn(round_quotient(w, s, rcp, e.u), zr);
    e.inside = (q >= 0.0f) && (q <= Q);
    e.c = fminf(fmaxf(q, 0.0f), Q);
    return e;
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

// 8 consecutive elements as stored: one 16-byte word of bf16, two of fp32.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
    uint4 v;
};
template <>
struct Raw8<float> {
    float4 a, b;
};

template <typename T>
__device__ __forceinline__ Raw8<T> load_raw8(const T *p);
template <>
__device__ __forceinline__ Raw8<__nv_bfloat16> load_raw8<__nv_bfloat16>(const __nv_bfloat16 *p) {
    return Raw8<__nv_bfloat16>{__ldg(reinterpret_cast<const uint4 *>(p))};
}
template <>
__device__ __forceinline__ Raw8<float> load_raw8<float>(const float *p) {
    return Raw8<float>{__ldg(reinterpret_cast<const float4 *>(p)), __ldg(reinterpret_cast<const float4 *>(p) + 1)};
}

__device__ __forceinline__ void unpack8(const Raw8<__nv_bfloat16> &r, float (&v)[8]) {
    v[0] = bf16_lo(r.v.x); v[1] = bf16_hi(r.v.x);
    v[2] = bf16_lo(r.v.y); v[3] = bf16_hi(r.v.y);
    v[4] = bf16_lo(r.v.z); v[5] = bf16_hi(r.v.z);
    v[6] = bf16_lo(r.v.w); v[7] = bf16_hi(r.v.w);
}
__device__ __forceinline__ void unpack8(const Raw8<float> &r, float (&v)[8]) {
    v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
    v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
}

// Exact min and max of the 8 elements (bf16 min/max on packed pairs; the
// widening to fp32 is exact).
__device__ __forceinline__ void minmax8(const Raw8<__nv_bfloat16> &r, float &mn, float &mx) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r.v);
    __nv_bfloat162 lo = __hmin2(__hmin2(h[0], h[1]), __hmin2(h[2], h[3]));
    __nv_bfloat162 hi = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
    mn = fminf(__low2float(lo), __high2float(lo));
    mx = fmaxf(__low2float(hi), __high2float(hi));
}
__device__ __forceinline__ void minmax8(const Raw8<float> &r, float &mn, float &mx) {
    mn = fminf(fminf(fminf(r.a.x, r.a.y), fminf(r.a.z, r.a.w)), fminf(fminf(r.b.x, r.b.y), fminf(r.b.z, r.b.w)));
    mx = fmaxf(fmaxf(fmaxf(r.a.x, r.a.y), fmaxf(r.a.z, r.a.w)), fmaxf(fmaxf(r.b.x, r.b.y), fmaxf(r.b.z, r.b.w)));
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

// 32 bytes from 8 registers in one instruction (p 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                             uint32_t f, uint32_t g, uint32_t h) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d), "r"(e), "r"(f), "r"(g), "r"(h)
                 : "memory");
}

// 16 consecutive values. With V8 (p 32-byte aligned) every store instruction
// writes whole 32-byte sectors: a warp whose lanes store 32 consecutive bytes each
// as two 16-byte halves leaves every sector half written by each instruction, and
// such stores stream at about half the rate of whole-sector ones on B200 (3.5
// against 6.1-6.8 TB/s over a 1 GiB buffer).  Without V8, two 16-byte stores.
template <typename T, bool V8>
__device__ __forceinline__ void store16(T *p, const float (&v)[16]);

template <>
__device__ __forceinline__ void store16<__nv_bfloat16, true>(__nv_bfloat16 *p, const float (&v)[16]) {
    st_global_v8(p, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                 pack_bf16x2(v[6], v[7]), pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                 pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
}
template <>
__device__ __forceinline__ void store16<float, true>(float *p, const float (&v)[16]) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
        st_global_v8(p + 8 * h, __float_as_uint(v[8 * h]), __float_as_uint(v[8 * h + 1]), __float_as_uint(v[8 * h + 2]),
                     __float_as_uint(v[8 * h + 3]), __float_as_uint(v[8 * h + 4]), __float_as_uint(v[8 * h + 5]),
                     __float_as_uint(v[8 * h + 6]), __float_as_uint(v[8 * h + 7]));
}
template <>
__device__ __forceinline__ void store16<__nv_bfloat16, false>(__nv_bfloat16 *p, const float (&v)[16]) {
    store8<__nv_bfloat16>(p, *reinterpret_cast<const float(*)[8]>(&v[0]));
    store8<__nv_bfloat16>(p + 8, *reinterpret_cast<const float(*)[8]>(&v[8]));
}
template <>
__device__ __forceinline__ void store16<float, false>(float *p, const float (&v)[16]) {
    store8<float>(p, *reinterpret_cast<const float(*)[8]>(&v[0]));
    store8<float>(p + 8, *reinterpret_cast<const float(*)[8]>(&v[8]));
}

}  // namespace eqat
