// HBM-bound kernels of the quantizer: per-group min-max init, the fake-quant
// prepass (codes, mask, W-hat), packing to low-bit integers and the E2E-QP
// dequantization of frozen codes.
//
// Every kernel streams its input once with 16-byte loads; a group (g in
// {32, 64, 128} consecutive in-features of one row) is never split across
// warps, so per-group reductions are warp shuffles and per-group parameters are
// read once per thread from L1.  Grids are grid-stride loops sized to a whole
// number of waves of the SMs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "eqat_internal.h"
#include "eqat_qmath.cuh"

namespace eqat {
namespace {

constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 8;

// log2 of the group size (32, 64 or 128): index arithmetic by shifts, not division.
inline int group_shift(int group) { return group == 32 ? 5 : group == 64 ? 6 : 7; }

inline int grid_for(int64_t work_items, const DeviceInfo &dev, int per_thread = 1) {
    const int64_t threads = (work_items + per_thread - 1) / per_thread;
    const int64_t blocks = (threads + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(dev.sm_count) * kBlocksPerSm;
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, cap)));
}

// ------------------------------------------------------------------ min-max init
// A thread holds 8 consecutive weights of one group; TPG = G/8 threads cover a
// group and reduce min/max with xor shuffles; UNROLL independent groups per
// thread keep 128 bytes (bf16) of loads in flight per thread.
template <typename T, int G>
__global__ void __launch_bounds__(kThreads, 4) k_minmax_init(const T *__restrict__ W, int64_t n_groups,
                                                             float Q, float *__restrict__ s,
                                                             float *__restrict__ z) {
    constexpr int TPG = G / 8;
    constexpr int GPW = 32 / TPG;  // groups per warp per unrolled slot
    constexpr int UNROLL = 4;  // 16-byte words in flight per thread
    const int lane = threadIdx.x & 31;
    const int sub = lane % TPG;
    const int slot = lane / TPG;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    for (int64_t base = warp * (GPW * UNROLL); base < n_groups; base += nwarps * (GPW * UNROLL)) {
        Raw8<T> raw[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t g = base + u * GPW + slot;
            if (g < n_groups) raw[u] = load_raw8<T>(W + g * G + sub * 8);
        }
        // Reduce every chunk to (min, max) first so the raw words die before the
        // shuffles and the per-group divisions.
        float mn[UNROLL], mx[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            mn[u] = 0.0f;
            mx[u] = 0.0f;
            if (base + u * GPW + slot < n_groups) minmax8(raw[u], mn[u], mx[u]);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
#pragma unroll
            for (int off = TPG / 2; off > 0; off >>= 1) {
                mn[u] = fminf(mn[u], __shfl_xor_sync(0xffffffffu, mn[u], off));
                mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], off));
            }
        }
        // After the xor-shuffles every lane of a group holds its (min, max): lane
        // `sub` finishes chunks sub, sub + TPG, ... so the divisions spread over
        // the group's lanes instead of running one after another on one lane.
        constexpr int PER_LANE = (UNROLL + TPG - 1) / TPG;
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) {
            const int uu = sub + k * TPG;
            float a = 0.0f, b = 0.0f;
#pragma unroll
            for (int u = 0; u < UNROLL; ++u)
                if (u == uu) {
                    a = mn[u];
                    b = mx[u];
                }
            const int64_t g = base + uu * GPW + slot;
            if (uu < UNROLL && g < n_groups) {
                float sc, zz;
                minmax_step_zero(a, b, Q, sc, zz);
                s[g] = sc;
                z[g] = zz;
            }
        }
    }
}

// ------------------------------------------------------------------ fake-quant prepass
// A thread handles U = 2 chunks of 8 consecutive weights (each chunk inside one
// group) per iteration and issues both loads before any arithmetic.
template <typename T, typename O, bool CODES>
__device__ __forceinline__ void fake_quant_chunk(const float (&w)[8], float sc, float zr, float Q,
                                                 int64_t e0, O *__restrict__ W_hat,
                                                 uint8_t *__restrict__ code, uint8_t *__restrict__ mask) {
    const float rcp = __frcp_rn(sc);
    const float lo = kRoundMagic, hi = __fadd_rn(kRoundMagic, Q);
    const float mz = __fadd_rn(kRoundMagic, zr);  // W-hat = (M + code - (M + zr)) s
    float qm[8];
    bool inside[8];
    bool near = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float t = magic_decision(w[j], rcp, zr, near);  // M + round(u) + zr
        inside[j] = (t >= lo) && (t <= hi);
        qm[j] = fminf(fmaxf(t, lo), hi);
    }
    if (near) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            bool nj = false;
            (void)magic_decision(w[j], rcp, zr, nj);
            if (nj) qm[j] = exact_decision(w[j], sc, zr, Q, inside[j]);
        }
    }
    float wh[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) wh[j] = __fmul_rn(__fsub_rn(qm[j], mz), sc);
    if (W_hat) store8<O>(W_hat + e0, wh);
    if (CODES) {
        uint32_t c_lo = 0, c_hi = 0, m_lo = 0, m_hi = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t cb = static_cast<uint32_t>(__float_as_int(qm[j])) & 0xFFu;
            const uint32_t mb = inside[j] ? 1u : 0u;
            if (j < 4) {
                c_lo |= cb << (8 * j);
                m_lo |= mb << (8 * j);
            } else {
                c_hi |= cb << (8 * (j - 4));
                m_hi |= mb << (8 * (j - 4));
            }
        }
        if (code) *reinterpret_cast<uint2 *>(code + e0) = make_uint2(c_lo, c_hi);
        if (mask) *reinterpret_cast<uint2 *>(mask + e0) = make_uint2(m_lo, m_hi);
    }
}

template <typename T, typename O, bool CODES>
__global__ void __launch_bounds__(kThreads, 4)
    k_fake_quant(const T *__restrict__ W, const float *__restrict__ s, const float *__restrict__ z,
                 int64_t n_chunks, int gshift, float Q, O *__restrict__ W_hat,
                 uint8_t *__restrict__ code, uint8_t *__restrict__ mask) {
    constexpr int U = 2;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; base < n_chunks;
         base += nthreads * U) {
        Raw8<T> raw[U];
        float sc[U], zr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * nthreads;
            if (i < n_chunks) {
                raw[u] = load_raw8<T>(W + i * 8);
                const int64_t g = (i * 8) >> gshift;
                sc[u] = __ldg(s + g);
                zr[u] = rintf(__ldg(z + g));
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * nthreads;
            if (i < n_chunks) {
                float w[8];
                unpack8(raw[u], w);
                fake_quant_chunk<T, O, CODES>(w, sc[u], zr[u], Q, i * 8, W_hat, code, mask);
            }
        }
    }
}

// ------------------------------------------------------------------ pack
// One thread per 16 consecutive weights (same group).  zq = clamp(round(z), 0, Q)
// and the codes use zr := zq (z hard-rounded at pack time).  Output per thread:
// 4 bytes (2-bit), 8 bytes (4-bit) or 16 bytes (3-bit, one code per byte).
// Two fp32 lanes in one 64-bit register, and the packed-pair arithmetic of
// sm_100 (each lane an IEEE round-to-nearest operation, as the scalar forms).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

template <int BITS>
__device__ __forceinline__ void pack_chunk(const float (&w)[16], float sc, float zr, float Q, int64_t e0,
                                           uint8_t *__restrict__ codes) {
    const float rcp = __frcp_rn(sc);
    const float lo = kRoundMagic, hi = __fadd_rn(kRoundMagic, Q);
    // M + zr is exact; one add of it gives M + zr + round(u) for every u that is
    // not an exact tie (ties may break toward an odd total, but a tie lies in the
    // near band below and takes the exact path).
    const float mz = __fadd_rn(kRoundMagic, zr);
    const uint64_t rcp2 = f2_pack(rcp, rcp), mz2 = f2_pack(mz, mz);
    // Each code enters its word as the raw bits of M + code (one multiply-add);
    // the bits of M are taken out once per word at the end.
    uint32_t word[4] = {0u, 0u, 0u, 0u};  // 2-bit: word[0]; 4-bit: word[0..1]; 3-bit: word[0..3]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float cm[8];
        bool near = false;
        // two weights per step: u = RN(w rcp), t = RN(u + M + zr), and the
        // distance u - (t - M - zr) of u from its rounded value
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const uint64_t u2 = f2_mul(f2_pack(w[8 * h + j], w[8 * h + j + 1]), rcp2);
            const uint64_t t2 = f2_add(u2, mz2);
            const uint64_t r2 = f2_sub(u2, f2_sub(t2, mz2));
            float t0, t1, r0, r1;
            f2_unpack(t2, t0, t1);
            f2_unpack(r2, r0, r1);
            // |u - RN(w / s)| < |u| 2^-22: only a u within that of a half-integer can
            // round differently.  A code that is not clamped has |u| <= Q + zr + 1/2 < 64,
            // so a band of 2^-16 covers it; a clamped code does not depend on it.
            near |= fabsf(r0) >= 0.5f - 0x1p-16f;
            near |= fabsf(r1) >= 0.5f - 0x1p-16f;
            cm[j] = fminf(fmaxf(t0, lo), hi);
            cm[j + 1] = fminf(fmaxf(t1, lo), hi);
        }
        if (near) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                bool nj = false, inside;
                (void)magic_decision(w[8 * h + j], rcp, zr, nj);
                if (nj) cm[j] = exact_decision(w[8 * h + j], sc, zr, Q, inside);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t b = static_cast<uint32_t>(__float_as_int(cm[j]));
            const int k = 8 * h + j;
            if (BITS == 2) word[0] += b << (2 * k);
            else if (BITS == 4) word[k / 8] += b << (4 * (k % 8));
            else word[k / 4] += b << (8 * (k % 4));
        }
    }
    if (BITS == 2) {
        *reinterpret_cast<uint32_t *>(codes + e0 / 4) = word[0] - magic_word(2, 16);
    } else if (BITS == 4) {
        *reinterpret_cast<uint2 *>(codes + e0 / 2) =
            make_uint2(word[0] - magic_word(4, 8), word[1] - magic_word(4, 8));
    } else {
        constexpr uint32_t m = magic_word(8, 4);
        *reinterpret_cast<uint4 *>(codes + e0) = make_uint4(word[0] - m, word[1] - m, word[2] - m, word[3] - m);
    }
}

// A thread handles U = 2 chunks of 16 consecutive weights (each inside one group)
// per iteration, loads first.  zq = clamp(round(z), 0, Q) and the codes use
// zr := zq (z hard-rounded at pack time).  Output per chunk: 4 bytes (2-bit), 8
// bytes (4-bit) or 16 bytes (3-bit, one code per byte).
template <typename T, int BITS>
__global__ void __launch_bounds__(kThreads, 4)
    k_pack(const T *__restrict__ W, const float *__restrict__ s, const float *__restrict__ z,
           int64_t n_chunks, int gshift, float Q, uint8_t *__restrict__ codes,
           uint8_t *__restrict__ zq) {
    constexpr int U = 2;
    const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; base < n_chunks;
         base += nthreads * U) {
        Raw8<T> raw[U][2];
        float sc[U], zr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * nthreads;
            if (i < n_chunks) {
                raw[u][0] = load_raw8<T>(W + i * 16);
                raw[u][1] = load_raw8<T>(W + i * 16 + 8);
                const int64_t g = (i * 16) >> gshift;
                sc[u] = __ldg(s + g);
                zr[u] = fminf(fmaxf(rintf(__ldg(z + g)), 0.0f), Q);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + u * nthreads;
            if (i < n_chunks) {
                const int64_t e0 = i * 16;
                if ((e0 & ((int64_t(1) << gshift) - 1)) == 0) zq[e0 >> gshift] = static_cast<uint8_t>(zr[u]);
                float w[16];
                unpack8(raw[u][0], *reinterpret_cast<float(*)[8]>(&w[0]));
                unpack8(raw[u][1], *reinterpret_cast<float(*)[8]>(&w[8]));
                pack_chunk<BITS>(w, sc[u], zr[u], Q, e0, codes);
            }
        }
    }
}

// ------------------------------------------------------------------ E2E dequant
// One thread per 16 consecutive codes: W-hat = (W_q - zq) * s (Eq. 2).
template <int BITS>
__device__ __forceinline__ void unpack16(const uint8_t *codes, int64_t e0, uint32_t (&c)[16]) {
    if (BITS == 2) {
        const uint32_t word = __ldg(reinterpret_cast<const uint32_t *>(codes + e0 / 4));
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = (word >> (2 * j)) & 3u;
    } else if (BITS == 4) {
        const uint2 r = __ldg(reinterpret_cast<const uint2 *>(codes + e0 / 2));
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j] = (r.x >> (4 * j)) & 15u;
#pragma unroll
        for (int j = 0; j < 8; ++j) c[8 + j] = (r.y >> (4 * j)) & 15u;
    } else {
        const uint4 r = __ldg(reinterpret_cast<const uint4 *>(codes + e0));
        const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = (w4[j / 4] >> (8 * (j % 4))) & 0xFFu;
    }
}

__device__ __forceinline__ float step_value(const float *s, int64_t g) { return __ldg(s + g); }
__device__ __forceinline__ float step_value(const __half *s, int64_t g) { return __half2float(__ldg(s + g)); }

// S: fp32 step sizes, or fp16 ones (fp16 step-size storage), widened exactly.
template <int BITS, typename O, typename S>
__global__ void __launch_bounds__(kThreads)
    k_dequant(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ zq,
              const S *__restrict__ s, int64_t n_chunks, int gshift, O *__restrict__ W_hat) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n_chunks;
         i += stride) {
        const int64_t e0 = i * 16;
        const int64_t g = e0 >> gshift;
        const float sc = step_value(s, g);
        const float zf = static_cast<float>(__ldg(zq + g));
        uint32_t c[16];
        unpack16<BITS>(codes, e0, c);
        float a[8], b[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = dequant_elem(static_cast<float>(c[j]), zf, sc);
#pragma unroll
        for (int j = 0; j < 8; ++j) b[j] = dequant_elem(static_cast<float>(c[8 + j]), zf, sc);
        store8<O>(W_hat + e0, a);
        store8<O>(W_hat + e0 + 8, b);
    }
}

template <typename T>
cudaError_t minmax_dispatch(const T *W, int64_t n_groups, int group, float Q, float *s, float *z,
                            const DeviceInfo &dev, cudaStream_t st) {
    const int grid = grid_for(n_groups * group, dev, 8 * 4);
    switch (group) {
        case 32: k_minmax_init<T, 32><<<grid, kThreads, 0, st>>>(W, n_groups, Q, s, z); break;
        case 64: k_minmax_init<T, 64><<<grid, kThreads, 0, st>>>(W, n_groups, Q, s, z); break;
        case 128: k_minmax_init<T, 128><<<grid, kThreads, 0, st>>>(W, n_groups, Q, s, z); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t pack_dispatch(const T *W, const float *s, const float *z, int64_t n, int bits, int group,
                          uint8_t *codes, uint8_t *zq, const DeviceInfo &dev, cudaStream_t st) {
    const int gshift = group_shift(group);
    const int64_t chunks = n / 16;
    const int grid = grid_for(chunks, dev);
    const float Q = static_cast<float>((1 << bits) - 1);
    switch (bits) {
        case 2: k_pack<T, 2><<<grid, kThreads, 0, st>>>(W, s, z, chunks, gshift, Q, codes, zq); break;
        case 3: k_pack<T, 3><<<grid, kThreads, 0, st>>>(W, s, z, chunks, gshift, Q, codes, zq); break;
        case 4: k_pack<T, 4><<<grid, kThreads, 0, st>>>(W, s, z, chunks, gshift, Q, codes, zq); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename O, typename S>
cudaError_t dequant_dispatch(const uint8_t *codes, const uint8_t *zq, const S *s, int64_t n,
                             int bits, int group, O *W_hat, const DeviceInfo &dev,
                             cudaStream_t st) {
    const int gshift = group_shift(group);
    const int64_t chunks = n / 16;
    const int grid = grid_for(chunks, dev);
    switch (bits) {
        case 2: k_dequant<2, O, S><<<grid, kThreads, 0, st>>>(codes, zq, s, chunks, gshift, W_hat); break;
        case 3: k_dequant<3, O, S><<<grid, kThreads, 0, st>>>(codes, zq, s, chunks, gshift, W_hat); break;
        case 4: k_dequant<4, O, S><<<grid, kThreads, 0, st>>>(codes, zq, s, chunks, gshift, W_hat); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_minmax_init(const void *W, bool w_f32, int64_t N, int64_t K, int bits, int group,
                               float *s, float *z, const DeviceInfo &dev, cudaStream_t st) {
    const int64_t n_groups = N * (K / group);
    if (n_groups == 0) return cudaSuccess;
    const float Q = static_cast<float>((1 << bits) - 1);
    if (w_f32) return minmax_dispatch(static_cast<const float *>(W), n_groups, group, Q, s, z, dev, st);
    return minmax_dispatch(static_cast<const __nv_bfloat16 *>(W), n_groups, group, Q, s, z, dev, st);
}

cudaError_t launch_fake_quant(const void *W, bool w_f32, const float *s, const float *z, int64_t N,
                              int64_t K, int bits, int group, void *W_hat, bool out_f32,
                              uint8_t *code, uint8_t *mask, const DeviceInfo &dev,
                              cudaStream_t st) {
    const int64_t chunks = N * K / 8;
    if (chunks == 0) return cudaSuccess;
    const int grid = grid_for(chunks, dev);
    const float Q = static_cast<float>((1 << bits) - 1);
    using bf = __nv_bfloat16;
    const bool codes = code || mask;
    const int gshift = group_shift(group);
#define EQAT_FQ_LAUNCH(TW, TO)                                                                          \
    do {                                                                                                \
        if (codes)                                                                                      \
            k_fake_quant<TW, TO, true><<<grid, kThreads, 0, st>>>(static_cast<const TW *>(W), s, z, chunks, \
                                                                 gshift, Q, static_cast<TO *>(W_hat), code, mask); \
        else                                                                                            \
            k_fake_quant<TW, TO, false><<<grid, kThreads, 0, st>>>(static_cast<const TW *>(W), s, z, chunks, \
                                                                  gshift, Q, static_cast<TO *>(W_hat), code, mask); \
    } while (0)
    if (w_f32 && out_f32)
        EQAT_FQ_LAUNCH(float, float);
    else if (w_f32)
        EQAT_FQ_LAUNCH(float, bf);
    else if (out_f32)
        EQAT_FQ_LAUNCH(bf, float);
    else
        EQAT_FQ_LAUNCH(bf, bf);
#undef EQAT_FQ_LAUNCH
    return cudaGetLastError();
}

cudaError_t launch_pack(const void *W, bool w_f32, const float *s, const float *z, int64_t N,
                        int64_t K, int bits, int group, uint8_t *codes, uint8_t *zq,
                        const DeviceInfo &dev, cudaStream_t st) {
    const int64_t n = N * K;
    if (n == 0) return cudaSuccess;
    if (w_f32) return pack_dispatch(static_cast<const float *>(W), s, z, n, bits, group, codes, zq, dev, st);
    return pack_dispatch(static_cast<const __nv_bfloat16 *>(W), s, z, n, bits, group, codes, zq, dev, st);
}

cudaError_t launch_dequant(const uint8_t *codes, const uint8_t *zq, const void *s, bool s_f16, int64_t N,
                           int64_t K, int bits, int group, void *W_hat, bool out_f32,
                           const DeviceInfo &dev, cudaStream_t st) {
    const int64_t n = N * K;
    if (n == 0) return cudaSuccess;
    const float *s32 = static_cast<const float *>(s);
    const __half *s16 = static_cast<const __half *>(s);
    float *o32 = static_cast<float *>(W_hat);
    __nv_bfloat16 *o16 = static_cast<__nv_bfloat16 *>(W_hat);
    if (s_f16)
        return out_f32 ? dequant_dispatch(codes, zq, s16, n, bits, group, o32, dev, st)
                       : dequant_dispatch(codes, zq, s16, n, bits, group, o16, dev, st);
    return out_f32 ? dequant_dispatch(codes, zq, s32, n, bits, group, o32, dev, st)
                   : dequant_dispatch(codes, zq, s32, n, bits, group, o16, dev, st);
}

}  // namespace eqat
