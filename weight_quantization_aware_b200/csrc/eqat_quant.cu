// HBM-bound kernels of the quantizer: per-group min-max init, the fake-quant
// prepass (codes, mask, W-hat), packing to low-bit integers and the E2E-QP
// dequantization of frozen codes.
//
// Every kernel streams its input once with coalesced 16-byte loads and keeps a
// group (g in {32, 64, 128} consecutive in-features of one row) inside one warp:
// init reduces a group with warp shuffles; the prepass and pack form each group's
// constants once per warp tile in shared memory and decide two weights per
// packed-fp32 instruction.  Grids are sized to the resident CTAs of the SMs and
// loop over the work.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "eqat_internal.h"
#include "eqat_pdl.cuh"
#include "eqat_qmath.cuh"

namespace eqat {
namespace {

constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 8;

// Every kernel here is launched as a programmatic dependent (eqat_pdl.cuh): it
// waits for the preceding kernel before its first global access, then lets its
// own dependents be scheduled.
__device__ __forceinline__ void begin_dependent() {
    pdl_wait();
    pdl_allow_dependents();
}

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
//
// One launch covers NL weight matrices (NL = 1, or the linears of a block): the
// warps walk units of GPW * UNROLL groups, numbered through the layers in order
// (a unit never spans two layers), so small layers share the waves of large ones
// instead of paying a launch ramp and tail each.
constexpr int kInitUnroll = 4;  // 16-byte words in flight per thread
template <int G>
constexpr int kInitUnit = (32 / (G / 8)) * kInitUnroll;  // groups per warp unit

template <typename T, int NL>
struct InitLayers {
    const T *W[NL];
    float *s[NL];
    float *z[NL];
    int64_t n_groups[NL];
    int64_t unit_end[NL];  // units of layers 0..i; entries past the last layer repeat it
};

template <typename T, int G, int NL>
__global__ void __launch_bounds__(kThreads, 4) k_minmax_init(const __grid_constant__ InitLayers<T, NL> L, float Q) {
    begin_dependent();
    constexpr int TPG = G / 8;
    constexpr int GPW = 32 / TPG;  // groups per warp per unrolled slot
    constexpr int UNROLL = kInitUnroll;
    const int lane = threadIdx.x & 31;
    const int sub = lane % TPG;
    const int slot = lane / TPG;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    const int64_t n_units = L.unit_end[NL - 1];
    int li = 0;
    int64_t unit_begin = 0;
    for (int64_t unit = warp; unit < n_units; unit += nwarps) {
        if constexpr (NL > 1) {
            while (unit >= L.unit_end[li]) {
                unit_begin = L.unit_end[li];
                ++li;
            }
        }
        const T *__restrict__ W = L.W[li];
        float *__restrict__ s = L.s[li];
        float *__restrict__ z = L.z[li];
        const int64_t n_groups = L.n_groups[li];
        const int64_t base = (unit - unit_begin) * (GPW * UNROLL);
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

// ------------------------------------------------------------------ packed fp32 pairs
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

// Two fp32 values to one f16x2 word (round to nearest; hi in the upper half), and
// the per-half min / max of f16x2 words.
__device__ __forceinline__ uint32_t h2_from_f32(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ uint32_t h2_clamp(uint32_t a, uint32_t lo, uint32_t hi) {
    uint32_t d;
    asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(lo));
    asm("min.f16x2 %0, %1, %2;" : "=r"(d) : "r"(d), "r"(hi));
    return d;
}

// ------------------------------------------------------------------ warp tiles of groups
// The fake-quant prepass and pack walk the weights in warp tiles of whole groups.
// A warp first issues the loads of its tile (16-byte loads; lane l takes the
// 16-weight chunks l, l + 32, ..., so every load instruction is coalesced), then
// forms the constants of each group of the tile once, one lane per group (s,
// RN(1/s), zr and the near band), in its own slice of shared memory, and then
// decides every weight from them.  Warps never wait for one another.
//
// A chunk with a weight near a rounding boundary (with min-max init steps, ties of
// W/s are common: bf16 weights and their group's range) is queued and redone
// later with the weights reloaded, 32 chunks at a time, so that the exact
// decisions run on full warps instead of holding up every lane of a warp for one.
constexpr int kTileThreads = 256;
constexpr int kTileWarps = kTileThreads / 32;
constexpr int kTileBlocksPerSm = 3;
// CPL: 16-weight chunks per lane and warp tile (two or three 16-byte loads each in
// flight per lane).  Three for bf16 weights in the prepass and in multi-layer pack;
// four in single-layer pack.  The choice is measured (70B block, w2g64): with four,
// the prepass and multi-layer pack spill a few registers at the 80 that three CTAs
// per SM allow and lose 2-4%; single-layer pack runs 3.5% faster with four.
template <typename T>
constexpr int kChunksPerLane = sizeof(T) == 2 ? 3 : 2;
template <typename T, int NL>
constexpr int kPackChunksPerLane = (sizeof(T) == 2 && NL == 1) ? 4 : kChunksPerLane<T>;
template <int CPL>
constexpr int kWarpTile = 32 * CPL * 16;  // weights; a multiple of every group size
template <int CPL>
constexpr int kWarpGroups = kWarpTile<CPL> / 32;  // groups of a tile at most (g = 32)
template <int CPL>
constexpr int kLaneGroups = (kWarpGroups<CPL> + 31) / 32;

struct GroupConst {
    float sc, rcp, zr, band;  // s, RN(1/s), zr, near band (below)
};

// 16 consecutive elements as stored.
template <typename T>
struct Raw16 {
    Raw8<T> a, b;
};
template <typename T>
__device__ __forceinline__ Raw16<T> load_raw16(const T *p) {
    return Raw16<T>{load_raw8<T>(p), load_raw8<T>(p + 8)};
}
template <typename T>
__device__ __forceinline__ void unpack16(const Raw16<T> &r, float (&w)[16]) {
    unpack8(r.a, *reinterpret_cast<float(*)[8]>(&w[0]));
    unpack8(r.b, *reinterpret_cast<float(*)[8]>(&w[8]));
}

// Band around the half-integers inside which the fast decision of a weight is not
// trusted, one per group: |RN(w RN(1/s)) - RN(w / s)| < |u| 2^-22, and a weight
// whose code is not clamped has |u| <= |zr| + Q + 1/2, so a band of half-width
// (|zr| + Q + 1) 2^-21 (twice the bound) covers every such weight; a clamped code
// (or mask) does not change when round(u) is off by one.  A group with |zr| near
// 2^20 or beyond gets a band that takes every weight to the exact decision.
__device__ __forceinline__ float near_band(float zr, float Q) {
    return __fsub_rn(0.5f, __fmul_rn(__fadd_rn(__fadd_rn(fabsf(zr), Q), 1.0f), 0x1p-21f));
}

// Fast decisions for two weights at once: u = RN(w RN(1/s)) and v = RN(u + M + zr)
// - (M + zr) = round(u), exact for |u| < 2^22 (beyond that the code is clamped
// whatever v is), and r = u - v.  A tie of u has |r| = 1/2, inside every band.
__device__ __forceinline__ void pair_decision(uint64_t w2, uint64_t rcp2, uint64_t mz2, uint64_t &u2, uint64_t &v2,
                                              float &ra, float &rb) {
    u2 = f2_mul(w2, rcp2);
    v2 = f2_sub(f2_add(u2, mz2), mz2);
    f2_unpack(f2_sub(u2, v2), ra, rb);
}

// round(RN(w / s)) for one weight, without the division in the usual case.  With
// u = RN(w RN(1/s)), |w/s - u| < |u| 2^-22 < 2^-8 for |u| < 2^14:
// - u at least 2^-7 from every half-integer: w/s and RN(w/s) round as u does;
// - otherwise let h be that half-integer and e = fma(-h, s, w), the rounded
//   w - h s (its sign is exact).  T = s sp / 2, with sp the spacing of fp32 next
//   to h on the side of w/s (the side of e; half the spacing above |h| on the
//   side toward zero when |h| = 1/2, a power of two), is a power-of-two multiple
//   of s and exact.  RN is monotone and T representable, so |e| < T proves
//   |w/s - h| < sp / 2: RN(w/s) = h, which rounds half to even; |e| > T proves
//   RN(w/s) != h, on the side of e, which rounds to that side's integer.  The
//   IEEE division decides what is left (|e| = T, a tiny s, a large u).
__device__ __forceinline__ float exact_round(float w, float s, float u) {
    if (fabsf(u) < 0x1p14f) {
        const float v = rint_small(u);
        const float r = __fsub_rn(u, v);
        if (fabsf(r) < 0.5f - 0x1p-7f) return v;
        const float h = __fadd_rn(v, copysignf(0.5f, r));
        const float e = __fmaf_rn(-h, s, w);
        const float p = __int_as_float((__float_as_int(h) & 0x7F800000) - (24 << 23));  // half the spacing above |h|
        float T = __fmul_rn(s, p);
        if (fabsf(h) == 0.5f && ((e > 0.0f) != (h > 0.0f))) T = __fmul_rn(0.5f, T);
        if (T >= 0x1p-100f) {  // a normal T is the exact product
            const float ae = fabsf(e);
            if (ae < T) return rint_small(h);
            if (ae > T) return e > 0.0f ? __fadd_rn(h, 0.5f) : __fsub_rn(h, 0.5f);
        }
    }
    return __fadd_rn(rintf(__fdiv_rn(w, s)), 0.0f);  // round(-0.3) = +0, as the other branches give
}

// The constants of the groups of one warp tile: lane l takes groups l, l + 32.
// With clamp_z (pack) zr = zq = clamp(round(z), 0, Q), written to zq here.
template <int CPL>
__device__ __forceinline__ void tile_group_consts(const float *__restrict__ s, const float *__restrict__ z,
                                                  int64_t e_tile, int64_t n, int gshift, float Q, bool clamp_z,
                                                  int lane, GroupConst *gc, uint8_t *__restrict__ zq) {
    const int gpt = kWarpTile<CPL> >> gshift;
    const int64_t g0 = e_tile >> gshift, n_groups = n >> gshift;
#pragma unroll
    for (int k = 0; k < kLaneGroups<CPL>; ++k) {
        const int gi = lane + 32 * k;
        const int64_t g = g0 + gi;
        if (gi < gpt && g < n_groups) {
            const float sc = __ldg(s + g);
            float zr = rintf(__ldg(z + g));
            if (clamp_z) zr = fminf(fmaxf(zr, 0.0f), Q);
            if (zq) zq[g] = static_cast<uint8_t>(zr);
            gc[gi] = GroupConst{sc, __frcp_rn(sc), zr, near_band(zr, Q)};
        }
    }
}

// A chunk left for the exact pass: where it starts (the layer in the top byte)
// and its group's constants.
struct PendingChunk {
    int64_t e0;
    GroupConst c;
};
constexpr int kLayerShift = 56;
// Per warp: fewer than 32 entries wait between tiles, and a tile adds at most one
// per chunk.
template <int CPL>
constexpr int kQueue = 32 + 32 * CPL;

// Walks the warp tiles: chunk(w, group constants, e0, exact) handles the 16
// weights at e0 and returns true when the fast pass (exact = false) left one of
// them near a rounding boundary.  Such chunks go to the warp's queue in shared
// memory; every 32 of them are redone with exact = true, one per lane, with the
// weights reloaded, and the rest at the end.
//
// The tiles are numbered through NL weight matrices in order (NL = 1, or the
// linears of a block in one launch); chunk() also receives the layer.
template <typename T, int NL>
struct TileLayers {
    const T *W[NL];
    const float *s[NL];
    const float *z[NL];
    uint8_t *zq[NL];     // pack: zq out (NULL otherwise)
    uint8_t *codes[NL];  // pack: codes out
    int64_t n[NL];
    int32_t tile_end[NL];  // warp tiles of layers 0..i (< 2^31); entries past the last layer repeat it
};

template <typename T, bool CLAMP_Z, int NL, int CPL, typename Chunk>
__device__ __forceinline__ void walk_warp_tiles(const TileLayers<T, NL> &L, int gshift, float Q,
                                                GroupConst *gc_all, PendingChunk *queue_all, Chunk chunk) {
    constexpr int WT = kWarpTile<CPL>;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    GroupConst *gc = gc_all + wib * kWarpGroups<CPL>;
    PendingChunk *queue = queue_all + wib * kQueue<CPL>;
    int queued = 0;  // warp-uniform
    // tile indices: 32-bit with several layers (fewer live registers), 64-bit with one
    using TI = std::conditional_t<(NL > 1), int32_t, int64_t>;
    const TI n_tiles = NL > 1 ? L.tile_end[NL - 1] : (L.n[0] + WT - 1) / WT;
    const TI stride = static_cast<TI>(gridDim.x) * kTileWarps;
    int li = 0;
    for (TI tile = static_cast<TI>(blockIdx.x) * kTileWarps + wib; tile < n_tiles; tile += stride) {
        if constexpr (NL > 1) {
            while (tile >= L.tile_end[li]) ++li;
        }
        const T *__restrict__ W = L.W[li];
        const int64_t n = L.n[li];
        const int64_t e_tile = static_cast<int64_t>(NL > 1 && li > 0 ? tile - L.tile_end[li > 0 ? li - 1 : 0] : tile) * WT;
        const bool last_tile = tile + stride >= n_tiles;
        // A whole tile (every tile but the last of the layer) runs without bounds
        // checks.
        const bool whole = e_tile + WT <= n;
        Raw16<T> raw[CPL];
        if (whole) {
#pragma unroll
            for (int j = 0; j < CPL; ++j) raw[j] = load_raw16<T>(W + e_tile + (j * 32 + lane) * 16);
        } else {
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                const int64_t e0 = e_tile + (j * 32 + lane) * 16;
                if (e0 < n) raw[j] = load_raw16<T>(W + e0);
            }
        }
        __syncwarp();  // the previous tile's reads of gc are done
        tile_group_consts<CPL>(L.s[li], L.z[li], e_tile, n, gshift, Q, CLAMP_Z, lane, gc, L.zq[li]);
        __syncwarp();
        uint32_t pending = 0u;  // bit j: chunk j left for the exact pass
        auto fast_pass = [&](auto whole_tag) {
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                const int off = (j * 32 + lane) * 16;
                if (decltype(whole_tag)::value || e_tile + off < n) {
                    float w[16];
                    unpack16(raw[j], w);
                    if (chunk(w, gc[off >> gshift], e_tile + off, false, li)) pending |= 1u << j;
                }
            }
        };
        if (whole)
            fast_pass(std::true_type{});
        else
            fast_pass(std::false_type{});
        if (__any_sync(0xffffffffu, pending != 0u)) {
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                const int off = (j * 32 + lane) * 16;
                const bool p = (pending >> j) & 1u;
                const uint32_t ballot = __ballot_sync(0xffffffffu, p);
                if (p)
                    queue[queued + __popc(ballot & ((1u << lane) - 1u))] = PendingChunk{
                        NL > 1 ? (e_tile + off) | (static_cast<int64_t>(li) << kLayerShift) : e_tile + off,
                        gc[off >> gshift]};
                queued += __popc(ballot);
            }
        }
        // every 32 queued chunks, and the rest after the warp's last tile: the last
        // `count` entries, one per lane
        while (queued >= 32 || (last_tile && queued > 0)) {
            const int count = queued < 32 ? queued : 32;
            __syncwarp();
            if (lane < count) {
                const PendingChunk pc = queue[queued - count + lane];
                const int pl = NL > 1 ? static_cast<int>(pc.e0 >> kLayerShift) : 0;
                const int64_t e0 = NL > 1 ? pc.e0 & ((int64_t{1} << kLayerShift) - 1) : pc.e0;
                float w[16];
                unpack16(load_raw16<T>(L.W[pl] + e0), w);
                (void)chunk(w, pc.c, e0, true, pl);
            }
            queued -= count;
            __syncwarp();
        }
    }
}

template <int CPL>
__host__ __device__ __forceinline__ int64_t warp_tiles(int64_t n) {
    return (n + kWarpTile<CPL> - 1) / kWarpTile<CPL>;
}

template <int CPL>
int tile_grid(int64_t n, const DeviceInfo &dev, int64_t tiles = -1) {
    if (tiles < 0) tiles = warp_tiles<CPL>(n);
    const int64_t blocks = (tiles + kTileWarps - 1) / kTileWarps;
    return static_cast<int>(
        std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(dev.sm_count) * kTileBlocksPerSm)));
}

// ------------------------------------------------------------------ fake-quant prepass
// W-hat = (clamp(round(W/s) + zr, 0, Q) - zr) s = clamp(round(W/s), -zr, Q - zr) s
// (all integer-valued until the one rounded product), with the code and the
// straight-through mask 0 <= round(W/s) + zr <= Q when asked for.
template <typename O, bool CODES, bool V8>
__device__ __forceinline__ bool fake_quant_chunk(const float (&w)[16], const GroupConst &c, float Q, int64_t e0,
                                                 bool exact, O *__restrict__ W_hat, uint8_t *__restrict__ code,
                                                 uint8_t *__restrict__ mask) {
    const float mz = __fadd_rn(kRoundMagic, c.zr);
    const uint64_t rcp2 = f2_pack(c.rcp, c.rcp), mz2 = f2_pack(mz, mz);
    float v[16];
    bool near = false;
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
        uint64_t u2, v2;
        float ra, rb;
        pair_decision(f2_pack(w[j], w[j + 1]), rcp2, mz2, u2, v2, ra, rb);
        f2_unpack(v2, v[j], v[j + 1]);
        if (exact) {
            float ua, ub;
            f2_unpack(u2, ua, ub);
            if (fabsf(ra) >= c.band) v[j] = exact_round(w[j], c.sc, ua);
            if (fabsf(rb) >= c.band) v[j + 1] = exact_round(w[j + 1], c.sc, ub);
        } else {
            near |= fabsf(ra) >= c.band;
            near |= fabsf(rb) >= c.band;
        }
    }
    if (near) return true;
    // 0 - zr, not -zr: a clamped code of a group with zr = 0 gives W-hat = +0, as
    // (c - zr) s does
    const float vlo = __fsub_rn(0.0f, c.zr), vhi = __fsub_rn(Q, c.zr);
    uint32_t mbits[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        if (CODES) mbits[j / 4] |= ((v[j] >= vlo) && (v[j] <= vhi) ? 1u : 0u) << (8 * (j % 4));
        v[j] = fminf(fmaxf(v[j], vlo), vhi);
    }
    if (W_hat) {
        const uint64_t s2 = f2_pack(c.sc, c.sc);
        float wh[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2) f2_unpack(f2_mul(f2_pack(v[j], v[j + 1]), s2), wh[j], wh[j + 1]);
        store16<O, V8>(W_hat + e0, wh);
    }
    if (CODES) {
        // code = v + zr: the low byte of M + zr + v (exact)
        uint32_t cbits[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
            float a, b;
            f2_unpack(f2_add(f2_pack(v[j], v[j + 1]), mz2), a, b);
            cbits[j / 4] |= (static_cast<uint32_t>(__float_as_int(a)) & 0xFFu) << (8 * (j % 4));
            cbits[j / 4] |= (static_cast<uint32_t>(__float_as_int(b)) & 0xFFu) << (8 * (j % 4 + 1));
        }
        if (code) *reinterpret_cast<uint4 *>(code + e0) = make_uint4(cbits[0], cbits[1], cbits[2], cbits[3]);
        if (mask) *reinterpret_cast<uint4 *>(mask + e0) = make_uint4(mbits[0], mbits[1], mbits[2], mbits[3]);
    }
    return false;
}

// V8: W_hat is 32-byte aligned (whole-sector stores).
template <typename T, typename O, bool CODES, bool V8>
__global__ void __launch_bounds__(kTileThreads, kTileBlocksPerSm)
    k_fake_quant(const T *__restrict__ W, const float *__restrict__ s, const float *__restrict__ z, int64_t n,
                 int gshift, float Q, O *__restrict__ W_hat, uint8_t *__restrict__ code,
                 uint8_t *__restrict__ mask) {
    begin_dependent();
    constexpr int CPL = kChunksPerLane<T>;
    __shared__ GroupConst gc[kTileWarps * kWarpGroups<CPL>];
    __shared__ PendingChunk queue[kTileWarps * kQueue<CPL>];
    TileLayers<T, 1> L;
    L.W[0] = W;
    L.s[0] = s;
    L.z[0] = z;
    L.zq[0] = nullptr;
    L.codes[0] = nullptr;
    L.n[0] = n;
    L.tile_end[0] = static_cast<int32_t>(warp_tiles<CPL>(n));
    walk_warp_tiles<T, false, 1, CPL>(L, gshift, Q, gc, queue,
                                 [&](const float (&w)[16], const GroupConst &c, int64_t e0, bool exact, int) {
                                     return fake_quant_chunk<O, CODES, V8>(w, c, Q, e0, exact, W_hat, code, mask);
                                 });
}

// ------------------------------------------------------------------ pack
// Codes of 16 weights of one group into their packed words (2-bit: one word,
// code k at bits 2k; 4-bit: two words, 4k; 3-bit: four words, one code per
// byte).  zr := zq = clamp(round(z), 0, Q) (z hard-rounded at pack time).
//
// Two codes per f16x2 word: 1024 + zr + round(u) is an integer that f16 holds
// exactly, so after a clamp of both halves to [1024, 1024 + Q] the low bits of
// each half are the code.  The weights of a pair sit 16 bits apart in their
// packed word (k and k + 8 for 2-bit codes, k and k + 4 for 4-bit, k and k + 2
// for 3-bit), so one shifted add places both; the bits of 1024 are taken out
// once per word at the end.
template <int BITS>
struct PackLayout {
    static constexpr int kSlot = BITS == 3 ? 8 : BITS;  // bits per code in a word
    static constexpr int kPerWord = 32 / kSlot;
    static constexpr int kWords = 16 / kPerWord;
    static constexpr int kHalf = kPerWord / 2;  // pair partner distance
};

// sum over i < count of bits(f16 1024, twice) << (step i), modulo 2^32.
__host__ __device__ constexpr uint32_t magic_h2_word(int step, int count) {
    uint32_t acc = 0;
    for (int i = 0; i < count; ++i) acc += 0x64006400u << (step * i);
    return acc;
}

template <int BITS>
__device__ __forceinline__ bool pack_chunk(const float (&w)[16], const GroupConst &c, float Q, int64_t e0,
                                           bool exact, uint8_t *__restrict__ codes) {
    using L = PackLayout<BITS>;
    const float mz = __fadd_rn(kRoundMagic, c.zr), zk = __fadd_rn(c.zr, 1024.0f);
    const uint64_t rcp2 = f2_pack(c.rcp, c.rcp), mz2 = f2_pack(mz, mz), zk2 = f2_pack(zk, zk);
    const uint32_t lo2 = 0x64006400u;  // f16 1024 in both halves
    const uint32_t qh = 0x6400u + static_cast<uint32_t>(Q);
    const uint32_t hi2 = qh | (qh << 16);
    uint32_t word[4];
    bool near = false;
#pragma unroll
    for (int m = 0; m < L::kWords; ++m) {
        uint32_t acc = 0u;
#pragma unroll
        for (int i = 0; i < L::kHalf; ++i) {
            const int a = m * L::kPerWord + i, b = a + L::kHalf;
            uint64_t u2, v2;
            float ra, rb;
            pair_decision(f2_pack(w[a], w[b]), rcp2, mz2, u2, v2, ra, rb);
            if (exact) {
                float ua, ub, va, vb;
                f2_unpack(u2, ua, ub);
                f2_unpack(v2, va, vb);
                if (fabsf(ra) >= c.band) va = exact_round(w[a], c.sc, ua);
                if (fabsf(rb) >= c.band) vb = exact_round(w[b], c.sc, ub);
                v2 = f2_pack(va, vb);
            } else {
                near |= fabsf(ra) >= c.band;
                near |= fabsf(rb) >= c.band;
            }
            float ea, eb;
            f2_unpack(f2_add(v2, zk2), ea, eb);
            acc += h2_clamp(h2_from_f32(ea, eb), lo2, hi2) << (L::kSlot * i);
        }
        word[m] = acc - magic_h2_word(L::kSlot, L::kHalf);
    }
    if (near) return true;
    if (BITS == 2) {
        *reinterpret_cast<uint32_t *>(codes + e0 / 4) = word[0];
    } else if (BITS == 4) {
        *reinterpret_cast<uint2 *>(codes + e0 / 2) = make_uint2(word[0], word[1]);
    } else {
        *reinterpret_cast<uint4 *>(codes + e0) = make_uint4(word[0], word[1], word[2], word[3]);
    }
    return false;
}

template <typename T, int BITS, int NL>
__global__ void __launch_bounds__(kTileThreads, kTileBlocksPerSm)
    k_pack(const __grid_constant__ TileLayers<T, NL> L, int gshift, float Q) {
    begin_dependent();
    constexpr int CPL = kPackChunksPerLane<T, NL>;
    __shared__ GroupConst gc[kTileWarps * kWarpGroups<CPL>];
    __shared__ PendingChunk queue[kTileWarps * kQueue<CPL>];
    // Several layers: the table goes to shared memory, where a layer's entries are
    // read per tile instead of being held in registers.
    if constexpr (NL > 1) {
        __shared__ TileLayers<T, NL> Ls;
        constexpr int kWords = sizeof(TileLayers<T, NL>) / 8;
        for (int i = threadIdx.x; i < kWords; i += kTileThreads)
            reinterpret_cast<uint64_t *>(&Ls)[i] = reinterpret_cast<const uint64_t *>(&L)[i];
        __syncthreads();
        walk_warp_tiles<T, true, NL, CPL>(Ls, gshift, Q, gc, queue,
                                          [&](const float (&w)[16], const GroupConst &c, int64_t e0, bool exact,
                                              int li) { return pack_chunk<BITS>(w, c, Q, e0, exact, Ls.codes[li]); });
    } else {
        walk_warp_tiles<T, true, 1, CPL>(L, gshift, Q, gc, queue,
                                         [&](const float (&w)[16], const GroupConst &c, int64_t e0, bool exact, int) {
                                             return pack_chunk<BITS>(w, c, Q, e0, exact, L.codes[0]);
                                         });
    }
}

// ------------------------------------------------------------------ E2E dequant
// One thread per 16 consecutive codes: W-hat = (W_q - zq) s (Eq. 2).  A code and
// zq enter fp32 as the raw bits of M + code and M + zq (exact), so W_q - zq is
// one subtraction and W-hat one rounded product, two weights per instruction.
template <int BITS>
__device__ __forceinline__ void codes16_magic(const uint8_t *codes, int64_t e0, float (&f)[16]) {
    constexpr uint32_t kM = 0x4B400000u;  // bits of M = 1.5 * 2^23
    if (BITS == 2) {
        const uint32_t word = __ldg(reinterpret_cast<const uint32_t *>(codes + e0 / 4));
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = __uint_as_float(((word >> (2 * j)) & 3u) | kM);
    } else if (BITS == 4) {
        const uint2 r = __ldg(reinterpret_cast<const uint2 *>(codes + e0 / 2));
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = __uint_as_float(((r.x >> (4 * j)) & 15u) | kM);
#pragma unroll
        for (int j = 0; j < 8; ++j) f[8 + j] = __uint_as_float(((r.y >> (4 * j)) & 15u) | kM);
    } else {
        const uint4 r = __ldg(reinterpret_cast<const uint4 *>(codes + e0));
        const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = __uint_as_float(((w4[j / 4] >> (8 * (j % 4))) & 0xFFu) | kM);
    }
}

__device__ __forceinline__ float step_value(const float *s, int64_t g) { return __ldg(s + g); }
__device__ __forceinline__ float step_value(const __half *s, int64_t g) { return __half2float(__ldg(s + g)); }

// S: fp32 step sizes, or fp16 ones (fp16 step-size storage), widened exactly.
// V8: W_hat is 32-byte aligned (whole-sector stores).
template <int BITS, typename O, typename S, bool V8>
__global__ void __launch_bounds__(kThreads)
    k_dequant(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ zq,
              const S *__restrict__ s, int64_t n_chunks, int gshift, O *__restrict__ W_hat) {
    begin_dependent();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n_chunks;
         i += stride) {
        const int64_t e0 = i * 16;
        const int64_t g = e0 >> gshift;
        const float sc = step_value(s, g);
        const float mz = __uint_as_float(static_cast<uint32_t>(__ldg(zq + g)) | 0x4B400000u);  // M + zq
        float f[16];
        codes16_magic<BITS>(codes, e0, f);
        const uint64_t mz2 = f2_pack(mz, mz), s2 = f2_pack(sc, sc);
        float wh[16];
#pragma unroll
        for (int j = 0; j < 16; j += 2)
            f2_unpack(f2_mul(f2_sub(f2_pack(f[j], f[j + 1]), mz2), s2), wh[j], wh[j + 1]);
        store16<O, V8>(W_hat + e0, wh);
    }
}

// Layers per multi-layer launch (a Llama block has seven linears); more are
// launched in batches of this many.
constexpr int kMultiLayers = 8;

// One launch over layers a[0..n) (1 <= n <= NL, every layer non-empty).
template <typename T, int G, int NL>
cudaError_t minmax_launch(const QuantLayerArgs *a, int n, float Q, const DeviceInfo &dev, cudaStream_t st) {
    InitLayers<T, NL> L{};
    int64_t units = 0, weights = 0;
    for (int i = 0; i < NL; ++i) {
        const QuantLayerArgs &x = a[i < n ? i : n - 1];
        const int64_t ng = x.N * (x.K / G);
        L.W[i] = static_cast<const T *>(x.W);
        L.s[i] = x.s_out;
        L.z[i] = x.z_out;
        L.n_groups[i] = ng;
        if (i < n) {
            units += (ng + kInitUnit<G> - 1) / kInitUnit<G>;
            weights += ng * G;
        }
        L.unit_end[i] = units;
    }
    return launch_pdl(k_minmax_init<T, G, NL>, dim3(grid_for(weights, dev, 8 * 4)), dim3(kThreads), 0, st, L, Q);
}

template <typename T, int NL>
cudaError_t minmax_dispatch(const QuantLayerArgs *a, int n, int group, float Q, const DeviceInfo &dev,
                            cudaStream_t st) {
    switch (group) {
        case 32: return minmax_launch<T, 32, NL>(a, n, Q, dev, st);
        case 64: return minmax_launch<T, 64, NL>(a, n, Q, dev, st);
        case 128: return minmax_launch<T, 128, NL>(a, n, Q, dev, st);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, int NL>
cudaError_t pack_dispatch(const QuantLayerArgs *a, int n, int bits, int group, const DeviceInfo &dev,
                          cudaStream_t st) {
    TileLayers<T, NL> L{};
    int64_t tiles = 0;
    for (int i = 0; i < NL; ++i) {
        const QuantLayerArgs &x = a[i < n ? i : n - 1];
        L.W[i] = static_cast<const T *>(x.W);
        L.s[i] = x.s;
        L.z[i] = x.z;
        L.zq[i] = x.zq;
        L.codes[i] = x.codes;
        L.n[i] = x.N * x.K;
        if (i < n) tiles += warp_tiles<kPackChunksPerLane<T, NL>>(x.N * x.K);
        if (tiles > INT32_MAX) return cudaErrorInvalidValue;  // beyond any device memory
        L.tile_end[i] = static_cast<int32_t>(tiles);
    }
    const int gshift = group_shift(group);
    const int grid = tile_grid<kPackChunksPerLane<T, NL>>(0, dev, tiles);
    const float Q = static_cast<float>((1 << bits) - 1);
    switch (bits) {
        case 2: return launch_pdl(k_pack<T, 2, NL>, dim3(grid), dim3(kTileThreads), 0, st, L, gshift, Q);
        case 3: return launch_pdl(k_pack<T, 3, NL>, dim3(grid), dim3(kTileThreads), 0, st, L, gshift, Q);
        case 4: return launch_pdl(k_pack<T, 4, NL>, dim3(grid), dim3(kTileThreads), 0, st, L, gshift, Q);
        default: return cudaErrorInvalidValue;
    }
}

// Drops empty layers, then one launch per kMultiLayers layers (single-layer
// kernels for one layer).
template <typename Launch>
cudaError_t for_layer_batches(const QuantLayerArgs *layers, int n, Launch launch) {
    QuantLayerArgs batch[kMultiLayers];
    int m = 0;
    for (int i = 0; i < n; ++i) {
        if (layers[i].N * layers[i].K == 0) continue;
        batch[m++] = layers[i];
        if (m == kMultiLayers || i == n - 1) {
            const cudaError_t e = launch(batch, m);
            if (e != cudaSuccess) return e;
            m = 0;
        }
    }
    return m ? launch(batch, m) : cudaSuccess;
}

template <typename O, typename S, bool V8>
cudaError_t dequant_dispatch_v(const uint8_t *codes, const uint8_t *zq, const S *s, int64_t n,
                               int bits, int group, O *W_hat, const DeviceInfo &dev,
                               cudaStream_t st) {
    const int gshift = group_shift(group);
    const int64_t chunks = n / 16;
    const int grid = grid_for(chunks, dev);
    switch (bits) {
        case 2: return launch_pdl(k_dequant<2, O, S, V8>, dim3(grid), dim3(kThreads), 0, st, codes, zq, s, chunks, gshift, W_hat);
        case 3: return launch_pdl(k_dequant<3, O, S, V8>, dim3(grid), dim3(kThreads), 0, st, codes, zq, s, chunks, gshift, W_hat);
        case 4: return launch_pdl(k_dequant<4, O, S, V8>, dim3(grid), dim3(kThreads), 0, st, codes, zq, s, chunks, gshift, W_hat);
        default: return cudaErrorInvalidValue;
    }
}

inline bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

template <typename O, typename S>
cudaError_t dequant_dispatch(const uint8_t *codes, const uint8_t *zq, const S *s, int64_t n,
                             int bits, int group, O *W_hat, const DeviceInfo &dev,
                             cudaStream_t st) {
    if (aligned32(W_hat)) return dequant_dispatch_v<O, S, true>(codes, zq, s, n, bits, group, W_hat, dev, st);
    return dequant_dispatch_v<O, S, false>(codes, zq, s, n, bits, group, W_hat, dev, st);
}

}  // namespace

cudaError_t launch_minmax_init_multi(const QuantLayerArgs *layers, int n, bool w_f32, int bits, int group,
                                     const DeviceInfo &dev, cudaStream_t st) {
    const float Q = static_cast<float>((1 << bits) - 1);
    return for_layer_batches(layers, n, [&](const QuantLayerArgs *b, int m) {
        using bf = __nv_bfloat16;
        if (m == 1)
            return w_f32 ? minmax_dispatch<float, 1>(b, 1, group, Q, dev, st)
                         : minmax_dispatch<bf, 1>(b, 1, group, Q, dev, st);
        return w_f32 ? minmax_dispatch<float, kMultiLayers>(b, m, group, Q, dev, st)
                     : minmax_dispatch<bf, kMultiLayers>(b, m, group, Q, dev, st);
    });
}

cudaError_t launch_minmax_init(const void *W, bool w_f32, int64_t N, int64_t K, int bits, int group,
                               float *s, float *z, const DeviceInfo &dev, cudaStream_t st) {
    QuantLayerArgs a{};
    a.W = W;
    a.s_out = s;
    a.z_out = z;
    a.N = N;
    a.K = K;
    return launch_minmax_init_multi(&a, 1, w_f32, bits, group, dev, st);
}

cudaError_t launch_fake_quant(const void *W, bool w_f32, const float *s, const float *z, int64_t N,
                              int64_t K, int bits, int group, void *W_hat, bool out_f32,
                              uint8_t *code, uint8_t *mask, const DeviceInfo &dev,
                              cudaStream_t st) {
    const int64_t n = N * K;
    if (n == 0) return cudaSuccess;
    if (warp_tiles<kChunksPerLane<float>>(n) > INT32_MAX) return cudaErrorInvalidValue;  // beyond any memory
    const float Q = static_cast<float>((1 << bits) - 1);
    using bf = __nv_bfloat16;
    const bool codes = code || mask;
    const int gshift = group_shift(group);
    const bool v8 = aligned32(W_hat);
#define EQAT_FQ_LAUNCH_V(TW, TO, CODES, V8)                                                                  \
    launch_pdl(k_fake_quant<TW, TO, CODES, V8>, dim3(tile_grid<kChunksPerLane<TW>>(n, dev)), dim3(kTileThreads), 0, \
               st, static_cast<const TW *>(W), s, z, n, gshift, Q, static_cast<TO *>(W_hat), code, mask)
#define EQAT_FQ_LAUNCH(TW, TO)                                                                              \
    (codes && v8 ? EQAT_FQ_LAUNCH_V(TW, TO, true, true)                                                     \
     : codes     ? EQAT_FQ_LAUNCH_V(TW, TO, true, false)                                                    \
     : v8        ? EQAT_FQ_LAUNCH_V(TW, TO, false, true)                                                    \
                 : EQAT_FQ_LAUNCH_V(TW, TO, false, false))
    cudaError_t e;
    if (w_f32 && out_f32)
        e = EQAT_FQ_LAUNCH(float, float);
    else if (w_f32)
        e = EQAT_FQ_LAUNCH(float, bf);
    else if (out_f32)
        e = EQAT_FQ_LAUNCH(bf, float);
    else
        e = EQAT_FQ_LAUNCH(bf, bf);
#undef EQAT_FQ_LAUNCH
#undef EQAT_FQ_LAUNCH_V
    return e;
}

cudaError_t launch_pack_multi(const QuantLayerArgs *layers, int n, bool w_f32, int bits, int group,
                              const DeviceInfo &dev, cudaStream_t st) {
    return for_layer_batches(layers, n, [&](const QuantLayerArgs *b, int m) {
        using bf = __nv_bfloat16;
        if (m == 1)
            return w_f32 ? pack_dispatch<float, 1>(b, 1, bits, group, dev, st)
                         : pack_dispatch<bf, 1>(b, 1, bits, group, dev, st);
        return w_f32 ? pack_dispatch<float, kMultiLayers>(b, m, bits, group, dev, st)
                     : pack_dispatch<bf, kMultiLayers>(b, m, bits, group, dev, st);
    });
}

cudaError_t launch_pack(const void *W, bool w_f32, const float *s, const float *z, int64_t N,
                        int64_t K, int bits, int group, uint8_t *codes, uint8_t *zq,
                        const DeviceInfo &dev, cudaStream_t st) {
    QuantLayerArgs a{};
    a.W = W;
    a.s = s;
    a.z = z;
    a.codes = codes;
    a.zq = zq;
    a.N = N;
    a.K = K;
    return launch_pack_multi(&a, 1, w_f32, bits, group, dev, st);
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
