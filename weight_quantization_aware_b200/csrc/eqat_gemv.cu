// Batch-1..8 inference on frozen codes (E2E-QP forward at decode sizes):
//   Y[m, n] = sum_k X[m, k] (W_q[n, k] - zq[n, g]) s[n, g]
// (zhaoyang97 ACL2025 notes, Eq. 2; modelfoundations note, Phase 2: only
// dequantization is left in the graph), read straight from the packed codes.
//
// At M <= 8 the layer is bound by HBM: 2-bit codes are 0.25 B per weight plus
// 5/g B of s and zq, against 2 B per weight for a bf16 matrix.  The codes are
// streamed once and W-hat is never formed in memory:
//   - in k_dq_gemv a producer warp moves 128-row x 128-byte code tiles into a
//     shared-memory ring with TMA (128-byte swizzle, so the per-lane reads hit
//     distinct banks).  The B-operand fragments of mma.sync m16n8k16 (X permuted
//     and pre-scaled to match the A registers below) and the per-group sums that
//     remove the conversion offset and the zero point come in one of two ways:
//     in build mode the producer warp copies the stage's columns of X with the
//     code tile and turns them into fragments and sums two stages later; in
//     fragment mode k_gemv_xprep writes them for all of K beforehand (one more
//     dependent launch, no per-stage work) and the stages copy their slices;
//   - eight consumer warps each own 16 rows.  A lane turns 16 codes of a row into
//     eight bf16x2 registers with one AND-OR per register (the "magic number"
//     conversion: code bits placed in the mantissa of 128.0 give 128 + code * 4^j
//     exactly) and feeds them to mma.sync as the A operand:
//       sum_k (c_k - zq) x_k = [sum_k (128 + c_k 4^j) (x_k 4^-j)] - xoff_g - zq xsum_g.
//   - the eight mma columns carry (group slot, token) pairs: with M padded to a
//     power of two MP, SL = 8 / MP consecutive groups of a stage (at most the
//     stage's group count) accumulate side by side in the same registers, each
//     in its own columns, so the per-group correction above, the accumulator
//     reset and the s / zq reads run once per SL groups.  At M = 1 that is once
//     per stage instead of once per group.
// The tensor core is only a multiply-add engine for register-resident operands;
// the roofline is HBM.
//
// Work: the stages (row tile, 128-byte column slab) in row-major order are split
// into equal contiguous ranges, one per CTA, so each CTA streams along K of the
// same rows (whole DRAM pages, s / zq sectors reused at once).  A CTA writes one
// fp32 partial per row tile it touches; k_gemv_reduce sums the partials of each
// row tile in CTA order (deterministic).  Layers with few row tiles (build mode)
// instead give each row tile a cluster of C CTAs that split its K range; the
// CTAs leave their partials in shared memory and the cluster's rank 0 sums them in
// rank order through distributed shared memory and writes Y: one kernel per call.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>

#include "eqat_internal.h"
#include "eqat_pdl.cuh"
#include "eqat_ptx.cuh"

namespace eqat {
namespace {

constexpr int kConsumers = 8;              // consumer warps, 16 rows each
constexpr int kRows = 16 * kConsumers;     // rows of a tile
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kRowBytes = 128;             // code bytes of one row per TMA box
constexpr int kMaxSets = 8;                // 64-column sets per stage, at most (2-bit)
constexpr int kMaxGps = 8;                 // groups per stage, at most (2-bit, g = 64)
constexpr int kTableSlice = kMaxSets * 1024;  // B fragments of one stage
constexpr int kXoSlice = kMaxGps * 64;        // {xoff, xsum} x 8 tokens of one stage
constexpr int kXSlice = 8 * 512 * 2;          // the stage's columns of X, 8 tokens (2-bit: 512 columns)
constexpr int kSlots = 2;                  // s / zq staging slots per consumer warp
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr int kSzBytes = kConsumers * kSlots * 16 * kMaxGps * 8;

// Codes of one lane for one 64-column set of a row: 16 codes (columns 16t..16t+15
// of the set).  extract() produces eight bf16x2 registers; register e holds codes
// lo(e) (low half) and hi(e) (high half), scaled by 4^scale_exp(e), plus 128.
constexpr uint32_t kMagic = 0x43004300u;  // bf16x2 {128.0, 128.0}

// (w & MASK) | magic in one logic op (truth table 0xEA = (a & b) | c).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t w, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "r"(magic));
    return d;
}

template <int BITS>
struct Codes;

// 2-bit: one 32-bit word, code q at bits 2q.  Only mantissa bits 0..5 of each
// half are usable, so three codes per half are taken per shift.
template <>
struct Codes<2> {
    static constexpr int kBytes = 4;         // per lane per set
    static constexpr int kCodeBits = 2;
    __device__ static void extract(const uint32_t *w, uint32_t (&a)[8], uint32_t mg) {
        const uint32_t w0 = w[0], w6 = w[0] >> 6, w12 = w[0] >> 12;
        a[0] = and_or<0x00030003u>(w0, mg);
        a[1] = and_or<0x000C000Cu>(w0, mg);
        a[2] = and_or<0x00300030u>(w0, mg);
        a[3] = and_or<0x00030003u>(w6, mg);
        a[4] = and_or<0x000C000Cu>(w6, mg);
        a[5] = and_or<0x00300030u>(w6, mg);
        a[6] = and_or<0x00030003u>(w12, mg);
        a[7] = and_or<0x000C000Cu>(w12, mg);
    }
    __host__ __device__ static constexpr int lo(int e) { return e; }
    __host__ __device__ static constexpr int hi(int e) { return e + 8; }
    __host__ __device__ static constexpr int scale_exp(int e) { return e % 3; }
    // scale exponent of the code at position q (0..15) of the lane's 16
    __host__ __device__ static constexpr int pos_exp(int q) { return (q % 8) % 3; }
};

// 4-bit: two words, code q at bits 4(q % 8) of word q / 8.
template <>
struct Codes<4> {
    static constexpr int kBytes = 8;
    static constexpr int kCodeBits = 4;
    __device__ static void extract(const uint32_t *w, uint32_t (&a)[8], uint32_t mg) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const uint32_t v = w[p];
            a[4 * p + 0] = and_or<0x000F000Fu>(v, mg);
            a[4 * p + 1] = and_or<0x000F000Fu>(v >> 4, mg);
            a[4 * p + 2] = and_or<0x000F000Fu>(v >> 8, mg);
            a[4 * p + 3] = and_or<0x000F000Fu>(v >> 12, mg);
        }
    }
    __host__ __device__ static constexpr int lo(int e) { return e < 4 ? e : e + 4; }
    __host__ __device__ static constexpr int hi(int e) { return lo(e) + 4; }
    __host__ __device__ static constexpr int scale_exp(int) { return 0; }
    __host__ __device__ static constexpr int pos_exp(int) { return 0; }
};

// 3-bit codes stored one per byte: four words, byte q = code q.  Seven mantissa
// bits are taken so that any byte below 128 converts exactly.
template <>
struct Codes<3> {
    static constexpr int kBytes = 16;
    static constexpr int kCodeBits = 8;
    __device__ static void extract(const uint32_t *w, uint32_t (&a)[8], uint32_t mg) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            a[2 * p] = and_or<0x007F007Fu>(w[p], mg);
            a[2 * p + 1] = and_or<0x007F007Fu>(w[p] >> 8, mg);
        }
    }
    __host__ __device__ static constexpr int lo(int e) { return 4 * (e / 2) + (e % 2); }
    __host__ __device__ static constexpr int hi(int e) { return lo(e) + 2; }
    __host__ __device__ static constexpr int scale_exp(int) { return 0; }
    __host__ __device__ static constexpr int pos_exp(int) { return 0; }
};

// Codes per stage along K: one 128-byte row segment.
// Code bytes of one row per stage: one 128-byte TMA box for 2-bit codes (eight
// 64-column sets), two for 4-bit codes and for 3-bit codes (stored one per byte),
// so that a stage holds eight or four sets and its fixed cost is shared.
template <int BITS>
constexpr int stage_row_bytes() {
    return BITS == 2 ? kRowBytes : 2 * kRowBytes;
}

template <int BITS>
constexpr int stage_codes() {
    return stage_row_bytes<BITS>() * 8 / Codes<BITS>::kCodeBits;
}

// A stage slot: codes (one 128-row x 128-byte swizzled tile per box) | fragments |
// group sums | (build mode) X columns.  Codes at the start of a slot: 1024-byte
// aligned for the 128-byte swizzle.  The ring has as many slots as fit in shared
// memory next to the s / zq slots: six, or five / four for the two-tile stages.
template <int BITS>
constexpr int kCodeTile = kRows * stage_row_bytes<BITS>();
template <int BITS>
constexpr int kOffTable = kCodeTile<BITS>;
template <int BITS>
constexpr int kOffXo = kOffTable<BITS> + kTableSlice;
template <int BITS>
constexpr int kOffX = kOffXo<BITS> + kXoSlice;
template <int BITS, bool BUILD>
constexpr int kStageBytes = (kOffX<BITS> + (BUILD ? kXSlice : 0) + 1023) / 1024 * 1024;
template <int BITS, bool BUILD>
constexpr int kStages = BITS == 2 ? 6 : (BUILD ? 4 : 5);
// Shared-memory layout (after 1024-byte alignment): the stage ring, then the
// s / zq slots, then the barriers (full, empty, X-arrived per slot, abort flag).
template <int BITS, bool BUILD>
constexpr int kOffSz = kStages<BITS, BUILD> * kStageBytes<BITS, BUILD>;
template <int BITS, bool BUILD>
constexpr int kOffBar = kOffSz<BITS, BUILD> + kSzBytes;
template <int BITS, bool BUILD>
constexpr int kSmemBytes = 1024 + kOffBar<BITS, BUILD> + 256;

// Byte `byte` of row r of a stage's code tiles (box byte / 128, 128-byte swizzle).
template <int BITS>
__device__ __forceinline__ uint32_t code_offset(int r, int byte) {
    return static_cast<uint32_t>((byte >> 7) * (kRows * kRowBytes) + r * kRowBytes +
                                 ((((byte >> 4) & 7) ^ (r & 7)) << 4) + (byte & 15));
}


// Contiguous global -> shared copy whose completion is counted on `bar` (both
// addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

struct GemvParams {
    const uint8_t *zq;
    const void *s;
    const __nv_bfloat16 *X;  // [M][K]
    const uint4 *table;  // fragment mode only: B fragments of X from k_gemv_xprep, [sets_pad][2][32]
    const float2 *xso;   // fragment mode only: {xoff, xsum}, [groups_pad][8 tokens]
    float *partials;     // [row_tiles][maxseg][M][kRows]
    __nv_bfloat16 *Y;    // cluster mode: written by each cluster's rank 0
    int clu;             // cluster mode: CTAs per row tile (the cluster size)
    int M, N, G;
    int64_t K;
    int spr;             // stages per row tile (along K)
    int row_tiles;
    int maxseg;          // partial slots per row tile
    int vec;             // s / zq rows allow vector loads (G a multiple of the per-thread run)
    int64_t total_stages;
    int *err;
    uint64_t wait_limit_ns;
};

// The CTA whose stage range holds stage x, for ranges [c S / grid, (c+1) S / grid).
__host__ __device__ __forceinline__ int cta_of_stage(int64_t x, int64_t S, int grid) {
    return static_cast<int>(((x + 1) * grid - 1) / S);
}


// Stage x = rt * spr + ks, advanced without divisions.
struct StageCursor {
    int64_t x;
    int rt, ks;
    __device__ __forceinline__ void init(int64_t x0, int spr) {
        x = x0;
        rt = static_cast<int>(x0 / spr);
        ks = static_cast<int>(x0 - static_cast<int64_t>(rt) * spr);
    }
    __device__ __forceinline__ void next(int spr) {
        ++x;
        if (++ks == spr) {
            ks = 0;
            ++rt;
        }
    }
};

// The stage's mma fragments (the B operand) and group sums from its columns of
// X, by the 32 lanes of the producer warp.  Fragment column n = lane / 4 is
// (slot n / MPC, token n % MPC), MPC = 8 / SL.  Lane (n, t) writes the entries of
// the sets of the groups of its slot (the group's index within the stage, modulo
// SL), built from columns 16t .. 16t + 15 of each set: the same entries that lane
// reads as a consumer.  Entry (set m, ip) holds registers e = 4 ip .. 4 ip + 3, and
// register e pairs columns lo(e) (low half) and hi(e), scaled by 4^-scale_exp(e).
// The four lanes of a quad then add up the group's sums: xsum = sum x and
// xoff = sum 128 4^-j x (j the exponent of the column's code position).  Entries
// of the other slots, and of tokens beyond M, stay zero (set once).  Columns at or
// beyond kcols (the end of K) read as zero; kcols is a multiple of 64.
template <int BITS, int GROUP, int SL>
__device__ __forceinline__ void build_stage(uint8_t *slot, int M, int kcols, int lane) {
    using C = Codes<BITS>;
    constexpr int KS = stage_codes<BITS>();
    constexpr int SPG = GROUP / 64;
    constexpr int GPS = KS / GROUP;
    constexpr int MPC = 8 / SL;
    const int n = lane >> 2, t = lane & 3;
    const int sl = n / MPC, tok = n % MPC;
    uint4 *table = reinterpret_cast<uint4 *>(slot + kOffTable<BITS>);
    float2 *xo = reinterpret_cast<float2 *>(slot + kOffXo<BITS>);
    const uint4 *xs = reinterpret_cast<const uint4 *>(slot + kOffX<BITS>);  // [token][KS] bf16
#pragma unroll
    for (int i = 0; i < GPS / SL; ++i) {
        const int gs = sl + SL * i;
        float xsum = 0.0f, xoff = 0.0f;
#pragma unroll
        for (int q = 0; q < SPG; ++q) {
            const int m = gs * SPG + q;
            const int c0 = 64 * m + 16 * t;  // the lane's first column in the stage
            uint32_t xw[8];                  // word k: columns c0 + 2k (low half), c0 + 2k + 1
            if (tok < M && c0 < kcols) {
                const uint4 a = xs[(tok * KS + c0) / 8], b = xs[(tok * KS + c0) / 8 + 1];
                xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
                xw[4] = b.x; xw[5] = b.y; xw[6] = b.z; xw[7] = b.w;
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) xw[k] = 0u;
            }
            uint32_t r[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int lo = C::lo(e), hi = C::hi(e);
                // bytes of column lo for the low half, of column hi for the high half
                const uint32_t sel = (2u * (lo & 1)) | ((2u * (lo & 1) + 1u) << 4) | ((4u + 2u * (hi & 1)) << 8) |
                                     ((5u + 2u * (hi & 1)) << 12);
                uint32_t v = __byte_perm(xw[lo >> 1], xw[hi >> 1], sel);
                if (C::scale_exp(e) != 0) {
                    const __nv_bfloat162 f = __float2bfloat162_rn(C::scale_exp(e) == 1 ? 0.25f : 0.0625f);
                    __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&v);
                    h = __hmul2(h, f);
                    v = *reinterpret_cast<const uint32_t *>(&h);
                }
                r[e] = v;
            }
            table[(m * 2 + 0) * 32 + lane] = make_uint4(r[0], r[1], r[2], r[3]);
            table[(m * 2 + 1) * 32 + lane] = make_uint4(r[4], r[5], r[6], r[7]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float x0 = __uint_as_float(xw[k] << 16), x1 = __uint_as_float(xw[k] & 0xFFFF0000u);
                constexpr float kw[3] = {128.0f, 32.0f, 8.0f};
                xsum += x0;
                xsum += x1;
                xoff = fmaf(x0, kw[C::pos_exp(2 * k)], xoff);
                xoff = fmaf(x1, kw[C::pos_exp(2 * k + 1)], xoff);
            }
        }
        xsum += __shfl_xor_sync(0xffffffffu, xsum, 1);
        xsum += __shfl_xor_sync(0xffffffffu, xsum, 2);
        xoff += __shfl_xor_sync(0xffffffffu, xoff, 1);
        xoff += __shfl_xor_sync(0xffffffffu, xoff, 2);
        if (t == 0 && tok < M) xo[gs * 8 + tok] = make_float2(xoff, xsum);
    }
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// X -> B fragments and per-group sums, for the whole of K (padded with zeros to
// whole stages).  One block per group, GROUP threads.  Thread i builds entry
// (set j, ip, l) of the group's sets = {mma 2ip: b0b1, b2b3; mma 2ip+1: b0b1,
// b2b3} for token l / 4 and column quad l % 4 (b0b1 of mma i pair with A register
// 2i: columns lo, hi scaled by 4^-scale_exp; b2b3 with register 2i + 1).  It also
// reads column i of the group for the 8 tokens, and the block sums them into
// xoff = sum 128 x 4^-j and xsum = sum x per token.
//
// Column n of the fragments is (slot n / MPC, token n % MPC), MPC = 8 / slots:
// a set's entries are nonzero only in the columns of its group's slot (the
// group's index within its stage, modulo `slots`).
template <int BITS, int GROUP>
__global__ void __launch_bounds__(GROUP) k_gemv_xprep(const __nv_bfloat16 *__restrict__ X, int M, int64_t K,
                                                        int slots, uint4 *__restrict__ table,
                                                        float2 *__restrict__ xso) {
    using C = Codes<BITS>;
    constexpr int WARPS = GROUP / 32;
    __shared__ float red[WARPS][16];
    // the workspace may still be read by the preceding call's kernels
    pdl_wait();
    pdl_allow_dependents();
    const int gidx = blockIdx.x;
    auto xv = [&](int tok, int64_t k) -> float {
        return (tok < M && k < K) ? __bfloat162float(X[static_cast<int64_t>(tok) * K + k]) : 0.0f;
    };
    {
        const int j = gidx * (GROUP / 64) + (threadIdx.x >> 6);
        const int ip = (threadIdx.x >> 5) & 1, l = threadIdx.x & 31;
        const int n = l >> 2, t = l & 3;
        const int mpc = 8 / slots;
        const int gs = (j % (stage_codes<BITS>() / 64)) / (GROUP / 64);  // the set's group within its stage
        const int tok = (n / mpc == gs % slots) ? n % mpc : 8;           // 8: no token, zeros
        const int64_t kb = 64 * static_cast<int64_t>(j) + 16 * t;
        uint32_t r[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
                const int e = 2 * (2 * ip + h) + sl;
                const float sc = (C::scale_exp(e) == 0) ? 1.0f : (C::scale_exp(e) == 1 ? 0.25f : 0.0625f);
                r[2 * h + sl] = bf16x2_bits(xv(tok, kb + C::lo(e)) * sc, xv(tok, kb + C::hi(e)) * sc);
            }
        }
        table[(static_cast<int64_t>(j) * 2 + ip) * 32 + l] = make_uint4(r[0], r[1], r[2], r[3]);
    }
    // column sums
    const int64_t k = static_cast<int64_t>(gidx) * GROUP + threadIdx.x;
    const int ex = C::pos_exp(threadIdx.x & 15);
    const float w = ex == 0 ? 128.0f : (ex == 1 ? 32.0f : 8.0f);
    float so[8], ss[8];
#pragma unroll
    for (int tok = 0; tok < 8; ++tok) {
        ss[tok] = xv(tok, k);
        so[tok] = ss[tok] * w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int tok = 0; tok < 8; ++tok) {
            ss[tok] += __shfl_xor_sync(0xffffffffu, ss[tok], off);
            so[tok] += __shfl_xor_sync(0xffffffffu, so[tok], off);
        }
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int tok = 0; tok < 8; ++tok) {
            red[warp][tok] = so[tok];
            red[warp][8 + tok] = ss[tok];
        }
    }
    __syncthreads();
    if (threadIdx.x < 8) {
        float a = 0.0f, b = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < WARPS; ++w2) {
            a += red[w2][threadIdx.x];
            b += red[w2][8 + threadIdx.x];
        }
        xso[static_cast<int64_t>(gidx) * 8 + threadIdx.x] = make_float2(a, b);
    }
}

// s and zq of one stage (128 rows x GPS groups), four values per consumer thread
// at most, loaded into registers two stages ahead of their use.  The registers
// hold the raw bits; they are converted only when stored to shared memory, so
// that nothing waits for the loads before then.
struct SzRegs {
    uint32_t s[4];  // fp32 value v in word v, or fp16 value v in half v % 2 of word v / 2
    uint32_t z;     // zq value v in byte v
};

// Each consumer warp stages the s and zq of its own 16 rows: lane l takes row
// l / 2 and VPT = GPS / 2 consecutive groups (GPS = 1: lanes 0..15, one each).
// When the row strides allow it (p.vec: G a multiple of VPT) and the stage lies
// inside K, s and zq come in one vector load each.
template <int BITS, int GROUP>
struct SzShape {
    static constexpr int GPS = stage_codes<BITS>() / GROUP;
    static constexpr int VPT = GPS >= 2 ? GPS / 2 : 1;
    static constexpr int TPR = GPS >= 2 ? 2 : 1;  // lanes per row
};

template <int BITS, int GROUP, bool S16>
__device__ __forceinline__ void load_sz(const GemvParams &p, const StageCursor &c, int64_t x_end, int row0,
                                        int lane, SzRegs &r) {
    using Sh = SzShape<BITS, GROUP>;
    constexpr int VPT = Sh::VPT, TPR = Sh::TPR;
#pragma unroll
    for (int v = 0; v < 4; ++v) r.s[v] = 0u;
    r.z = 0u;
    const int row = lane / TPR, part = lane % TPR;
    if (c.x >= x_end || row >= 16) return;
    const int64_t n = static_cast<int64_t>(c.rt) * kRows + row0 + row;
    const int64_t g = static_cast<int64_t>(c.ks) * Sh::GPS + part * VPT;
    if (n >= p.N) return;
    const int64_t i = n * p.G + g;
    const uint32_t *s32 = static_cast<const uint32_t *>(p.s);
    const unsigned short *s16 = static_cast<const unsigned short *>(p.s);
    if (p.vec && g + VPT <= p.G) {
        if (VPT == 4) {
            if (S16) {
                const uint2 h = __ldg(reinterpret_cast<const uint2 *>(s16 + i));
                r.s[0] = h.x;
                r.s[1] = h.y;
            } else {
                const uint4 f = __ldg(reinterpret_cast<const uint4 *>(s32 + i));
                r.s[0] = f.x;
                r.s[1] = f.y;
                r.s[2] = f.z;
                r.s[3] = f.w;
            }
            r.z = __ldg(reinterpret_cast<const uint32_t *>(p.zq + i));
        } else if (VPT == 2) {
            if (S16) {
                r.s[0] = __ldg(reinterpret_cast<const uint32_t *>(s16 + i));
            } else {
                const uint2 f = __ldg(reinterpret_cast<const uint2 *>(s32 + i));
                r.s[0] = f.x;
                r.s[1] = f.y;
            }
            r.z = __ldg(reinterpret_cast<const unsigned short *>(p.zq + i));
        } else {
            r.s[0] = S16 ? static_cast<uint32_t>(__ldg(s16 + i)) : __ldg(s32 + i);
            r.z = __ldg(p.zq + i);
        }
        return;
    }
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
        if (g + v < p.G) {
            if (S16)
                r.s[v / 2] |= static_cast<uint32_t>(__ldg(s16 + i + v)) << (16 * (v % 2));
            else
                r.s[v] = __ldg(s32 + i + v);
            r.z |= static_cast<uint32_t>(__ldg(p.zq + i + v)) << (8 * v);
        }
    }
}

// Into the warp's slot, entry row * GPS + group (rows local to the warp).
template <int BITS, int GROUP, bool S16>
__device__ __forceinline__ void store_sz(float2 *slot, int lane, const SzRegs &r) {
    using Sh = SzShape<BITS, GROUP>;
    const int row = lane / Sh::TPR, part = lane % Sh::TPR;
    if (row >= 16) return;
    float2 *d = slot + row * Sh::GPS + part * Sh::VPT;
#pragma unroll
    for (int v = 0; v < Sh::VPT; ++v) {
        const float sv = S16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(r.s[v / 2] >> (16 * (v % 2)))))
                             : __uint_as_float(r.s[v]);
        d[v] = make_float2(sv, static_cast<float>((r.z >> (8 * v)) & 0xFFu));
    }
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with a zero accumulator in.
__device__ __forceinline__ void mma_bf16_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

template <int BITS>
__device__ __forceinline__ void load_codes(const uint8_t *tile, int row, int byte, uint32_t *w) {
    const uint8_t *ptr = tile + code_offset<BITS>(row, byte);
    if (Codes<BITS>::kBytes == 4) {
        w[0] = *reinterpret_cast<const uint32_t *>(ptr);
    } else if (Codes<BITS>::kBytes == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(ptr);
        w[0] = v.x;
        w[1] = v.y;
    } else {
        const uint4 v = *reinterpret_cast<const uint4 *>(ptr);
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
    }
}


// BUILD: the producer warp builds each stage's fragments from X (build mode);
// otherwise they come by bulk copy from the table of k_gemv_xprep (fragment mode).
// CLU: cluster mode (grid = row tiles x p.clu, one row tile per cluster).
template <int BITS, int GROUP, bool S16, int SL, bool BUILD, bool CLU>
__global__ void __launch_bounds__(kThreads, 1)
    k_dq_gemv(const __grid_constant__ CUtensorMap tm_codes, const GemvParams p) {
    using C = Codes<BITS>;
    constexpr int KS = stage_codes<BITS>();
    constexpr int SETS = KS / 64;                     // 64-column sets per stage
    constexpr int SET_BYTES = 64 * C::kCodeBits / 8;  // code bytes of a set in one row
    constexpr int SPG = GROUP / 64;                   // sets per group
    constexpr int GPS = KS / GROUP;                   // groups per stage
    constexpr int MPC = 8 / SL;  // token columns per slot
    static_assert(SL >= 1 && SL <= 8 && GPS % SL == 0, "slots divide the stage's groups");
    extern __shared__ uint8_t smem_raw[];
    // aligned by an offset from the array itself, so that every pointer below
    // stays in the shared window (shared loads, 32-bit addresses)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    constexpr int NST = kStages<BITS, BUILD>;
    constexpr int kSlot = kStageBytes<BITS, BUILD>;
    constexpr int kCT = kCodeTile<BITS>;
    constexpr int oTable = kOffTable<BITS>, oXo = kOffXo<BITS>, oX = kOffX<BITS>;
    float2 *sz = reinterpret_cast<float2 *>(smem + kOffSz<BITS, BUILD>);
    // Build mode: full[s] = the slot's fragments are built (the producer warp's 32
    // lanes), xfull[s] = its code tile and X columns have landed (transaction
    // bytes).  Fragment mode: full[s] = the code tile, fragments and sums have
    // landed (transaction bytes); xfull is unused.  empty[s]: the consumers are
    // done with the slot.
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kOffBar<BITS, BUILD>);
    uint64_t *empty = full + NST;
    uint64_t *xfull = empty + NST;
    // cluster mode: red_full (rank 0's) counts the consumer warps of the cluster whose
    // partials are in shared memory; red_done (each CTA's) rank 0's warps, once read
    uint64_t *red_full = xfull + NST;
    uint64_t *red_done = red_full + 1;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(red_done + 1);
    // the code tile of stage (ks, rt): one TMA box per 128 bytes of each row
    auto load_code_tile = [&](uint8_t *dst, uint64_t *bar, int ks, int rt) {
#pragma unroll
        for (int bx = 0; bx < stage_row_bytes<BITS>() / kRowBytes; ++bx)
            tma_load_2d(dst + bx * (kRows * kRowBytes), &tm_codes, bar, ks * stage_row_bytes<BITS>() + bx * kRowBytes,
                        rt * kRows);
    };
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], BUILD ? 32 : 1);
            mbar_init(&empty[i], kConsumers);
            mbar_init(&xfull[i], 1);
        }
        if (CLU) {
            mbar_init(red_full, kConsumers * p.clu);
            mbar_init(red_done, kConsumers);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tm_codes);
        pdl_allow_dependents();
    }
    if constexpr (BUILD) {
        // fragment entries that no stage writes (other slots, tokens beyond M) are zero
        for (int s = 0; s < NST; ++s) {
            uint4 *z = reinterpret_cast<uint4 *>(smem + s * kSlot + oTable);
            for (int i = threadIdx.x; i < (kTableSlice + kXoSlice) / 16; i += kThreads)
                z[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __syncthreads();
    if constexpr (CLU) cluster_sync();  // every CTA's barriers exist before any remote arrival
    // Build mode: X, the codes, s and zq may come from the preceding kernel.  In
    // fragment mode the preceding kernel is k_gemv_xprep, which waited for them;
    // the producer waits for k_gemv_xprep itself (below).
    if constexpr (BUILD) pdl_wait();

    const int64_t S = p.total_stages;
    const int64_t x_begin = static_cast<int64_t>(blockIdx.x) * S / gridDim.x;
    const int64_t x_end = static_cast<int64_t>(blockIdx.x + 1) * S / gridDim.x;

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        if constexpr (!BUILD) {
            // Fragment mode: one elected lane requests each stage's code tile (TMA)
            // and its slices of the fragment table and the group sums (bulk copies) on
            // full[s].  The code tiles do not depend on X: the first ring's worth is
            // requested before waiting for the preceding k_gemv_xprep.
            if (elect_one_sync()) {
                uint32_t armed = 0, armed_parity = 0;
                bool ok = true;
                uint32_t it = 0;
                StageCursor c;
                c.init(x_begin, p.spr);
                constexpr uint32_t kFragBytes = SETS * 1024 + GPS * 64;
                const int pre = static_cast<int>(x_end - x_begin < NST ? x_end - x_begin : NST);
                {
                    StageCursor cp = c;
                    for (int i = 0; i < pre; ++i, cp.next(p.spr)) {
                        mbar_arrive_expect_tx(&full[i], kCT + kFragBytes);
                        load_code_tile(smem + i * kSlot, &full[i], cp.ks, cp.rt);
                    }
                    armed = (1u << pre) - 1u;  // parity 0
                }
                pdl_wait();
                for (; static_cast<int>(it) < pre; c.next(p.spr), ++it) {
                    uint8_t *stage = smem + it * kSlot;
                    bulk_load(stage + oTable, p.table + static_cast<int64_t>(c.ks) * SETS * 64, SETS * 1024,
                              &full[it]);
                    bulk_load(stage + oXo, p.xso + static_cast<int64_t>(c.ks) * GPS * 8, GPS * 64, &full[it]);
                }
                for (; c.x < x_end; c.next(p.spr), ++it) {
                    const int st = it % NST;
                    const uint32_t ph = (it / NST) & 1u;
                    if (!mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *stage = smem + st * kSlot;
                    mbar_arrive_expect_tx(&full[st], kCT + kFragBytes);
                    armed |= 1u << st;
                    armed_parity = (armed_parity & ~(1u << st)) | (ph << st);
                    load_code_tile(stage, &full[st], c.ks, c.rt);
                    bulk_load(stage + oTable, p.table + static_cast<int64_t>(c.ks) * SETS * 64, SETS * 1024,
                              &full[st]);
                    bulk_load(stage + oXo, p.xso + static_cast<int64_t>(c.ks) * GPS * 8, GPS * 64, &full[st]);
                }
                if (!ok) {
                    // let issued copies land before the block can exit
                    for (int st = 0; st < NST; ++st)
                        if (armed & (1u << st)) {
                            const uint32_t a = smem_u32(&full[st]);
                            const uint64_t t0 = globaltimer_ns();
                            while (!mbar_try_wait(a, (armed_parity >> st) & 1u) &&
                                   globaltimer_ns() - t0 < 100000000ull) {
                            }
                        }
                }
            }
            __syncwarp();
            return;
        }
        // Build mode: lane 0 requests each stage's code tile (TMA) and the stage's
        // columns of X (one bulk copy per token) on xfull[s].  kLag stages behind,
        // the whole warp turns those columns into the stage's fragments and group
        // sums and arrives on full[s].  In the steady state the consumers are
        // NST - 1 stages behind the requests, so each stage is built well
        // before its use.
        uint32_t armed = 0, armed_parity = 0;
        bool ok = true;
        StageCursor ci, cb;
        ci.init(x_begin, p.spr);
        cb = ci;
        const int64_t n = x_end - x_begin;
        constexpr int kLag = 2;
        for (int64_t i = 0; i < n + kLag; ++i) {
            if (i < n) {
                const int st = static_cast<int>(i % NST);
                const uint32_t ph = static_cast<uint32_t>(i / NST) & 1u;
                ok = mbar_wait_bounded(&empty[st], ph ^ 1u, abort_flag, p.err, p.wait_limit_ns) && ok;
                if (!__all_sync(0xffffffffu, ok)) break;
                if (lane == 0) {
                    const int64_t k0 = static_cast<int64_t>(ci.ks) * KS;
                    const uint32_t xbytes = static_cast<uint32_t>((p.K - k0 < KS ? p.K - k0 : KS) * 2);
                    uint8_t *stage = smem + st * kSlot;
                    mbar_arrive_expect_tx(&xfull[st], kCT + p.M * xbytes);
                    armed |= 1u << st;
                    armed_parity = (armed_parity & ~(1u << st)) | (ph << st);
                    load_code_tile(stage, &xfull[st], ci.ks, ci.rt);
                    for (int tok = 0; tok < p.M; ++tok)
                        bulk_load(stage + oX + tok * KS * 2, p.X + tok * p.K + k0, xbytes, &xfull[st]);
                }
                __syncwarp();
                ci.next(p.spr);
            }
            if (i >= kLag) {
                const int64_t b = i - kLag;
                const int st = static_cast<int>(b % NST);
                const uint32_t ph = static_cast<uint32_t>(b / NST) & 1u;
                ok = mbar_wait_bounded(&xfull[st], ph, abort_flag, p.err, p.wait_limit_ns) && ok;
                if (!__all_sync(0xffffffffu, ok)) break;
                const int64_t k0 = static_cast<int64_t>(cb.ks) * KS;
                build_stage<BITS, GROUP, SL>(smem + st * kSlot, p.M, static_cast<int>(p.K - k0 < KS ? p.K - k0 : KS),
                                             lane);
                mbar_arrive(&full[st]);
                cb.next(p.spr);
            }
        }
        if (!ok && lane == 0) {
            // let issued copies land before the block can exit
            for (int st = 0; st < NST; ++st)
                if (armed & (1u << st)) {
                    const uint32_t a = smem_u32(&xfull[st]);
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(a, (armed_parity >> st) & 1u) && globaltimer_ns() - t0 < 100000000ull) {
                    }
                }
        }
        __syncwarp();
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Lane (r0, t) holds the accumulators of rows row_a, row_b and columns 2t,
    // 2t + 1, i.e. slot slot0 with tokens tok0, tok0 + 1 (MPC >= 2), or slots
    // 2t, 2t + 1 of token 0 (MPC = 1).
    const int r0 = lane >> 2, t = lane & 3;
    const int row_a = warp * 16 + r0, row_b = row_a + 8;
    const int slot0 = (2 * t) / MPC, tok0 = (2 * t) % MPC;
    const uint32_t magic = kMagic;
    // this warp's s / zq slots: [kSlots][16 rows][GPS] float2
    float2 *szw = sz + warp * (kSlots * 16 * kMaxGps);

    // s / zq pipeline, per warp: stage x's values are loaded at the start of stage
    // x - 3 into one of three register sets and stored to the warp's slot at the
    // end of stage x - 1.
    SzRegs sa_, sb_, sc_;
    StageCursor cur, pf;
    cur.init(x_begin, p.spr);
    pf = cur;
    load_sz<BITS, GROUP, S16>(p, pf, x_end, warp * 16, lane, sa_);
    pf.next(p.spr);
    store_sz<BITS, GROUP, S16>(szw, lane, sa_);
    load_sz<BITS, GROUP, S16>(p, pf, x_end, warp * 16, lane, sb_);
    pf.next(p.spr);
    load_sz<BITS, GROUP, S16>(p, pf, x_end, warp * 16, lane, sc_);
    pf.next(p.spr);
    float y[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    bool ok = true;
    __syncwarp();

    uint32_t it = 0;
    auto stage = [&](SzRegs &load_into, const SzRegs &store_from) {
        load_sz<BITS, GROUP, S16>(p, pf, x_end, warp * 16, lane, load_into);
        pf.next(p.spr);
        const int st = it % NST;
        const uint32_t ph = (it / NST) & 1u;
        // build mode: the code tile (written by TMA), then the fragments (by the
        // producer warp); fragment mode: all of it by copies on full[st]
        if constexpr (BUILD) ok = mbar_wait_bounded(&xfull[st], ph, abort_flag, p.err, p.wait_limit_ns) && ok;
        ok = mbar_wait_bounded(&full[st], ph, abort_flag, p.err, p.wait_limit_ns) && ok;
        const uint8_t *tile = smem + st * kSlot;
        const uint4 *table = reinterpret_cast<const uint4 *>(tile + oTable);
        const float2 *xo = reinterpret_cast<const float2 *>(tile + oXo);
        const float2 *szs = szw + (it % kSlots) * (16 * kMaxGps);
        // Runs of SL groups: the four mmas of a set go to four accumulator chains,
        // and the run's groups share them (each in its own columns).
#pragma unroll
        for (int g0 = 0; g0 < GPS; g0 += SL) {
            float acc[4][4];
#pragma unroll
            for (int gs = 0; gs < SL; ++gs) {
#pragma unroll
                for (int q = 0; q < SPG; ++q) {
                    const int m = (g0 + gs) * SPG + q;
                    uint32_t wa[C::kBytes / 4], wb[C::kBytes / 4];
                    load_codes<BITS>(tile, row_a, m * SET_BYTES + t * C::kBytes, wa);
                    load_codes<BITS>(tile, row_b, m * SET_BYTES + t * C::kBytes, wb);
                    uint32_t ea[8], eb[8];
                    C::extract(wa, ea, magic);
                    C::extract(wb, eb, magic);
                    const uint4 b01 = table[(m * 2 + 0) * 32 + lane];
                    const uint4 b23 = table[(m * 2 + 1) * 32 + lane];
                    if (gs == 0 && q == 0) {
                        mma_bf16_z(acc[0], ea[0], eb[0], ea[1], eb[1], b01.x, b01.y);
                        mma_bf16_z(acc[1], ea[2], eb[2], ea[3], eb[3], b01.z, b01.w);
                        mma_bf16_z(acc[2], ea[4], eb[4], ea[5], eb[5], b23.x, b23.y);
                        mma_bf16_z(acc[3], ea[6], eb[6], ea[7], eb[7], b23.z, b23.w);
                    } else {
                        mma_bf16(acc[0], ea[0], eb[0], ea[1], eb[1], b01.x, b01.y);
                        mma_bf16(acc[1], ea[2], eb[2], ea[3], eb[3], b01.z, b01.w);
                        mma_bf16(acc[2], ea[4], eb[4], ea[5], eb[5], b23.x, b23.y);
                        mma_bf16(acc[3], ea[6], eb[6], ea[7], eb[7], b23.z, b23.w);
                    }
                }
            }
            float c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) c[i] = (acc[0][i] + acc[1][i]) + (acc[2][i] + acc[3][i]);
            // c = {row_a col 2t, row_a col 2t+1, row_b col 2t, row_b col 2t+1}
            if constexpr (MPC == 1) {
                // columns 2t, 2t + 1 are groups g0 + 2t, g0 + 2t + 1 of token 0
                const float4 sa = *reinterpret_cast<const float4 *>(szs + r0 * GPS + g0 + 2 * t);
                const float4 sb = *reinterpret_cast<const float4 *>(szs + (r0 + 8) * GPS + g0 + 2 * t);
                const float2 o0 = xo[(g0 + 2 * t) * 8], o1 = xo[(g0 + 2 * t + 1) * 8];
                y[0] = fmaf(sa.x, c[0] - fmaf(sa.y, o0.y, o0.x), y[0]);
                y[1] = fmaf(sa.z, c[1] - fmaf(sa.w, o1.y, o1.x), y[1]);
                y[2] = fmaf(sb.x, c[2] - fmaf(sb.y, o0.y, o0.x), y[2]);
                y[3] = fmaf(sb.z, c[3] - fmaf(sb.w, o1.y, o1.x), y[3]);
            } else {
                // both columns are group g0 + slot0; tokens tok0, tok0 + 1
                const float2 sa = szs[r0 * GPS + g0 + slot0], sb = szs[(r0 + 8) * GPS + g0 + slot0];
                const float4 o = *reinterpret_cast<const float4 *>(xo + (g0 + slot0) * 8 + tok0);
                y[0] = fmaf(sa.x, c[0] - fmaf(sa.y, o.y, o.x), y[0]);
                y[1] = fmaf(sa.x, c[1] - fmaf(sa.y, o.w, o.z), y[1]);
                y[2] = fmaf(sb.x, c[2] - fmaf(sb.y, o.y, o.x), y[2]);
                y[3] = fmaf(sb.x, c[3] - fmaf(sb.y, o.w, o.z), y[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);

        // s / zq of the next stage into its slot
        store_sz<BITS, GROUP, S16>(szw + ((it + 1) % kSlots) * (16 * kMaxGps), lane, store_from);

        const int rt = cur.rt;
        cur.next(p.spr);
        ++it;
        if (cur.x == x_end || cur.ks == 0) {
            // this CTA is done with row tile rt: its partial goes to slot
            // (rt, cta - first cta of rt).  The lanes of a quad that hold the
            // same tokens in different slots are summed first.
            float v[4] = {y[0], y[1], y[2], y[3]};
            if constexpr (MPC == 1) {
                v[0] += v[1];
                v[2] += v[3];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (MPC <= 2) {
                    v[i] += __shfl_xor_sync(0xffffffffu, v[i], 1);
                    v[i] += __shfl_xor_sync(0xffffffffu, v[i], 2);
                } else if (MPC == 4) {
                    v[i] += __shfl_xor_sync(0xffffffffu, v[i], 2);
                }
            }
            if constexpr (CLU) {
                // cluster mode (one row tile per CTA): into this warp's s / zq
                // area, which no stage reads any more: [token][16 rows]
                __syncwarp();
                float *Pw = reinterpret_cast<float *>(szw);
                if (slot0 == 0) {
                    const int m0 = tok0, m1 = tok0 + 1;
                    if (m0 < p.M) {
                        Pw[m0 * 16 + r0] = v[0];
                        Pw[m0 * 16 + r0 + 8] = v[2];
                    }
                    if (MPC > 1 && m1 < p.M) {
                        Pw[m1 * 16 + r0] = v[1];
                        Pw[m1 * 16 + r0 + 8] = v[3];
                    }
                }
            } else {
                const int seg = static_cast<int>(blockIdx.x) -
                                cta_of_stage(static_cast<int64_t>(rt) * p.spr, S, static_cast<int>(gridDim.x));
                float *P = p.partials + (static_cast<int64_t>(rt) * p.maxseg + seg) * p.M * kRows;
                if (slot0 == 0) {
                    const int m0 = tok0, m1 = tok0 + 1;
                    if (m0 < p.M) {
                        P[m0 * kRows + row_a] = v[0];
                        P[m0 * kRows + row_b] = v[2];
                    }
                    if (MPC > 1 && m1 < p.M) {
                        P[m1 * kRows + row_a] = v[1];
                        P[m1 * kRows + row_b] = v[3];
                    }
                }
            }
            y[0] = y[1] = y[2] = y[3] = 0.0f;
        }
        __syncwarp();  // the next stage's slot is written
    };
    while (cur.x < x_end) {
        stage(sa_, sb_);
        if (cur.x >= x_end) break;
        stage(sb_, sc_);
        if (cur.x >= x_end) break;
        stage(sc_, sa_);
    }
    if constexpr (CLU) {
        // Each warp's partial of this CTA's K range is in its s / zq area.  Rank 0's
        // warp w sums warp w's partials of the cluster's CTAs in rank order and
        // writes its 16 rows of Y; the other CTAs keep their shared memory until
        // rank 0 is done with it.
        const uint32_t rank = cluster_rank();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(map_to_rank(red_full, 0));
        if (rank == 0) {
            ok = mbar_wait_bounded<true>(red_full, 0, abort_flag, p.err, p.wait_limit_ns) && ok;
            if (__all_sync(0xffffffffu, ok)) {
                const int rt = static_cast<int>(x_begin / p.spr);
                const uint32_t base = smem_u32(szw);
                for (int i = lane; i < p.M * 16; i += 32) {
                    const int m = i >> 4, rr = i & 15;
                    float a = 0.0f;
                    for (int c = 0; c < p.clu; ++c) {
                        uint32_t addr;
                        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(base + 4u * i), "r"(c));
                        float v;
                        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
                        a += v;
                    }
                    const int n = rt * kRows + warp * 16 + rr;
                    if (n < p.N) p.Y[static_cast<int64_t>(m) * p.N + n] = __float2bfloat16_rn(a);
                }
            }
            __syncwarp();
            if (lane > 0 && lane < p.clu) mbar_arrive_cluster(map_to_rank(red_done, lane));
        } else {
            (void)mbar_wait_bounded<true>(red_done, 0, abort_flag, p.err, p.wait_limit_ns);
        }
    }
    (void)ok;
}

// Y[m][n] = sum over the CTAs that touched row tile n / kRows, in CTA order, of
// their partials.
__global__ void k_gemv_reduce(const float *__restrict__ partials, int M, int N, int spr, int maxseg,
                              int64_t S, int grid, __nv_bfloat16 *__restrict__ Y) {
    pdl_wait();  // the partials of the preceding k_dq_gemv
    pdl_allow_dependents();
    const int64_t MN = static_cast<int64_t>(M) * N;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < MN;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int m = static_cast<int>(i / N), n = static_cast<int>(i % N);
        const int rt = n / kRows, row = n % kRows;
        const int c0 = cta_of_stage(static_cast<int64_t>(rt) * spr, S, grid);
        const int c1 = cta_of_stage(static_cast<int64_t>(rt) * spr + spr - 1, S, grid);
        float a = 0.0f;
        for (int c = c0; c <= c1; ++c)
            a += partials[((static_cast<int64_t>(rt) * maxseg + (c - c0)) * M + m) * kRows + row];
        Y[i] = __float2bfloat16_rn(a);
    }
}

struct Plan {
    int spr, row_tiles, maxseg, grid;
    int64_t S;
    bool build;  // fragments built in the streaming kernel (else by k_gemv_xprep)
    int clu;     // build mode with few row tiles: CTAs per row tile (cluster), else 1
    size_t table_bytes, xso_bytes, partial_bytes;
};

// Build mode saves the k_gemv_xprep launch (about 2.4 us per call on B200) but
// puts the fragment build (work in proportion to M) on the producer warp's
// scheduler for every stage.  Measured, it pays for M = 1 below about 32 MB of
// codes, s and zq, and for M = 2 below about 8 MB; fragment mode elsewhere.
inline bool build_mode(int64_t M, int64_t N, int64_t K, int bits, int group) {
    const int64_t bytes = N * K * (bits == 3 ? 8 : bits) / 8 + N * (K / group) * 5;
    return (M == 1 && bytes <= (int64_t(32) << 20)) || (M == 2 && bytes <= (int64_t(8) << 20));
}

Plan make_plan(int64_t M, int64_t N, int64_t K, int bits, int group, int sms) {
    Plan pl{};
    const int ks = bits == 2 ? stage_codes<2>() : bits == 4 ? stage_codes<4>() : stage_codes<3>();
    pl.spr = static_cast<int>((K + ks - 1) / ks);
    pl.row_tiles = static_cast<int>((N + kRows - 1) / kRows);
    pl.S = static_cast<int64_t>(pl.spr) * pl.row_tiles;
    pl.grid = static_cast<int>(std::min<int64_t>(pl.S, sms));
    pl.maxseg = 1;
    for (int rt = 0; rt < pl.row_tiles; ++rt) {
        const int c0 = cta_of_stage(static_cast<int64_t>(rt) * pl.spr, pl.S, pl.grid);
        const int c1 = cta_of_stage(static_cast<int64_t>(rt) * pl.spr + pl.spr - 1, pl.S, pl.grid);
        pl.maxseg = std::max(pl.maxseg, c1 - c0 + 1);
    }
    pl.build = build_mode(M, N, K, bits, group);
    // Cluster mode: when two CTAs per row tile still fit on the SMs at once, each row
    // tile gets a cluster of C CTAs (a power of two, at most 8 and at most its stages)
    // and the partial sums never leave the chip: no second kernel.
    pl.clu = 1;
    if (pl.build && static_cast<int64_t>(pl.row_tiles) * 2 <= sms) {
        int c = 2;
        while (c * 2 <= 8 && c * 2 <= pl.spr && static_cast<int64_t>(pl.row_tiles) * c * 2 <= sms) c *= 2;
        if (c <= pl.spr) {
            pl.clu = c;
            pl.grid = pl.row_tiles * c;
            pl.maxseg = c;
        }
    }
    const int64_t sets = static_cast<int64_t>(pl.spr) * (ks / 64);
    const int64_t groups = static_cast<int64_t>(pl.spr) * (ks / group);
    pl.table_bytes = pl.build ? 0 : static_cast<size_t>(sets) * 1024;
    pl.xso_bytes = pl.build ? 0 : (static_cast<size_t>(groups) * 64 + 255) / 256 * 256;
    pl.partial_bytes = static_cast<size_t>(pl.row_tiles) * pl.maxseg * M * kRows * 4;
    return pl;
}

template <int BITS, int GROUP, bool S16, int SL, bool BUILD>
cudaError_t launch_main(const CUtensorMap &map, const GemvParams &p, int grid, int dev_id, cudaStream_t st) {
    if (BUILD && p.clu > 1) {
        auto kern = k_dq_gemv<BITS, GROUP, S16, SL, BUILD, true>;
        static std::atomic<uint64_t> done{0};
        const uint64_t bit = 1ull << (dev_id & 63);
        if (!(done.load() & bit)) {
            cudaError_t e =
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes<BITS, BUILD>);
            if (e != cudaSuccess) return e;
            done.fetch_or(bit);
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes<BITS, BUILD>;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(p.clu);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return cudaLaunchKernelEx(&cfg, kern, map, p);
    }
    auto kern = k_dq_gemv<BITS, GROUP, S16, SL, BUILD, false>;
    static std::atomic<uint64_t> done{0};
    const uint64_t bit = 1ull << (dev_id & 63);
    if (!(done.load() & bit)) {
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes<BITS, BUILD>);
        if (e != cudaSuccess) return e;
        done.fetch_or(bit);
    }
    return launch_pdl(kern, dim3(grid), dim3(kThreads), kSmemBytes<BITS, BUILD>, st, map, p);
}

template <int BITS, int GROUP, bool S16>
cudaError_t launch_slots(int slots, bool build, const CUtensorMap &map, const GemvParams &p, int grid, int dev_id,
                         cudaStream_t st) {
    constexpr int GPS = stage_codes<BITS>() / GROUP;
    constexpr int SL1 = GPS < 8 ? GPS : 8;  // slots at M = 1
    constexpr int SL2 = GPS < 4 ? GPS : 4;  // slots at M = 2
    if (build) {
        // build mode runs at M <= 2 only
        if (slots == SL1) return launch_main<BITS, GROUP, S16, SL1, true>(map, p, grid, dev_id, st);
        if constexpr (SL2 != SL1)
            if (slots == SL2) return launch_main<BITS, GROUP, S16, SL2, true>(map, p, grid, dev_id, st);
        return cudaErrorInvalidValue;
    }
    if (slots == 1) return launch_main<BITS, GROUP, S16, 1, false>(map, p, grid, dev_id, st);
    if constexpr (GPS >= 2)
        if (slots == 2) return launch_main<BITS, GROUP, S16, 2, false>(map, p, grid, dev_id, st);
    if constexpr (GPS >= 4)
        if (slots == 4) return launch_main<BITS, GROUP, S16, 4, false>(map, p, grid, dev_id, st);
    if constexpr (GPS >= 8)
        if (slots == 8) return launch_main<BITS, GROUP, S16, 8, false>(map, p, grid, dev_id, st);
    return cudaErrorInvalidValue;
}

// Slots per run: 8 / MP groups share the mma columns (MP = M rounded up to a
// power of two), at most the stage's groups.
inline int gemv_slots(int M, int gps) {
    const int mp = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
    return std::min(8 / mp, gps);
}

template <int BITS, int GROUP>
cudaError_t launch_all(const CUtensorMap &map, GemvParams p, const Plan &pl, bool s_f16, __nv_bfloat16 *Y,
                       const DeviceInfo &dev, cudaStream_t st) {
    constexpr int GPS = stage_codes<BITS>() / GROUP;
    const int slots = gemv_slots(p.M, GPS);
    if (!pl.build) {
        const int64_t groups = static_cast<int64_t>(pl.spr) * GPS;
        cudaError_t e = launch_pdl(k_gemv_xprep<BITS, GROUP>, dim3(static_cast<unsigned>(groups)), dim3(GROUP), 0,
                                   st, p.X, p.M, p.K, slots, const_cast<uint4 *>(p.table),
                                   const_cast<float2 *>(p.xso));
        if (e != cudaSuccess) return e;
    }
    p.clu = pl.clu;
    p.Y = Y;
    cudaError_t e = s_f16 ? launch_slots<BITS, GROUP, true>(slots, pl.build, map, p, pl.grid, dev.device, st)
                          : launch_slots<BITS, GROUP, false>(slots, pl.build, map, p, pl.grid, dev.device, st);
    if (e != cudaSuccess) return e;
    if (pl.clu > 1) return cudaSuccess;  // rank 0 of each cluster wrote Y
    const int64_t MN = static_cast<int64_t>(p.M) * p.N;
    const unsigned rblocks = static_cast<unsigned>(std::min<int64_t>((MN + 255) / 256, 2 * dev.sm_count));
    return launch_pdl(k_gemv_reduce, dim3(rblocks), dim3(256), 0, st, static_cast<const float *>(p.partials), p.M,
                      p.N, pl.spr, pl.maxseg, pl.S, pl.grid, Y);
}

}  // namespace

size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int group, int sm_count) {
    const Plan pl = make_plan(M, N, K, bits, group, sm_count);
    return pl.table_bytes + pl.xso_bytes + pl.partial_bytes;
}

size_t gemv_workspace_bound(int64_t M, int64_t N, int64_t K, int bits, int group) {
    // at most one CTA per stage, so at most S partial slots in all
    const Plan pl = make_plan(M, N, K, bits, group, 1);
    return pl.table_bytes + pl.xso_bytes + static_cast<size_t>(pl.S) * M * kRows * 4;
}

cudaError_t launch_dq_gemv(const void *X, const uint8_t *codes, const uint8_t *zq, const void *s, bool s_f16,
                           void *Y, int64_t M, int64_t N, int64_t K, int bits, int group, void *ws,
                           const DeviceInfo &dev, cudaStream_t st) {
    if (M < 1 || M > 8 || N <= 0 || K <= 0 || (group != 64 && group != 128)) return cudaErrorInvalidValue;
    if (bits != 2 && bits != 3 && bits != 4) return cudaErrorInvalidValue;
    if (N > INT32_MAX - kRows || K > INT32_MAX) return cudaErrorInvalidValue;
    const Plan pl = make_plan(M, N, K, bits, group, dev.sm_count);
    const int code_bits = bits == 3 ? 8 : bits;
    const uint64_t row_bytes = static_cast<uint64_t>(K) * code_bits / 8;
    CUtensorMap map;
    cudaError_t e = encode_map_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, row_bytes, static_cast<uint64_t>(N),
                                  row_bytes, kRowBytes, kRows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    uint8_t *w = static_cast<uint8_t *>(ws);
    GemvParams p{};
    p.zq = zq;
    p.s = s;
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.table = reinterpret_cast<const uint4 *>(w);
    p.xso = reinterpret_cast<const float2 *>(w + pl.table_bytes);
    p.partials = reinterpret_cast<float *>(w + pl.table_bytes + pl.xso_bytes);
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.G = static_cast<int>(K / group);
    p.K = K;
    p.spr = pl.spr;
    p.row_tiles = pl.row_tiles;
    p.maxseg = pl.maxseg;
    {
        const int gps = (bits == 2 ? stage_codes<2>() : bits == 4 ? stage_codes<4>() : stage_codes<3>()) / group;
        const int vpt = gps >= 2 ? gps / 2 : 1;
        p.vec = (p.G % vpt == 0) ? 1 : 0;
    }
    p.total_stages = pl.S;
    p.err = device_error_word();
    p.wait_limit_ns = kWaitLimitNs;
    __nv_bfloat16 *Yb = static_cast<__nv_bfloat16 *>(Y);
#define EQAT_GEMV_CASE(B, GR) \
    if (bits == B && group == GR) return launch_all<B, GR>(map, p, pl, s_f16, Yb, dev, st);
    EQAT_GEMV_CASE(2, 64)
    EQAT_GEMV_CASE(2, 128)
    EQAT_GEMV_CASE(3, 64)
    EQAT_GEMV_CASE(3, 128)
    EQAT_GEMV_CASE(4, 64)
    EQAT_GEMV_CASE(4, 128)
#undef EQAT_GEMV_CASE
    return cudaErrorInvalidValue;
}

}  // namespace eqat
