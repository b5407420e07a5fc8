// The three contractions of the fake-quantized linear layer on sm_100a tensor
// cores (tcgen05), with the straight-through and E2E-QP reductions fused into
// the epilogue:
//   forward        Y[M,N]  = X[M,K]  . W-hat[N,K]^T   A = X  (K-major), B = W-hat (K-major)
//   input grad     dX[M,K] = dY[M,N] . W-hat[N,K]     A = dY (K-major), B = W-hat (MN-major)
//   weight grad    dW-hat[N,K] = dY^T . X             A = dY (MN-major), B = X (MN-major)
// dW-hat stays in tensor memory: the epilogue turns it into dW (masked), ds and
// dz (Block-AP, paperlayer appendix A) or ds = sum dW-hat (W_q - zq) (E2E-QP,
// modelfoundations note Phase 2) and never writes it to HBM.
//
// Kernel structure (one CTA per SM, persistent over output tiles):
//   warp 0       TMA producer: 128x64 A and 256x64 B bf16 tiles, 128-byte
//                swizzle, into a 4-stage shared-memory ring (48 KB per stage)
//   warp 1       MMA issuer: one thread issues tcgen05.mma 128x256x16 into one
//                of two 256-column fp32 accumulators in tensor memory
//   warp 2       allocates / frees the 512 tensor-memory columns
//   warps 4..    epilogue: tcgen05.ld 32 columns at a time (thread i of warp w
//                owns accumulator row 32*(w%4)+i), then the fused epilogue
// The two accumulators let the epilogue of tile i overlap the main loop of
// tile i+1.  Every mbarrier wait is bounded (see eqat_ptx.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <queue>
#include <type_traits>
#include <utility>
#include <vector>

#include "eqat_internal.h"
#include "eqat_pdl.cuh"
#include "eqat_ptx.cuh"
#include "eqat_qmath.cuh"

namespace eqat {

__device__ int g_dev_error = 0;

namespace {

constexpr int BM = 128;
constexpr int BN = 256;  // widest N tile; a problem may use 128 (Prob::bn)
constexpr int BK = 64;  // one 128-byte swizzle row of bf16
constexpr int UK = 16;  // K of one tcgen05.mma kind::f16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int ACC_COLS = BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int MN_BOX = 64;                  // MN extent of one MN-major TMA box
constexpr int MN_BOX_BYTES = MN_BOX * 2 * BK;  // 64 columns x 64 k-rows of bf16
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s: far above any legitimate wait

// One contraction of a grouped launch.  Tiles of problem 0 come first in the
// global tile order, then those of problem 1.
struct Prob {
    int GM, GN, GK;
    int tiles_m, tiles_n, tile_begin, m_fast;
    int bn;  // N-tile width of this problem: 256 or 128
    int a_mn, b_mn;  // operand majorness (1 = MN-major)
    // epilogue
    void *out;
    int64_t ldo;
    const void *W;
    const float *s;
    const float *z;
    void *dW;
    float *ds;
    float *dz;
    const uint8_t *codes;
    const uint8_t *zq;
    const void *s_e2e;  // E2E step sizes (read for dz only), fp32 or fp16
    int s_f16;
    const void *target; // reconstruction target (bf16, row stride ldo)
    double *loss;
    float mse_scale;
    int clamp_pass;     // Block-AP: the clamp is straight-through as well
    int group;
    int gshift;  // log2(group)
    float Q;
    // B made on load from packed codes (pair kernel, CVT variants): W-hat [w_rows, w_cols]
    // = (W_q - zq) s, converted in shared memory from the code tile that B's tensor map
    // (then a map of the codes) brings in
    int b_cvt;
    int w_rows, w_cols, w_groups;
    const uint8_t *cvt_zq;
    const void *cvt_s;
    int cvt_s_f16;
};

struct KParams {
    Prob pr[2];
    int nprob;
    int total_tiles;
    int split_begin;  // pair kernel, one problem: tiles from here on are halves (-1: none)
    int *err;
    uint64_t wait_limit_ns;
    int cvt_cluster_scope;  // converter hand-off: release/acquire at cluster (1) or CTA (0) scope
};

// The tiles of a pair launch are dealt round-robin (pair q takes q, q + npairs, ...)
// unless the launch carries a TileSched: a host-made deal, pair q taking
// tile[begin[q] .. begin[q + 1]).  Used for grouped launches whose two problems
// have tiles of very different cost (a dW-hat contraction 2048 deep beside a dX
// contraction 8192-28672 deep), where round-robin leaves some pairs one long tile
// more than others and no fewer short ones.
constexpr int kSchedTiles = 8192;
constexpr int kSchedPairs = 128;
struct TileSched {
    uint16_t begin[kSchedPairs + 1];
    uint16_t tile[kSchedTiles];
};
struct NoSched {
    int unused;
};
template <int SCHED>
using SchedParam = typename std::conditional<SCHED != 0, TileSched, NoSched>::type;
// kernel parameters of a scheduled pair launch: six tensor maps, KParams, the deal
static_assert(6 * sizeof(CUtensorMap) + sizeof(KParams) + sizeof(TileSched) <= 32000,
              "a scheduled pair launch must fit the kernel-parameter limit");

// This pair's tiles: positions first, first + step, ... below end; tile_at maps a
// position to the tile.
template <int SCHED>
__device__ __forceinline__ void sched_range(const SchedParam<SCHED> &sc, int total_tiles, int pair, int npairs,
                                            int &first, int &end, int &step) {
    if constexpr (SCHED != 0) {
        first = sc.begin[pair];
        end = sc.begin[pair + 1];
        step = 1;
    } else {
        first = pair;
        end = total_tiles;
        step = npairs;
    }
}
template <int SCHED>
__device__ __forceinline__ int sched_tile(const SchedParam<SCHED> &sc, int i) {
    if constexpr (SCHED != 0)
        return sc.tile[i];
    else
        return i;
}

struct SharedCtl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

struct SharedCtl2 {
    uint64_t full[6];
    uint64_t empty[6];
    uint64_t cfull[6];     // this CTA's code tile of the stage has landed (CVT variants)
    uint64_t cvt_full[6];  // the leader's: both CTAs' B tiles of the stage are converted
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Problem index and tile coordinates of global tile t.
__device__ __forceinline__ int tile_coords(const KParams &p, int t, int &tm, int &tn) {
    const int pi = (p.nprob > 1 && t >= p.pr[1].tile_begin) ? 1 : 0;
    const int lt = t - (pi ? p.pr[1].tile_begin : 0);
    const int tiles_m = pi ? p.pr[1].tiles_m : p.pr[0].tiles_m;
    const int tiles_n = pi ? p.pr[1].tiles_n : p.pr[0].tiles_n;
    const int m_fast = pi ? p.pr[1].m_fast : p.pr[0].m_fast;
    if (m_fast) {
        tm = lt % tiles_m;
        tn = lt / tiles_m;
    } else {
        tn = lt % tiles_n;
        tm = lt / tiles_n;
    }
    return pi;
}

// Tile t of a pair launch: problem, tile row, first column and width.  In a
// one-problem launch the wide tiles from p.split_begin on (the last, partial wave)
// are each split into two tiles of half the width, so that the wave ends sooner.
struct TileInfo {
    int pi, tm, n0, bn;
    bool narrow;
};

__device__ __forceinline__ TileInfo tile_info(const KParams &p, int t) {
    int tt = t, sub = -1;
    if (p.split_begin >= 0 && t >= p.split_begin) {
        const int r = t - p.split_begin;
        tt = p.split_begin + (r >> 1);
        sub = r & 1;
    }
    int tm, tn;
    TileInfo ti;
    ti.pi = tile_coords(p, tt, tm, tn);
    const int bn = ti.pi ? p.pr[1].bn : p.pr[0].bn;
    ti.tm = tm;
    ti.narrow = sub >= 0;
    ti.bn = ti.narrow ? bn / 2 : bn;
    ti.n0 = tn * bn + (ti.narrow ? sub * (bn / 2) : 0);
    return ti;
}

// Epilogue chunk: 32 consecutive accumulator columns of one row.
template <int EPI, int BITS>
struct Epilogue;

// Each epilogue kind computes the row's 32 values of a chunk; those with an output
// matrix (kinds 0, 1 and 3) leave them in o[], which drain_accumulator writes out.
// Rows at or beyond GM and columns at or beyond GN compute nothing that is stored.

// D -> bf16 output.
template <int BITS>
struct Epilogue<0, BITS> {
    float acc_s = 0.0f, acc_z = 0.0f;
    __device__ __forceinline__ void chunk(const Prob &, int, int, const float (&v)[32], float (&o)[32]) {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = v[j];
    }
};

// Block-AP straight-through: D is dW-hat[N, K] (bf16 W); row = n, col = k.
//   dW = D * mask,  ds += D ((code - zr) - mask * u),  dz = -s * sum_{clamped} D.
// With clamp_pass the mask is 1 everywhere (the clamp is straight-through too).
template <int BITS>
struct Epilogue<1, BITS> {
    float acc_s = 0.0f, acc_z = 0.0f;
    __device__ __forceinline__ void chunk(const Prob &p, int row, int col, const float (&v)[32],
                                          float (&dwv)[32]) {
        if (row >= p.GM || col >= p.GN) {
#pragma unroll
            for (int j = 0; j < 32; ++j) dwv[j] = 0.0f;
            return;
        }
        const int64_t K = p.GN;
        const int64_t G = K >> p.gshift;
        const int64_t gi = static_cast<int64_t>(row) * G + (col >> p.gshift);
        const float sc = __ldg(p.s + gi);
        const float rcp = __frcp_rn(sc);
        const float zr = rintf(__ldg(p.z + gi));
        const int64_t e0 = static_cast<int64_t>(row) * K + col;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float w[8];
            load8<__nv_bfloat16>(static_cast<const __nv_bfloat16 *>(p.W) + e0 + 8 * q, w);
            float r[8], u[8];
            round_quotients<8>(w, sc, rcp, r, u);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float d = v[8 * q + j];
                const float qv = __fadd_rn(r[j], zr);
                const bool inside = ((qv >= 0.0f) && (qv <= p.Q)) || p.clamp_pass;
                const float c = fminf(fmaxf(qv, 0.0f), p.Q);
                const float dwds = __fsub_rn(__fsub_rn(c, zr), inside ? u[j] : 0.0f);
                acc_s = fmaf(d, dwds, acc_s);
                acc_z += inside ? 0.0f : d;
                dwv[8 * q + j] = inside ? d : 0.0f;
            }
        }
        if (((col + 32) & (p.group - 1)) == 0) {
            if (p.ds) p.ds[gi] = acc_s;
            if (p.dz) p.dz[gi] = -sc * acc_z;
            acc_s = 0.0f;
            acc_z = 0.0f;
        }
    }
};

// E2E-QP: D is dW-hat[N, K]; ds = sum_group D * (W_q - zq), dz = -s sum_group D
// (the zero point trained as a float at zq).
template <int BITS>
struct Epilogue<2, BITS> {
    float acc_s = 0.0f, acc_z = 0.0f;
    __device__ __forceinline__ void chunk(const Prob &p, int row, int col, const float (&v)[32], float (&)[32]) {
        if (row >= p.GM || col >= p.GN) return;
        const int64_t K = p.GN;
        const int64_t G = K >> p.gshift;
        const int64_t gi = static_cast<int64_t>(row) * G + (col >> p.gshift);
        const float zf = static_cast<float>(__ldg(p.zq + gi));
        uint32_t c[32];
        if (BITS == 2) {
            const uint2 r = __ldg(reinterpret_cast<const uint2 *>(p.codes + (static_cast<int64_t>(row) * K + col) / 4));
#pragma unroll
            for (int j = 0; j < 16; ++j) c[j] = (r.x >> (2 * j)) & 3u;
#pragma unroll
            for (int j = 0; j < 16; ++j) c[16 + j] = (r.y >> (2 * j)) & 3u;
        } else if (BITS == 4) {
            const uint4 r = __ldg(reinterpret_cast<const uint4 *>(p.codes + (static_cast<int64_t>(row) * K + col) / 2));
            const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int j = 0; j < 32; ++j) c[j] = (w4[j / 8] >> (4 * (j % 8))) & 15u;
        } else {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.codes + static_cast<int64_t>(row) * K + col);
            const uint4 r0 = __ldg(src), r1 = __ldg(src + 1);
            const uint32_t w8[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
            for (int j = 0; j < 32; ++j) c[j] = (w8[j / 4] >> (8 * (j % 4))) & 0xFFu;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) acc_s = fmaf(v[j], __fsub_rn(static_cast<float>(c[j]), zf), acc_s);
        if (p.dz) {
#pragma unroll
            for (int j = 0; j < 32; ++j) acc_z += v[j];
        }
        if (((col + 32) & (p.group - 1)) == 0) {
            if (p.ds) p.ds[gi] = acc_s;
            if (p.dz) {
                const float sc = p.s_f16 ? __half2float(static_cast<const __half *>(p.s_e2e)[gi])
                                         : static_cast<const float *>(p.s_e2e)[gi];
                p.dz[gi] = -sc * acc_z;
            }
            acc_s = 0.0f;
            acc_z = 0.0f;
        }
    }
};

// Block-AP reconstruction loss against the full-precision output T: D is Y[M, N]
// (fp32, never stored).  dY = mse_scale (D - T) in bf16, and the thread's sum of
// (D - T)^2 goes to *loss (fp64) when the drain ends.
template <int BITS>
struct Epilogue<3, BITS> {
    float acc_s = 0.0f, acc_z = 0.0f;
    __device__ __forceinline__ void chunk(const Prob &p, int row, int col, const float (&v)[32], float (&o)[32]) {
        if (row >= p.GM) {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0.0f;
            return;
        }
        const int64_t off = static_cast<int64_t>(row) * p.ldo + col;
        const __nv_bfloat16 *T = static_cast<const __nv_bfloat16 *>(p.target) + off;
        if (col + 32 <= p.GN) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float t[8];
                load8<__nv_bfloat16>(T + 8 * q, t);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float d = __fsub_rn(v[8 * q + j], t[j]);
                    acc_s = fmaf(d, d, acc_s);
                    o[8 * q + j] = __fmul_rn(d, p.mse_scale);
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                o[j] = 0.0f;
                if (col + j < p.GN) {
                    const float d = __fsub_rn(v[j], __bfloat162float(T[j]));
                    acc_s = fmaf(d, d, acc_s);
                    o[j] = __fmul_rn(d, p.mse_scale);
                }
            }
        }
    }
};

template <int EPI>
__device__ __forceinline__ void finish_drain(const Prob &p, float acc) {
    if (EPI == 3) {
        double a = acc;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        // mse_scale = 2 / (M N): the loss is the mean
        if ((threadIdx.x & 31) == 0) atomicAdd(p.loss, a * (0.5 * static_cast<double>(p.mse_scale)));
    }
}

// The output of one epilogue warp: 32 rows x 32 columns of bf16 per chunk.  With a
// tensor map (CTA-pair kernel) the warp writes the chunk into its 2 KB of shared
// memory in the 64-byte-swizzled layout of the map's box, and lane 0 stores it with
// a TMA: the lanes do not wait on the stores, and each leaves the SM as whole
// sectors (a lane owns one output row, so direct stores touch 32 rows per
// instruction).  The TMA clips rows and columns beyond the matrix.  Without a map
// (one-CTA kernel) the lanes store their rows directly.
struct OutStage {
    uint8_t *buf;            // this warp's staging buffer (512-byte aligned)
    const CUtensorMap *map;  // nullptr: direct stores
    bool pending;            // a TMA store may still read buf
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <int EPI>
constexpr bool kHasOut = EPI == 0 || EPI == 1 || EPI == 3;

__device__ __forceinline__ void write_chunk(OutStage &os, void *dst, int64_t ld, int64_t GM, int64_t GN, int row0,
                                            int col, const float (&o)[32]) {
    const int lane = threadIdx.x & 31;
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
    if (os.map) {
        if (os.pending) {  // the previous chunk's store has read the buffer
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
        }
        uint8_t *rp = os.buf + lane * 64;
        const int sw = (lane >> 1) & 3;  // 64-byte swizzle: 16-byte unit q of row r at q ^ ((r >> 1) & 3)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(rp + ((q ^ sw) << 4)) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < GM && col < GN) {
            tma_store_2d(os.map, os.buf, col, row0);
            bulk_commit();
        }
        os.pending = true;
        return;
    }
    const int row = row0 + lane;
    if (row >= GM || col >= GN) return;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(dst) + row * ld + col;
    if (col + 32 <= GN) {
        uint4 *q4 = reinterpret_cast<uint4 *>(out);
#pragma unroll
        for (int q = 0; q < 4; ++q) q4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (col + j < GN) out[j] = __float2bfloat16_rn(o[j]);
    }
}

// Drains one accumulator (this warp's 32 rows, columns [c_begin, c_end)) through
// the epilogue of kind EPI.  row = row0 + lane.
template <int EPI, int BITS>
__device__ __forceinline__ void drain_accumulator(const Prob &pr, uint32_t taddr, int row0, int col0,
                                                  int c_begin, int c_end, OutStage &os) {
    Epilogue<EPI, BITS> epi;
    const int row = row0 + (threadIdx.x & 31);
    void *dst = EPI == 1 ? pr.dW : pr.out;
    const int64_t ld = EPI == 1 ? static_cast<int64_t>(pr.GN) : pr.ldo;
#pragma unroll 1
    for (int c0 = c_begin; c0 < c_end; c0 += 32) {
        float v[32];
        tmem_ld_32cols(taddr + c0, v);
        float o[32];
        epi.chunk(pr, row, col0 + c0, v, o);
        if (kHasOut<EPI> && dst) write_chunk(os, dst, ld, pr.GM, pr.GN, row0, col0 + c0, o);
    }
    finish_drain<EPI>(pr, epi.acc_s);
}

// Persistent grouped GEMM: problem 0 uses epilogue EPI0, problem 1 (if any)
// EPI1; operand majorness is a per-problem runtime property.
template <int EPI0, int EPI1, int BITS, int EPI_WARPS>
__global__ void __launch_bounds__((4 + EPI_WARPS) * 32, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
              const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
              const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    SharedCtl *ctl = reinterpret_cast<SharedCtl *>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5;
    constexpr int EPI_THREADS = EPI_WARPS * 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&ctl->full[i], 1);
            mbar_init(&ctl->empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->acc_full[i], 1);
            mbar_init(&ctl->acc_empty[i], EPI_THREADS);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmB0);
        if (p.nprob > 1) {
            tma_prefetch_desc(&tmA1);
            tma_prefetch_desc(&tmB1);
        }
    }
    // A programmatic dependent (eqat_pdl.cuh): everything above touched only this
    // CTA's shared memory and the kernel parameters; tensor and global memory come
    // after the preceding kernel has completed.
    pdl_wait();
    if (threadIdx.x == 0) pdl_allow_dependents();
    if (warp == 2) {
        tmem_alloc(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int *abort_flag = &ctl->abort_flag;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (elect_one_sync()) {
            uint32_t it = 0;
            uint32_t armed = 0;         // stages with a load issued
            uint32_t armed_parity = 0;  // parity of the last phase armed per stage
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
                int tm, tn;
                const int pi = tile_coords(p, t, tm, tn);
                const CUtensorMap *ma = pi ? &tmA1 : &tmA0;
                const CUtensorMap *mb = pi ? &tmB1 : &tmB0;
                const int a_mn = pi ? p.pr[1].a_mn : p.pr[0].a_mn;
                const int b_mn = pi ? p.pr[1].b_mn : p.pr[0].b_mn;
                const int nkb = ((pi ? p.pr[1].GK : p.pr[0].GK) + BK - 1) / BK;
                const int bn = pi ? p.pr[1].bn : p.pr[0].bn;
                const int m0 = tm * BM, n0 = tn * bn;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int st = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait_bounded(&ctl->empty[st], ph ^ 1u, abort_flag, p.err, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + st * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&ctl->full[st], A_BYTES + bn * BK * 2);
                    armed |= 1u << st;
                    armed_parity = (armed_parity & ~(1u << st)) | (ph << st);
                    const int k0 = kb * BK;
                    if (a_mn) {
#pragma unroll
                        for (int b = 0; b < BM / MN_BOX; ++b)
                            tma_load_2d(sa + b * MN_BOX_BYTES, ma, &ctl->full[st], m0 + b * MN_BOX, k0);
                    } else {
                        tma_load_2d(sa, ma, &ctl->full[st], k0, m0);
                    }
                    if (b_mn) {
#pragma unroll
                        for (int b = 0; b < bn / MN_BOX; ++b)
                            tma_load_2d(sb + b * MN_BOX_BYTES, mb, &ctl->full[st], n0 + b * MN_BOX, k0);
                    } else {
                        tma_load_2d(sb, mb, &ctl->full[st], k0, n0);
                    }
                }
            }
            if (!ok) {
                // Let the copies already issued land before the block exits.
                for (int st = 0; st < STAGES; ++st)
                    if (armed & (1u << st)) {
                        const uint32_t a = smem_u32(&ctl->full[st]);
                        const uint64_t t0 = globaltimer_ns();
                        while (!mbar_try_wait(a, (armed_parity >> st) & 1u) &&
                               globaltimer_ns() - t0 < 100000000ull) {
                        }
                    }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (elect_one_sync()) {
            uint32_t it = 0;
            uint32_t local = 0;
            bool ok = true;
            bool issued = false;
            for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x, ++local) {
                int tm, tn;
                const int pi = tile_coords(p, t, tm, tn);
                const int a_mn = pi ? p.pr[1].a_mn : p.pr[0].a_mn;
                const int b_mn = pi ? p.pr[1].b_mn : p.pr[0].b_mn;
                const int nkb = ((pi ? p.pr[1].GK : p.pr[0].GK) + BK - 1) / BK;
                const int bn = pi ? p.pr[1].bn : p.pr[0].bn;
                const uint32_t idesc = idesc_bf16_f32(BM, bn, a_mn != 0, b_mn != 0);
                // K-major: advance 16 elements (32 B) inside the 128 B swizzle row,
                // LBO unused (16), SBO = 8 rows x 128 B.  MN-major: advance 16 k-rows
                // (2 KB), LBO = next 64-wide MN box, SBO = 8 k-rows x 128 B.
                const uint32_t a_step = a_mn ? UK * 128 : UK * 2, a_lbo = a_mn ? MN_BOX_BYTES : 16;
                const uint32_t b_step = b_mn ? UK * 128 : UK * 2, b_lbo = b_mn ? MN_BOX_BYTES : 16;
                const uint32_t acc = local & 1u;
                const uint32_t aph = (local >> 1) & 1u;
                if (!mbar_wait_bounded(&ctl->acc_empty[acc], aph ^ 1u, abort_flag, p.err, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int st = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait_bounded(&ctl->full[st], ph, abort_flag, p.err, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + st * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        const uint64_t ad = smem_desc_sw128(sa + kk * a_step, a_lbo, 1024);
                        const uint64_t bd = smem_desc_sw128(sb + kk * b_step, b_lbo, 1024);
                        tc_mma_f16(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(&ctl->empty[st]);
                }
                if (!ok) break;
                tc_commit(&ctl->acc_full[acc]);
            }
            if (!ok && issued) {
                // Wait for the MMAs already issued before tensor memory is freed.
                tc_commit(&ctl->drain);
                const uint32_t a = smem_u32(&ctl->drain);
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < 100000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------------------------- epilogue
        const int ew = warp - 4;
        const int quad = warp & 3;  // tensor-memory lane quadrant of this warp
        const int half = ew >> 2;   // column slice of the accumulator
        constexpr int SLICES = EPI_WARPS / 4;

        uint32_t local = 0;
        for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++local) {
            const uint32_t acc = local & 1u;
            const uint32_t aph = (local >> 1) & 1u;
            // Every lane waits; the warp leaves together (tcgen05.ld is .sync.aligned).
            const bool ok = mbar_wait_bounded(&ctl->acc_full[acc], aph, abort_flag, p.err, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            int tm, tn;
            const int pi = tile_coords(p, t, tm, tn);
            const int row0 = tm * BM + quad * 32;
            const uint32_t taddr = tmem_base + acc * ACC_COLS + ((quad * 32) << 16);
            const int bn = pi ? p.pr[1].bn : p.pr[0].bn;
            const int cols = bn / SLICES;  // a multiple of 64, hence of every group size
            OutStage os{nullptr, nullptr, false};  // direct stores
            if (pi == 0)
                drain_accumulator<EPI0, BITS>(p.pr[0], taddr, row0, tn * bn, half * cols, (half + 1) * cols, os);
            else
                drain_accumulator<EPI1, BITS>(p.pr[1], taddr, row0, tn * bn, half * cols, (half + 1) * cols, os);
            tc_fence_before();
            mbar_arrive(&ctl->acc_empty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------- CTA pairs
// The same grouped GEMM on pairs of SMs (cta_group::2, cluster of two CTAs):
// one tcgen05.mma covers a 256-row tile, each CTA stages its 128 rows of A and
// half of the tile's B columns, the even CTA issues the MMAs, and each CTA's
// tensor memory holds its 128 accumulator rows.  Per SM, a 256 x bn pair tile
// reads a third less operand data from shared memory per FLOP than a 128 x bn
// tile of one CTA (B is split between the two SMs), the limiter of the one-CTA
// kernel.  Protocol:
//   full[s]      the leader's: armed by the leader with both CTAs' bytes, completed
//                by both CTAs' TMA loads (each into its own shared memory)
//   empty[s]     each CTA's: the leader's MMA commit arrives on both (multicast)
//   acc_full[a]  each CTA's: the leader's commit after a tile's last MMA (multicast)
//   acc_empty[a] the leader's: both CTAs' epilogue threads arrive after draining
constexpr int BM2 = 256;              // rows of a pair tile
constexpr int A_HALF = 128 * BK * 2;  // this CTA's 128 rows of A per stage
constexpr int B_HALF = 128 * BK * 2;  // up to 128 rows of B per stage

// Stage layout of the pair kernel.  CVT variants add a slot for the stage's packed
// code tile (128 rows x 64 codes at most) behind A and B and four converter warps.
template <int CVT, int BITS, int EW = 8>
struct PairCfg {
    static constexpr int CODE_BITS = BITS == 3 ? 8 : BITS;  // stored bits per code (3-bit: one byte)
    static constexpr int CODE_SLOT = CVT ? 128 * 8 * CODE_BITS : 0;
    static constexpr int STAGE = A_HALF + B_HALF + CODE_SLOT;
    static constexpr int STAGES = (CVT && CODE_BITS > 2) ? 5 : 6;
    // Converter warps: one per ring slot; warp w converts every stage of slot w, a whole
    // stage per warp, so that all the ring's stages can be in conversion at once and
    // each warp has the time of STAGES stages of MMA for one of its own.
    static constexpr int CVT_WARPS = CVT ? STAGES : 0;
    // Epilogue warps: the plain store and the E2E ds epilogue keep up with four next to
    // the converters; otherwise EW (8, or 16 for the straight-through epilogue of a
    // shallow contraction, chosen per launch).
    static constexpr int EPI_WARPS = CVT ? 4 : EW;
    // Per converter warp: the group constants (s, zq as fp32) of the stage it converts,
    // two per B tile row (the two 32-code halves of its 64 codes).
    static constexpr int CONST_BYTES = CVT_WARPS * 256 * 8;
    // Per epilogue warp: one 32 x 32 bf16 output chunk on its way to a TMA store.
    static constexpr int OUT_BYTES = EPI_WARPS * 2048;
    static constexpr int SMEM = 1024 + STAGES * STAGE + CONST_BYTES + OUT_BYTES + 256;
};
static_assert(PairCfg<1, 3>::SMEM <= 232448 && PairCfg<1, 2>::SMEM <= 232448 && PairCfg<1, 4>::SMEM <= 232448 &&
                  PairCfg<0, 2, 16>::SMEM <= 232448,
              "pair kernel stages exceed the shared memory of a CTA");
static_assert(sizeof(SharedCtl2) <= 256, "control block exceeds its slot");

// ------------------------------------------------------------------ dequantize on load
// Eq. 2 on the way into the MMA (modelfoundations note, Phase 2: only dequantization
// sits in the E2E-QP graph): the B tile W-hat = (W_q - zq) s of a stage is made in
// shared memory from the stage's packed code tile, in the 128-byte-swizzled layout a
// TMA load of bf16 W-hat would have produced, so the MMA descriptors do not change.
//
// A B tile row ("row" below) is 64 consecutive in-features k of one W-hat row n: for
// the forward (K-major B) row r of the tile is n = n0 + r over the stage's k range; for
// the input gradient (MN-major B) row b*64 + r is n = k0 + r (the contraction index)
// over the columns n0 + 64 b ...  Its codes are 8 * CODE_BITS contiguous bytes.
//
// Exactness.  With 0 <= m < 2^23 the fp32 number with bits 0x4B000000 | m is exactly
// 2^23 + m.  A code c at bit offset CB*i of a 16-bit half word, masked in place, gives
// f = 2^23 + c 2^(CB i); o_i = 2^23 + zq 2^(CB i) likewise (zq <= 15 keeps both below
// 2^24), so f - o_i = (c - zq) 2^(CB i) exactly, and multiplying by s 2^(-CB i) (exact:
// a power-of-two scaling of a normal s) rounds once to RN((c - zq) s), the fp32 product
// of Eq. 2.  cvt.rn.bf16x2.f32 then rounds it to the bf16 operand as the dequantize
// kernel does.  Two weights per packed-fp32 instruction.
template <int BITS>
struct CodeFmt {
    static constexpr int CB = BITS == 3 ? 8 : BITS;  // stored bits per code
    static constexpr int PER_UNIT = 128 / CB;        // codes in one 16-byte unit: 64, 32, 16
    static constexpr int PER_HALF = 16 / CB;         // codes in a 16-bit half word: 8, 4, 2
    static constexpr int UPR = CB / 2;               // 16-byte units per 64-code row: 1, 2, 4
    static constexpr uint32_t MASK = (1u << CB) - 1u;
};

__device__ __forceinline__ uint64_t cf2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ uint64_t cf2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t cf2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// Two fp32 lanes (lo, hi) to one bf16x2 word, round to nearest even (lo in the low half).
__device__ __forceinline__ uint32_t cf2_to_bf16x2(uint64_t v) {
    uint32_t d;
    asm("{\n"
        ".reg .f32 lo, hi;\n"
        "mov.b64 {lo, hi}, %1;\n"
        "cvt.rn.bf16x2.f32 %0, hi, lo;\n"
        "}\n"
        : "=r"(d)
        : "l"(v));
    return d;
}

// The constants of one group for the codes of a half word: o_i, s_i as packed pairs
// (i, i + 1).
template <int BITS>
struct GroupPairs {
    uint64_t off[CodeFmt<BITS>::PER_HALF / 2];
    uint64_t sc[CodeFmt<BITS>::PER_HALF / 2];
    __device__ __forceinline__ void set(float s, uint32_t zq) {
        using F = CodeFmt<BITS>;
#pragma unroll
        for (int i = 0; i < F::PER_HALF; i += 2) {
            const float o0 = __uint_as_float(0x4B000000u + (zq << (F::CB * i)));
            const float o1 = __uint_as_float(0x4B000000u + (zq << (F::CB * (i + 1))));
            const float s0 = __fmul_rn(s, __uint_as_float(static_cast<uint32_t>(127 - F::CB * i) << 23));
            const float s1 = __fmul_rn(s, __uint_as_float(static_cast<uint32_t>(127 - F::CB * (i + 1)) << 23));
            off[i / 2] = cf2_pack(o0, o1);
            sc[i / 2] = cf2_pack(s0, s1);
        }
    }
};

// W-hat of the PER_HALF codes of half word h (codes at bit offsets CB*i) as
// PER_HALF / 2 bf16x2 words, code order.
template <int BITS>
__device__ __forceinline__ void convert_half(uint32_t h, const GroupPairs<BITS> &gp, uint32_t *out) {
    using F = CodeFmt<BITS>;
#pragma unroll
    for (int i = 0; i < F::PER_HALF; i += 2) {
        const float a = __uint_as_float((h & (F::MASK << (F::CB * i))) | 0x4B000000u);
        const float b = __uint_as_float((h & (F::MASK << (F::CB * (i + 1)))) | 0x4B000000u);
        out[i / 2] = cf2_to_bf16x2(cf2_mul(cf2_sub(cf2_pack(a, b), gp.off[i / 2]), gp.sc[i / 2]));
    }
}

// A 16-byte unit of the stage's code tile (units are numbered by their offset in the tile).
// Where a unit lies (tile row, first 16-byte chunk of the row it fills, W-hat n and k).
struct UnitPos {
    int row, chunk, n, k;
};

template <int BITS>
__device__ __forceinline__ UnitPos unit_pos(int u, int b_mn, int half, int n0, int k0) {
    using F = CodeFmt<BITS>;
    UnitPos p;
    if (!b_mn) {
        const int r = u / F::UPR, q = u % F::UPR;
        p.row = r;
        p.chunk = q * (F::PER_UNIT / 8);
        p.n = n0 + r;
        p.k = k0 + q * F::PER_UNIT;
    } else {
        const int per_row = half * F::CB / 128;  // units per code row (contraction index)
        const int r = u / per_row, w = u % per_row;
        const int b = w / F::UPR, q = w % F::UPR;
        p.row = b * 64 + r;
        p.chunk = q * (F::PER_UNIT / 8);
        p.n = k0 + r;
        p.k = n0 + 64 * b + q * F::PER_UNIT;
    }
    return p;
}

// Where the group constants of B tile row `row`, code half `hsub` (codes 32 hsub ..
// 32 hsub + 31 of the row's 64) come from: W-hat row n and in-feature k.
__device__ __forceinline__ void row_half_pos(int row, int hsub, int b_mn, int n0, int k0, int &n, int &k) {
    if (!b_mn) {
        n = n0 + row;
        k = k0 + 32 * hsub;
    } else {
        n = k0 + (row & 63);
        k = n0 + 64 * (row >> 6) + 32 * hsub;
    }
}

// The stage's constants, gathered by one warp into registers a stage ahead: entry
// e = lane + 32 i is (row e / 2, half e % 2) of the B tile; s = 0 and zq = 0 where the
// row or the in-feature lies outside W-hat.
constexpr int kConstPerLane = 256 / 32;

struct StageConsts {
    float s[kConstPerLane];
    uint32_t zq[kConstPerLane];
};

// With groups of 64 or more the two halves of a row share their group: entries
// e = lane + 32 i, i < 4, are then rows (one load per row) and stand for both halves.
__device__ __forceinline__ void gather_consts(const Prob &pr, int b_mn, int half, int n0, int k0, int lane,
                                              StageConsts &c) {
    const bool per_row = pr.gshift > 5;
#pragma unroll
    for (int i = 0; i < kConstPerLane; ++i) {
        const int e = lane + 32 * i;
        c.s[i] = 0.0f;
        c.zq[i] = 0u;
        if (per_row ? (e < half) : (e < 2 * half)) {
            int n, k;
            if (per_row)
                row_half_pos(e, 0, b_mn, n0, k0, n, k);
            else
                row_half_pos(e >> 1, e & 1, b_mn, n0, k0, n, k);
            if (n < pr.w_rows && k < pr.w_cols) {
                const int64_t gi = static_cast<int64_t>(n) * pr.w_groups + (k >> pr.gshift);
                c.s[i] = pr.cvt_s_f16 ? __half2float(__ldg(static_cast<const __half *>(pr.cvt_s) + gi))
                                      : __ldg(static_cast<const float *>(pr.cvt_s) + gi);
                c.zq[i] = __ldg(pr.cvt_zq + gi);
            }
        }
    }
}

// One warp converts a whole stage: code units u = lane, lane + 32, ... of the stage's
// code tile into the B slot.  `tab` holds the stage's constants (float2 {s, zq} per
// entry, written by this warp just before).
template <int BITS>
__device__ __forceinline__ void convert_stage_warp(const uint8_t *codes_smem, uint8_t *b_smem, int b_mn, int half,
                                                   bool two_groups, int lane, const float2 *tab) {
    using F = CodeFmt<BITS>;
    const int units = half * F::CB / 2;
#pragma unroll 2
    for (int u = lane; u < units; u += 32) {
        const UnitPos p = unit_pos<BITS>(u, b_mn, half, 0, 0);
        const uint4 raw = *reinterpret_cast<const uint4 *>(codes_smem + 16 * u);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint8_t *row = b_smem + p.row * 128;
        const int sw = p.row & 7;
        // the unit's codes start at code 8 * p.chunk of the row: half 0 or 1 of it
        const int h0 = (8 * p.chunk) >> 5;
        GroupPairs<BITS> gp;
        float2 c = tab[2 * p.row + h0];
        gp.set(c.x, static_cast<uint32_t>(c.y));
        constexpr int HALVES_PER_CHUNK = 8 / F::PER_HALF;
#pragma unroll
        for (int cc = 0; cc < F::PER_UNIT / 8; ++cc) {
            if (BITS == 2 && cc == 4 && two_groups) {  // codes 32..63 of the row: another group of 32
                c = tab[2 * p.row + 1];
                gp.set(c.x, static_cast<uint32_t>(c.y));
            }
            uint32_t o[4];
#pragma unroll
            for (int hh = 0; hh < HALVES_PER_CHUNK; ++hh) {
                const int hidx = cc * HALVES_PER_CHUNK + hh;  // half word index in the unit
                const uint32_t word = w[hidx >> 1];
                const uint32_t h = (hidx & 1) ? (word >> 16) : (word & 0xFFFFu);
                convert_half<BITS>(h, gp, o + hh * (F::PER_HALF / 2));
            }
            const int pos = (p.chunk + cc) ^ sw;
            *reinterpret_cast<uint4 *>(row + pos * 16) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// The converter warps' walk over the launch's stages, in the order of the producer and
// the MMA issuer: (tile, k block) with the global stage counter `it`.
struct StageWalk {
    int t, kb, nkb;
    uint32_t it;
    TileInfo ti;
};

// ---------------------------------------------------------------------------- CTA pairs
// The same grouped GEMM on pairs of SMs (cta_group::2, cluster of two CTAs):
// one tcgen05.mma covers a 256-row tile, each CTA stages its 128 rows of A and
// half of the tile's B columns, the even CTA issues the MMAs, and each CTA's
// tensor memory holds its 128 accumulator rows.  Per SM, a 256 x bn pair tile
// reads a third less operand data from shared memory per FLOP than a 128 x bn
// tile of one CTA (B is split between the two SMs), the limiter of the one-CTA
// kernel.  Protocol:
//   full[s]      the leader's: armed by the leader with both CTAs' bytes, completed
//                by both CTAs' TMA loads (each into its own shared memory)
//   empty[s]     each CTA's: the leader's MMA commit arrives on both (multicast)
//   acc_full[a]  each CTA's: the leader's commit after a tile's last MMA (multicast)
//   acc_empty[a] the leader's: both CTAs' epilogue threads arrive after draining
// CVT variants, for the stages of a problem whose B is made from codes on load:
//   cfull[s]     each CTA's: its own TMA load of the stage's code tile
//   cvt_full[s]  the leader's: one arrival per converter warp of both CTAs once the
//                warp's part of the B tile is written and fenced for the tensor core;
//                the MMA issuer waits on it besides full[s] (which then counts A only)
template <int EPI0, int EPI1, int BITS, int EPI_WARPS, int CVT, int SCHED>
__global__ void __launch_bounds__((4 + EPI_WARPS + PairCfg<CVT, BITS, EPI_WARPS>::CVT_WARPS) * 32, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
               const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
               const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
               const KParams p, const __grid_constant__ SchedParam<SCHED> sched) {
    using C = PairCfg<CVT, BITS, EPI_WARPS>;
    static_assert(EPI_WARPS == C::EPI_WARPS, "the staging area is sized for C::EPI_WARPS epilogue warps");
    constexpr int STAGES2 = C::STAGES;
    constexpr int STAGE2_BYTES = C::STAGE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    SharedCtl2 *ctl =
        reinterpret_cast<SharedCtl2 *>(smem + STAGES2 * STAGE2_BYTES + C::CONST_BYTES + C::OUT_BYTES);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    constexpr int EPI_THREADS = EPI_WARPS * 32;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES2; ++i) {
            mbar_init(&ctl->full[i], 1);
            mbar_init(&ctl->empty[i], 1);
            mbar_init(&ctl->cfull[i], 1);
            mbar_init(&ctl->cvt_full[i], 2);  // one converter warp of each CTA
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->acc_full[i], 1);
            mbar_init(&ctl->acc_empty[i], 2 * EPI_THREADS);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort_flag = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmB0);
        if (p.nprob > 1) {
            tma_prefetch_desc(&tmA1);
            tma_prefetch_desc(&tmB1);
        }
    }
    // A programmatic dependent (eqat_pdl.cuh): everything above touched only this
    // CTA's shared memory and the kernel parameters; tensor and global memory come
    // after the preceding kernel has completed.
    pdl_wait();
    if (threadIdx.x == 0) pdl_allow_dependents();
    if (warp == 2) {
        tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised and the pair's tensor memory is allocated
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    volatile int *abort_flag = &ctl->abort_flag;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const uint32_t full0 = map_to_rank(&ctl->full[0], 0);           // the leader's full barriers
    const uint32_t acc_empty0 = map_to_rank(&ctl->acc_empty[0], 0);  // the leader's accumulator-empty barriers

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer (both CTAs)
        if (elect_one_sync()) {
            uint32_t it = 0;
            uint32_t armed = 0, armed_parity = 0;     // the leader's full barriers with a phase armed
            uint32_t carmed = 0, carmed_parity = 0;   // this CTA's code barriers with a phase armed
            uint32_t cuse = 0;                        // per stage: parity of its next code phase
            bool ok = true;
            int w_first, w_end, w_step;
            sched_range<SCHED>(sched, p.total_tiles, pair, npairs, w_first, w_end, w_step);
            for (int w = w_first; ok && w < w_end; w += w_step) {
                const TileInfo ti = tile_info(p, sched_tile<SCHED>(sched, w));
                const int pi = ti.pi;
                const CUtensorMap *ma = pi ? &tmA1 : &tmA0;
                // the halves of a split wave take B through the second map (half the box rows)
                const CUtensorMap *mb = (pi || ti.narrow) ? &tmB1 : &tmB0;
                const int a_mn = pi ? p.pr[1].a_mn : p.pr[0].a_mn;
                const int b_mn = pi ? p.pr[1].b_mn : p.pr[0].b_mn;
                const bool cvt = CVT && (pi ? p.pr[1].b_cvt : p.pr[0].b_cvt);
                const int nkb = ((pi ? p.pr[1].GK : p.pr[0].GK) + BK - 1) / BK;
                const int half = ti.bn / 2;
                const int m0 = ti.tm * BM2 + 128 * static_cast<int>(rank);
                const int n0 = ti.n0 + half * static_cast<int>(rank);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int st = it % STAGES2;
                    const uint32_t ph = (it / STAGES2) & 1u;
                    if (!mbar_wait_bounded(&ctl->empty[st], ph ^ 1u, abort_flag, p.err, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + st * STAGE2_BYTES;
                    uint8_t *sb = sa + A_HALF;
                    if (leader) {
                        mbar_arrive_expect_tx(&ctl->full[st], 2 * (A_HALF + (cvt ? 0 : half * BK * 2)));
                        armed |= 1u << st;
                        armed_parity = (armed_parity & ~(1u << st)) | (ph << st);
                    }
                    const uint32_t bar = full0 + 8u * static_cast<uint32_t>(st);
                    const int k0 = kb * BK;
                    if (a_mn) {
#pragma unroll
                        for (int b = 0; b < 128 / MN_BOX; ++b)
                            tma_load_2d_pair(sa + b * MN_BOX_BYTES, ma, bar, m0 + b * MN_BOX, k0);
                    } else {
                        tma_load_2d_pair(sa, ma, bar, k0, m0);
                    }
                    if (cvt) {
                        // this CTA's code tile, on its own barrier: K-major rows n0.. at
                        // byte k0 * CB / 8; MN-major rows k0.. (the contraction index) at
                        // byte n0 * CB / 8
                        constexpr int CBITS = CodeFmt<BITS>::CB;
                        const uint32_t cph = (cuse >> st) & 1u;
                        cuse ^= 1u << st;
                        mbar_arrive_expect_tx(&ctl->cfull[st], half * 8 * CBITS);
                        carmed |= 1u << st;
                        carmed_parity = (carmed_parity & ~(1u << st)) | (cph << st);
                        uint8_t *sc = sb + B_HALF;
                        if (b_mn)
                            tma_load_2d(sc, mb, &ctl->cfull[st], n0 * CBITS / 8, k0);
                        else
                            tma_load_2d(sc, mb, &ctl->cfull[st], k0 * CBITS / 8, n0);
                    } else if (b_mn) {
                        for (int b = 0; b < half / MN_BOX; ++b)
                            tma_load_2d_pair(sb + b * MN_BOX_BYTES, mb, bar, n0 + b * MN_BOX, k0);
                    } else {
                        tma_load_2d_pair(sb, mb, bar, k0, n0);
                    }
                }
            }
            if (!ok) {
                // Copies this CTA issued for stages the leader has not armed count on
                // no phase that can complete: give them a fixed 2 ms to land.
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 2000000ull) {
                }
                // This CTA's code copies count on its own barriers: let them land.
                for (int st = 0; st < STAGES2; ++st)
                    if (carmed & (1u << st)) {
                        const uint32_t a = smem_u32(&ctl->cfull[st]);
                        const uint64_t t1 = globaltimer_ns();
                        while (!mbar_try_wait(a, (carmed_parity >> st) & 1u) &&
                               globaltimer_ns() - t1 < 100000000ull) {
                        }
                    }
            }
            if (!ok && leader) {
                // Let the pair's copies already issued land before the blocks exit.
                for (int st = 0; st < STAGES2; ++st)
                    if (armed & (1u << st)) {
                        const uint32_t a = smem_u32(&ctl->full[st]);
                        const uint64_t t0 = globaltimer_ns();
                        while (!mbar_try_wait(a, (armed_parity >> st) & 1u) &&
                               globaltimer_ns() - t0 < 100000000ull) {
                        }
                    }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer (the leader)
        if (leader && elect_one_sync()) {
            uint32_t it = 0, local = 0;
            uint32_t cuse = 0;  // per stage: parity of its next converted phase
            bool ok = true, issued = false;
            int w_first, w_end, w_step;
            sched_range<SCHED>(sched, p.total_tiles, pair, npairs, w_first, w_end, w_step);
            for (int w = w_first; ok && w < w_end; w += w_step, ++local) {
                const TileInfo ti = tile_info(p, sched_tile<SCHED>(sched, w));
                const int pi = ti.pi;
                const int a_mn = pi ? p.pr[1].a_mn : p.pr[0].a_mn;
                const int b_mn = pi ? p.pr[1].b_mn : p.pr[0].b_mn;
                const bool cvt = CVT && (pi ? p.pr[1].b_cvt : p.pr[0].b_cvt);
                const int nkb = ((pi ? p.pr[1].GK : p.pr[0].GK) + BK - 1) / BK;
                const uint32_t idesc = idesc_bf16_f32(BM2, ti.bn, a_mn != 0, b_mn != 0);
                const uint32_t a_step = a_mn ? UK * 128 : UK * 2, a_lbo = a_mn ? MN_BOX_BYTES : 16;
                const uint32_t b_step = b_mn ? UK * 128 : UK * 2, b_lbo = b_mn ? MN_BOX_BYTES : 16;
                const uint32_t acc = local & 1u;
                const uint32_t aph = (local >> 1) & 1u;
                if (!mbar_wait_bounded(&ctl->acc_empty[acc], aph ^ 1u, abort_flag, p.err, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int st = it % STAGES2;
                    const uint32_t ph = (it / STAGES2) & 1u;
                    if (!mbar_wait_bounded(&ctl->full[st], ph, abort_flag, p.err, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    if (cvt) {
                        const uint32_t cph = (cuse >> st) & 1u;
                        cuse ^= 1u << st;
                        const bool w = p.cvt_cluster_scope
                                           ? mbar_wait_bounded<true>(&ctl->cvt_full[st], cph, abort_flag, p.err,
                                                                     p.wait_limit_ns)
                                           : mbar_wait_bounded<false>(&ctl->cvt_full[st], cph, abort_flag, p.err,
                                                                      p.wait_limit_ns);
                        if (!w) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + st * STAGE2_BYTES);
                    const uint32_t sb = sa + A_HALF;
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        const uint64_t ad = smem_desc_sw128(sa + kk * a_step, a_lbo, 1024);
                        const uint64_t bd = smem_desc_sw128(sb + kk * b_step, b_lbo, 1024);
                        tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit_pair(&ctl->empty[st], 0x3);
                }
                if (!ok) break;
                tc_commit_pair(&ctl->acc_full[acc], 0x3);
            }
            if (!ok && issued) {
                tc_commit_pair(&ctl->drain, 0x1);
                const uint32_t a = smem_u32(&ctl->drain);
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < 100000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 4 + EPI_WARPS) {
        // ---------------------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 4;
        const int quad = warp & 3;
        const int half_slice = ew >> 2;
        constexpr int SLICES = EPI_WARPS / 4;
        uint32_t local = 0;
        OutStage os{smem + STAGES2 * STAGE2_BYTES + C::CONST_BYTES + ew * 2048, nullptr, false};
        int w_first, w_end, w_step;
        sched_range<SCHED>(sched, p.total_tiles, pair, npairs, w_first, w_end, w_step);
        for (int w = w_first; w < w_end; w += w_step, ++local) {
            const uint32_t acc = local & 1u;
            const uint32_t aph = (local >> 1) & 1u;
            const bool ok = mbar_wait_bounded(&ctl->acc_full[acc], aph, abort_flag, p.err, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const TileInfo ti = tile_info(p, sched_tile<SCHED>(sched, w));
            const int row0 = ti.tm * BM2 + 128 * static_cast<int>(rank) + quad * 32;
            const uint32_t taddr = tmem_base + acc * ACC_COLS + ((quad * 32) << 16);
            // a slice holds whole groups where the epilogue reduces over groups (then
            // some warps may have none)
            const Prob &pe = ti.pi ? p.pr[1] : p.pr[0];
            const bool reduces = ti.pi ? (EPI1 == 1 || EPI1 == 2) : (EPI0 == 1 || EPI0 == 2);
            int cols = ti.bn / SLICES;
            if (reduces && cols < pe.group) cols = pe.group;
            const int c_begin = half_slice * cols;
            const int c_end = c_begin + cols < ti.bn ? c_begin + cols : ti.bn;
            os.map = ti.pi ? &tmO1 : &tmO0;
            if (ti.pi == 0)
                drain_accumulator<EPI0, BITS>(p.pr[0], taddr, row0, ti.n0, c_begin, c_end, os);
            else
                drain_accumulator<EPI1, BITS>(p.pr[1], taddr, row0, ti.n0, c_begin, c_end, os);
            tc_fence_before();
            mbar_arrive_cluster(acc_empty0 + 8u * acc);
        }
        // the warp's output stores have completed (and read their shared memory)
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    } else if (CVT && warp >= 4 + EPI_WARPS) {
        // ---------------------------------------------------------- converters (both CTAs)
        // Warp cw converts the stages of B-from-codes problems whose global stage
        // counter is cw modulo CVT_WARPS (so it owns the ring slots cw, cw + CVT_WARPS,
        // ...: each slot's phases are waited on in order by one warp).  It gathers the
        // group constants of its next stage into registers before it waits for the
        // current one, so their L2 latency hides behind the other warps' stages.
        constexpr int CW = C::CVT_WARPS > 0 ? C::CVT_WARPS : 1;  // never 0 where this role runs (CVT)
        const int cw = warp - (4 + EPI_WARPS);
        float2 *tab = reinterpret_cast<float2 *>(smem + STAGES2 * STAGE2_BYTES) + cw * 256;
        const uint32_t cvt_full0 = map_to_rank(&ctl->cvt_full[0], 0);
        uint32_t cuse = 0;  // per owned slot: parity of its next code phase
        // this warp's next stage at or after (t, kb)
        auto seek = [&](StageWalk &w) -> bool {
            while (w.t < p.total_tiles) {
                if (w.kb == 0) {
                    w.ti = tile_info(p, w.t);
                    w.nkb = ((w.ti.pi ? p.pr[1].GK : p.pr[0].GK) + BK - 1) / BK;
                }
                const bool cvt = w.ti.pi ? p.pr[1].b_cvt : p.pr[0].b_cvt;
                if (cvt) {
                    const int skip = (cw - static_cast<int>(w.it % CW) + CW) % CW;
                    if (w.kb + skip < w.nkb) {
                        w.kb += skip;
                        w.it += static_cast<uint32_t>(skip);
                        return true;
                    }
                }
                w.it += static_cast<uint32_t>(w.nkb - w.kb);  // the rest of this tile
                w.t += npairs;
                w.kb = 0;
            }
            return false;
        };
        auto consts = [&](const StageWalk &w, StageConsts &c) {
            const Prob &pr = w.ti.pi ? p.pr[1] : p.pr[0];
            const int half = w.ti.bn / 2;
            gather_consts(pr, pr.b_mn, half, w.ti.n0 + half * static_cast<int>(rank), w.kb * BK, lane, c);
        };
        StageWalk cur{pair, 0, 0, 0u, TileInfo{}};
        bool have = seek(cur);
        StageConsts c_cur, c_nxt;
        if (have) consts(cur, c_cur);
        while (have) {
            StageWalk nxt = cur;
            ++nxt.kb;
            ++nxt.it;
            if (nxt.kb >= nxt.nkb) {
                nxt.t += npairs;
                nxt.kb = 0;
            }
            const bool have_nxt = seek(nxt);
            if (have_nxt) consts(nxt, c_nxt);
            const int st = cur.it % STAGES2;
            const uint32_t cph = (cuse >> st) & 1u;
            cuse ^= 1u << st;
            const Prob &pr = cur.ti.pi ? p.pr[1] : p.pr[0];
            const int half = cur.ti.bn / 2;
            // the constants into the warp's table (the previous stage's reads are done)
            __syncwarp();
            if (pr.gshift > 5) {
#pragma unroll
                for (int i = 0; i < kConstPerLane / 2; ++i) {
                    const float2 v = make_float2(c_cur.s[i], static_cast<float>(c_cur.zq[i]));
                    tab[2 * (lane + 32 * i)] = v;
                    tab[2 * (lane + 32 * i) + 1] = v;
                }
            } else {
#pragma unroll
                for (int i = 0; i < kConstPerLane; ++i)
                    tab[lane + 32 * i] = make_float2(c_cur.s[i], static_cast<float>(c_cur.zq[i]));
            }
            __syncwarp();
            const bool ok = mbar_wait_bounded(&ctl->cfull[st], cph, abort_flag, p.err, p.wait_limit_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            uint8_t *sb = smem + st * STAGE2_BYTES + A_HALF;
            convert_stage_warp<BITS>(sb + B_HALF, sb, pr.b_mn, half, pr.gshift == 5, lane, tab);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (p.cvt_cluster_scope)
                    mbar_arrive_cluster(cvt_full0 + 8u * static_cast<uint32_t>(st));
                else
                    mbar_arrive_cluster_cta_scope(cvt_full0 + 8u * static_cast<uint32_t>(st));
            }
            cur = nxt;
            have = have_nxt;
            c_cur = c_nxt;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair's MMAs may still read its shared memory
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encode() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// K-major operand stored [rows][GK] (row stride ld): box {64 k, box_rows}.
// MN-major operand stored [GK][rows] (row stride ld): box {64 mn, 64 k}.
cudaError_t make_map(CUtensorMap &map, const Operand &op, int64_t rows, int64_t GK, int box_rows) {
    cuuint64_t dims[2];
    cuuint32_t box[2];
    if (op.mn_major) {
        dims[0] = static_cast<cuuint64_t>(rows);
        dims[1] = static_cast<cuuint64_t>(GK);
        box[0] = MN_BOX;
        box[1] = BK;
    } else {
        dims[0] = static_cast<cuuint64_t>(GK);
        dims[1] = static_cast<cuuint64_t>(rows);
        box[0] = BK;
        box[1] = static_cast<cuuint32_t>(box_rows);
    }
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(op.ld) * 2};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(op.ptr), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int code_bits_stored(int bits) { return bits == 3 ? 8 : bits; }

// The packed codes of W-hat [w_rows, w_cols] as a 2-D byte tensor, one box per stage and
// CTA: K-major (forward) 64 codes of `half` rows; MN-major (input gradient) `half`
// codes of 64 rows (the contraction index).  No swizzle: the converter warps read it.
cudaError_t make_code_map(CUtensorMap &map, const CvtArgs &c, bool mn_major, int half) {
    const int cb = code_bits_stored(c.bits);
    const uint64_t row_bytes = static_cast<uint64_t>(c.w_cols) * cb / 8;
    cuuint64_t dims[2] = {row_bytes, static_cast<cuuint64_t>(c.w_rows)};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2];
    if (mn_major) {
        box[0] = static_cast<cuuint32_t>(half * cb / 8);
        box[1] = BK;
    } else {
        box[0] = static_cast<cuuint32_t>(BK * cb / 8);
        box[1] = static_cast<cuuint32_t>(half);
    }
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(c.codes), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// A bf16 output matrix [rows, cols] (row stride ld elements) as the target of the
// epilogue's TMA stores: one box of 32 x 32 per warp and chunk, 64-byte swizzle.
cudaError_t make_out_map(CUtensorMap &map, const void *ptr, int64_t rows, int64_t cols, int64_t ld) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

constexpr int kEpiWarps = 8;

template <int EPI0, int EPI1, int BITS>
cudaError_t launch_variant(const CUtensorMap (&maps)[6], const KParams &p, int grid, int dev_id,
                           cudaStream_t st) {
    auto kern = k_gemm_tc<EPI0, EPI1, BITS, kEpiWarps>;
    // The shared-memory opt-in is a per-device function attribute; setting it
    // twice from racing threads is harmless.
    static std::atomic<uint64_t> done{0};
    const uint64_t bit = 1ull << (dev_id & 63);
    if (!(done.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        done.fetch_or(bit);
    }
    return launch_pdl(kern, dim3(grid), dim3((4 + kEpiWarps) * 32), SMEM_BYTES, st, maps[0], maps[1], maps[2],
                      maps[3], p);
}

// Tile costs of a two-problem launch, for a host-made deal (tile_cost per tile of
// problem 0 and problem 1).
struct SchedSpec {
    int tiles0, tiles1;
    int cost0, cost1;
};

// Longest tiles first, each to the least-loaded pair (ties: the lowest pair); a pair
// takes its tiles in the order dealt.  The last deal is kept: a training loop
// launches the same shapes over and over.
bool build_sched(const SchedSpec &sp, int npairs, TileSched &out) {
    const int total = sp.tiles0 + sp.tiles1;
    if (npairs < 1 || npairs > kSchedPairs || total > kSchedTiles) return false;
    static std::mutex mu;
    static SchedSpec last{};
    static int last_pairs = 0;
    static TileSched cached;
    std::lock_guard<std::mutex> lock(mu);
    if (last_pairs == npairs && last.tiles0 == sp.tiles0 && last.tiles1 == sp.tiles1 && last.cost0 == sp.cost0 &&
        last.cost1 == sp.cost1) {
        out = cached;
        return true;
    }
    std::vector<std::vector<uint16_t>> lists(static_cast<size_t>(npairs));
    using Load = std::pair<int64_t, int>;  // (load, pair): the smallest on top
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int q = 0; q < npairs; ++q) heap.push({0, q});
    const bool first1 = sp.cost1 > sp.cost0;
    for (int k = 0; k < 2; ++k) {
        const int prob = (k == 0) == first1 ? 1 : 0;
        const int n = prob ? sp.tiles1 : sp.tiles0, base = prob ? sp.tiles0 : 0, cost = prob ? sp.cost1 : sp.cost0;
        for (int i = 0; i < n; ++i) {
            const Load top = heap.top();
            heap.pop();
            lists[static_cast<size_t>(top.second)].push_back(static_cast<uint16_t>(base + i));
            heap.push({top.first + cost, top.second});
        }
    }
    int pos = 0;
    for (int q = 0; q < npairs; ++q) {
        out.begin[q] = static_cast<uint16_t>(pos);
        for (uint16_t t : lists[static_cast<size_t>(q)]) out.tile[pos++] = t;
    }
    for (int q = npairs; q <= kSchedPairs; ++q) out.begin[q] = static_cast<uint16_t>(pos);
    last = sp;
    last_pairs = npairs;
    cached = out;
    return true;
}

template <int EPI0, int EPI1, int BITS, int CVT = 0, int EW = 8, int SCHED = 0>
cudaError_t launch_pair_variant(const CUtensorMap (&maps)[6], const KParams &p, int grid, int dev_id,
                                cudaStream_t st, const SchedSpec *spec = nullptr) {
    using C = PairCfg<CVT, BITS, CVT ? 4 : EW>;
    auto kern = k_gemm_tc2<EPI0, EPI1, BITS, C::EPI_WARPS, CVT, SCHED>;
    static std::atomic<uint64_t> done{0};
    const uint64_t bit = 1ull << (dev_id & 63);
    if (!(done.load() & bit)) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        done.fetch_or(bit);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3((4 + C::EPI_WARPS + C::CVT_WARPS) * 32, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Persistent pairs: no more clusters than can be resident at once.
    static std::atomic<int> resident[64];
    int n = resident[dev_id & 63].load();
    if (n == 0) {
        cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return e;
        if (n <= 0) return cudaErrorInvalidConfiguration;
        resident[dev_id & 63].store(n);
    }
    const int launched = std::min(grid, 2 * n);
    SchedParam<SCHED> sc{};
    if constexpr (SCHED != 0) {
        if (!spec || !build_sched(*spec, launched / 2, sc)) return cudaErrorInvalidValue;
    }
    return launch_pdl_ex(kern, dim3(static_cast<unsigned>(launched)), cfg.blockDim, C::SMEM, st, attr[0], maps[0],
                         maps[1], maps[2], maps[3], maps[4], maps[5], p, sc);
}

// EQAT_GEMM_SCHED=0: grouped launches deal tiles round-robin always (measurement aid).
bool sched_disabled() {
    static const bool off = [] {
        const char *v = std::getenv("EQAT_GEMM_SCHED");
        return v && v[0] == '0';
    }();
    return off;
}

// EQAT_CVT_SCOPE=cta: converter hand-off at CTA scope (measurement aid).
bool cvt_scope_cluster() {
    static const bool on = [] {
        const char *v = std::getenv("EQAT_CVT_SCOPE");
        return !(v && v[0] == 'c' && v[1] == 't');
    }();
    return on;
}

// EQAT_GEMM_SPLIT_TAIL=0 keeps the last wave whole (measurement aid).
bool split_tail_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("EQAT_GEMM_SPLIT_TAIL");
        return !(v && v[0] == '0');
    }();
    return on;
}

int *device_error_ptr() {
    int *ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&ptr), g_dev_error) != cudaSuccess) return nullptr;
    return ptr;
}

// tile_m: rows of an output tile (128 for one CTA, 256 for a CTA pair, where each
// CTA loads 128 rows of A and bn / 2 rows of B).
cudaError_t fill_prob(Prob &q, const GemmProblem &g, int tile_begin, int bn, int tile_m, CUtensorMap &ma,
                      CUtensorMap &mb) {
    const int64_t GM = g.GM, GN = g.GN, GK = g.GK;
    if (GM <= 0 || GN <= 0 || GK <= 0) return cudaErrorInvalidValue;
    if (GM > INT32_MAX - BM2 || GN > INT32_MAX - BN || GK > INT32_MAX - BK) return cudaErrorInvalidValue;
    cudaError_t e;
    const bool pair = tile_m == BM2;
    if ((e = make_map(ma, g.A, GM, GK, BM)) != cudaSuccess) return e;
    if (g.cvt.on) {
        if (!pair) return cudaErrorInvalidValue;
        if ((e = make_code_map(mb, g.cvt, g.B.mn_major, bn / 2)) != cudaSuccess) return e;
    } else if ((e = make_map(mb, g.B, GN, GK, pair ? bn / 2 : bn)) != cudaSuccess) {
        return e;
    }
    q = Prob{};
    q.GM = static_cast<int>(GM);
    q.GN = static_cast<int>(GN);
    q.GK = static_cast<int>(GK);
    q.tiles_m = static_cast<int>((GM + tile_m - 1) / tile_m);
    q.tiles_n = static_cast<int>((GN + bn - 1) / bn);
    q.bn = bn;
    q.tile_begin = tile_begin;
    // Consecutive CTAs share the operand whose tiles are the larger total, so
    // that the smaller one stays hot in L2 while the larger streams once.
    q.m_fast = (GM <= GN) ? 1 : 0;
    q.a_mn = g.A.mn_major ? 1 : 0;
    q.b_mn = g.B.mn_major ? 1 : 0;
    const EpiArgs &epi = g.epi;
    q.out = epi.out;
    q.ldo = epi.ldo;
    q.W = epi.W;
    q.s = epi.s;
    q.z = epi.z;
    q.dW = epi.dW;
    q.ds = epi.ds;
    q.dz = epi.dz;
    q.codes = epi.codes;
    q.zq = epi.zq;
    q.s_e2e = epi.s_e2e;
    q.target = epi.target;
    q.loss = epi.loss;
    q.mse_scale = epi.mse_scale;
    q.s_f16 = epi.s_f16 ? 1 : 0;
    q.clamp_pass = epi.clamp_pass ? 1 : 0;
    q.group = epi.group;
    q.gshift = epi.group == 32 ? 5 : epi.group == 64 ? 6 : 7;
    q.Q = static_cast<float>((1 << epi.bits) - 1);
    if (g.cvt.on) {
        if (g.cvt.w_rows > INT32_MAX || g.cvt.w_cols > INT32_MAX) return cudaErrorInvalidValue;
        q.b_cvt = 1;
        q.w_rows = static_cast<int>(g.cvt.w_rows);
        q.w_cols = static_cast<int>(g.cvt.w_cols);
        q.w_groups = static_cast<int>(g.cvt.w_cols / g.cvt.group);
        q.cvt_zq = g.cvt.zq;
        q.cvt_s = g.cvt.s;
        q.cvt_s_f16 = g.cvt.s_f16 ? 1 : 0;
        q.gshift = g.cvt.group == 32 ? 5 : g.cvt.group == 64 ? 6 : 7;
        q.group = g.cvt.group;
    }
    return cudaSuccess;
}

struct Tiling {
    bool pair;  // 256-row tiles on CTA pairs, else 128-row tiles on one CTA
    int bn;     // N-tile width, 128 or 256
};

// Tile shape for a launch, from a wave model: estimated time = waves x the time
// one wave of that shape takes, relative to a wave of 128 x 256 tiles on single
// CTAs.  Measured on B200 (4096^3 forward, CUDA events):
//   one CTA,  128 x 128: 0.72  (42% more time per FLOP: operand bytes per FLOP
//                               read from shared memory)
//   CTA pair, 256 x 256: 0.89  (B split over the two SMs: a third fewer operand
//                               bytes per FLOP; the same per-SM work per wave)
//   CTA pair, 256 x 128: 0.89 x 0.66 (0.64-0.69 of a 256 x 256 pair wave on four shapes)
// A pair covers 256 rows, so concurrent tiles are half the SM count.  Group
// reductions need a whole group inside one epilogue slice (bn / 2 columns).
// EQAT_GEMM_BN=128|256 and EQAT_GEMM_PAIR=0|1 force a choice (measurement aid).
Tiling choose_tiling(const GemmProblem *probs, int nprob, int sms) {
    bool narrow_ok = true;
    for (int i = 0; i < nprob; ++i)
        if (probs[i].epi.kind != Epi::kStore && probs[i].epi.group > 64) narrow_ok = false;
    static const int forced_bn = [] {
        const char *v = std::getenv("EQAT_GEMM_BN");
        return v ? std::atoi(v) : 0;
    }();
    static const int forced_pair = [] {
        const char *v = std::getenv("EQAT_GEMM_PAIR");
        return v ? std::atoi(v) : -1;
    }();
    auto estimate = [&](bool pair, int bn) {
        const int64_t tile_m = pair ? BM2 : BM;
        const int64_t units = pair ? sms / 2 : sms;
        int64_t tiles = 0;
        for (int i = 0; i < nprob; ++i)
            tiles += ((probs[i].GM + tile_m - 1) / tile_m) * ((probs[i].GN + bn - 1) / bn);
        const int64_t waves = (tiles + units - 1) / units;
        const double cost = pair ? (bn == 256 ? 0.89 : 0.89 * 0.66) : (bn == 256 ? 1.0 : 0.72);
        return static_cast<double>(waves) * cost;
    };
    bool need_pair = false;  // B made from codes on load: the pair kernel only
    for (int i = 0; i < nprob; ++i) need_pair |= probs[i].cvt.on;
    Tiling best{need_pair, 256};
    double best_t = 1e300;
    for (int pair = 0; pair < 2; ++pair) {
        if (need_pair && !pair) continue;
        if (!need_pair && forced_pair >= 0 && pair != (forced_pair != 0)) continue;
        for (int bn = 256; bn >= 128; bn -= 128) {
            if (bn == 128 && (!narrow_ok || forced_bn == 256)) continue;
            if (bn == 256 && forced_bn == 128 && narrow_ok) continue;
            const double t = estimate(pair != 0, bn);
            if (t < best_t) {
                best_t = t;
                best = Tiling{pair != 0, bn};
            }
        }
    }
    return best;
}

}  // namespace

int *device_error_word() { return device_error_ptr(); }

bool cvt_supported(int64_t w_rows, int64_t w_cols, int bits, int group) {
    if (w_rows <= 0 || w_cols <= 0 || w_rows > INT32_MAX || w_cols > INT32_MAX) return false;
    if (bits != 2 && bits != 3 && bits != 4) return false;
    if (group != 32 && group != 64 && group != 128) return false;
    const int64_t row_bytes = w_cols * code_bits_stored(bits) / 8;
    return w_cols % group == 0 && row_bytes % 16 == 0;
}

cudaError_t encode_map_2d(CUtensorMap &map, CUtensorMapDataType type, const void *base, uint64_t inner,
                          uint64_t outer, uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swizzle) {
    cudaError_t e = get_encode();
    if (e != cudaSuccess) return e;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(&map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_gemm_tc_group(const GemmProblem *probs, int nprob, const DeviceInfo &dev,
                                 cudaStream_t st) {
    if (nprob < 1 || nprob > 2) return cudaErrorInvalidValue;
    for (int i = 0; i < nprob; ++i) {
        const EpiArgs &e = probs[i].epi;
        if (e.kind == Epi::kStore && e.out_f32) return cudaErrorInvalidValue;
        if (e.kind == Epi::kFqGrad && e.w_f32) return cudaErrorInvalidValue;
        if (i == 1 && e.kind != Epi::kStore) return cudaErrorInvalidValue;
    }
    cudaError_t e = get_encode();
    if (e != cudaSuccess) return e;
    CUtensorMap maps[6];  // A, B of problem 0; A, B of problem 1; the outputs of problems 0 and 1
    KParams p{};
    int tiles = 0;
    const Tiling tiling = choose_tiling(probs, nprob, dev.sm_count);
    const bool pair = tiling.pair;
    const int tile_m = pair ? BM2 : BM;
    const int units = pair ? dev.sm_count / 2 : dev.sm_count;  // concurrent tiles
    const int bn = tiling.bn;
    for (int i = 0; i < nprob; ++i) {
        if ((e = fill_prob(p.pr[i], probs[i], tiles, bn, tile_m, maps[2 * i], maps[2 * i + 1])) != cudaSuccess)
            return e;
        const int64_t t = static_cast<int64_t>(p.pr[i].tiles_m) * p.pr[i].tiles_n;
        if (tiles + t > INT32_MAX) return cudaErrorInvalidValue;
        tiles += static_cast<int>(t);
    }
    if (nprob == 1) {  // unused slots still travel as kernel parameters
        maps[2] = maps[0];
        maps[3] = maps[1];
    }
    // The epilogue's output matrices (bf16 store, MSE and straight-through dW).
    for (int i = 0; i < 2; ++i) {
        maps[4 + i] = maps[0];  // placeholder: no output matrix
        if (i >= nprob) continue;
        const EpiArgs &ea = probs[i].epi;
        if (ea.kind == Epi::kStore || ea.kind == Epi::kMse) {
            if ((e = make_out_map(maps[4 + i], ea.out, probs[i].GM, probs[i].GN, ea.ldo)) != cudaSuccess) return e;
        } else if (ea.kind == Epi::kFqGrad && ea.dW) {
            if ((e = make_out_map(maps[4 + i], ea.dW, probs[i].GM, probs[i].GN, probs[i].GN)) != cudaSuccess)
                return e;
        }
    }
    p.nprob = nprob;
    p.total_tiles = tiles;
    p.split_begin = -1;
    // A one-problem pair launch whose last wave is partial, at most half full: split
    // that wave's 256-wide tiles into 128-wide halves (one wave of narrow tiles costs
    // about 0.66 of a wide one).  B must be K-major (one box per half) and the
    // epilogue's groups must fit a 64-column slice.
    if (pair && nprob == 1 && bn == 256 && !probs[0].B.mn_major && split_tail_enabled() &&
        (probs[0].epi.kind == Epi::kStore || probs[0].epi.kind == Epi::kMse || probs[0].epi.group <= 64)) {
        const int full = tiles / units, tail = tiles % units;
        if (full >= 1 && tail > 0 && 2 * tail <= units) {
            e = probs[0].cvt.on ? make_code_map(maps[3], probs[0].cvt, false, bn / 4)
                                : make_map(maps[3], probs[0].B, probs[0].GN, probs[0].GK, bn / 4);
            if (e != cudaSuccess) return e;
            p.split_begin = full * units;
            p.total_tiles = full * units + 2 * tail;
        }
    }
    p.err = device_error_ptr();
    if (!p.err) return cudaErrorInvalidSymbol;
    p.wait_limit_ns = kWaitLimitNs;
    p.cvt_cluster_scope = cvt_scope_cluster() ? 1 : 0;
    bool any_cvt = false;
    int cvt_bits = 2;
    for (int i = 0; i < nprob; ++i)
        if (probs[i].cvt.on) {
            if (any_cvt && probs[i].cvt.bits != cvt_bits) return cudaErrorInvalidValue;
            any_cvt = true;
            cvt_bits = probs[i].cvt.bits;
        }
    if (pair && any_cvt) {
        // B from codes: the E2E-QP forward (one problem, plain store) or backward
        // (the ds epilogue on dY^T X, then dX = dY W-hat with W-hat made on load)
        const int grid = 2 * std::min(p.total_tiles, units);
        if (probs[0].epi.kind == Epi::kE2eDs && probs[0].epi.bits != cvt_bits) return cudaErrorInvalidValue;
        const bool ds = probs[0].epi.kind == Epi::kE2eDs;
        if (!ds && (probs[0].epi.kind != Epi::kStore || nprob > 1)) return cudaErrorInvalidValue;
        switch (cvt_bits) {
            case 2: return ds ? launch_pair_variant<2, 0, 2, 1>(maps, p, grid, dev.device, st)
                              : launch_pair_variant<0, 0, 2, 1>(maps, p, grid, dev.device, st);
            case 3: return ds ? launch_pair_variant<2, 0, 3, 1>(maps, p, grid, dev.device, st)
                              : launch_pair_variant<0, 0, 3, 1>(maps, p, grid, dev.device, st);
            case 4: return ds ? launch_pair_variant<2, 0, 4, 1>(maps, p, grid, dev.device, st)
                              : launch_pair_variant<0, 0, 4, 1>(maps, p, grid, dev.device, st);
            default: return cudaErrorInvalidValue;
        }
    }
    if (any_cvt) return cudaErrorInvalidValue;
    if (pair) {
        const int grid = 2 * std::min(p.total_tiles, units);
        // Two problems whose tiles differ in cost by 2x or more (main-loop k-blocks,
        // or the reducing epilogue's time where that is longer, about 24 k-blocks)
        // get a host-made deal instead of round-robin.
        SchedSpec spec{};
        bool sched = false;
        if (nprob == 2 && !sched_disabled()) {
            auto cost = [](const Prob &q, bool reduces) {
                const int nkb = (q.GK + BK - 1) / BK;
                return reduces ? std::max(nkb, 24) : nkb;
            };
            spec = SchedSpec{p.pr[0].tiles_m * p.pr[0].tiles_n, p.pr[1].tiles_m * p.pr[1].tiles_n,
                             cost(p.pr[0], probs[0].epi.kind != Epi::kStore), cost(p.pr[1], probs[1].epi.kind != Epi::kStore)};
            const int lo = std::min(spec.cost0, spec.cost1), hi = std::max(spec.cost0, spec.cost1);
            sched = hi >= 2 * lo && spec.tiles0 + spec.tiles1 <= kSchedTiles;
        }
        switch (probs[0].epi.kind) {
            case Epi::kStore:
                if (nprob > 1) return cudaErrorInvalidValue;
                return launch_pair_variant<0, 0, 2>(maps, p, grid, dev.device, st);
            case Epi::kFqGrad:
                // The straight-through epilogue outlasts a main loop 2048 deep with eight
                // warps (per-tile timestamps on the 70B gate backward: 13.7 us against
                // 10 us); sixteen keep up there (3% off that backward) but cost 1.7% on
                // 4096-deep contractions, where eight already hide behind the main loop.
                if (probs[0].GK <= 2048)
                    return sched ? launch_pair_variant<1, 0, 2, 0, 16, 1>(maps, p, grid, dev.device, st, &spec)
                                 : launch_pair_variant<1, 0, 2, 0, 16>(maps, p, grid, dev.device, st);
                return sched ? launch_pair_variant<1, 0, 2, 0, 8, 1>(maps, p, grid, dev.device, st, &spec)
                             : launch_pair_variant<1, 0, 2>(maps, p, grid, dev.device, st);
            case Epi::kE2eDs:
                switch (probs[0].epi.bits) {
                    case 2: return sched ? launch_pair_variant<2, 0, 2, 0, 8, 1>(maps, p, grid, dev.device, st, &spec)
                                         : launch_pair_variant<2, 0, 2>(maps, p, grid, dev.device, st);
                    case 3: return sched ? launch_pair_variant<2, 0, 3, 0, 8, 1>(maps, p, grid, dev.device, st, &spec)
                                         : launch_pair_variant<2, 0, 3>(maps, p, grid, dev.device, st);
                    case 4: return sched ? launch_pair_variant<2, 0, 4, 0, 8, 1>(maps, p, grid, dev.device, st, &spec)
                                         : launch_pair_variant<2, 0, 4>(maps, p, grid, dev.device, st);
                    default: return cudaErrorInvalidValue;
                }
            case Epi::kMse:
                if (nprob > 1) return cudaErrorInvalidValue;
                return launch_pair_variant<3, 0, 2>(maps, p, grid, dev.device, st);
        }
        return cudaErrorInvalidValue;
    }
    const int grid = std::min(tiles, dev.sm_count);
    switch (probs[0].epi.kind) {
        case Epi::kStore:
            if (nprob > 1) return cudaErrorInvalidValue;  // two plain contractions: launch separately
            return launch_variant<0, 0, 2>(maps, p, grid, dev.device, st);
        case Epi::kFqGrad:
            return launch_variant<1, 0, 2>(maps, p, grid, dev.device, st);
        case Epi::kE2eDs:
            switch (probs[0].epi.bits) {
                case 2: return launch_variant<2, 0, 2>(maps, p, grid, dev.device, st);
                case 3: return launch_variant<2, 0, 3>(maps, p, grid, dev.device, st);
                case 4: return launch_variant<2, 0, 4>(maps, p, grid, dev.device, st);
                default: return cudaErrorInvalidValue;
            }
        case Epi::kMse:
            if (nprob > 1) return cudaErrorInvalidValue;
            return launch_variant<3, 0, 2>(maps, p, grid, dev.device, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_tc(const Operand &A, const Operand &B, int64_t GM, int64_t GN, int64_t GK,
                           const EpiArgs &epi, const DeviceInfo &dev, cudaStream_t st) {
    if (GM <= 0 || GN <= 0 || GK <= 0) return cudaSuccess;
    GemmProblem g{A, B, GM, GN, GK, epi};
    return launch_gemm_tc_group(&g, 1, dev, st);
}

// ---------------------------------------------------------------------------- error word

cudaError_t read_and_clear_device_error(int &value) {
    value = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&value, g_dev_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (value != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int));
    }
    return e;
}

namespace {
// One thread waits on a barrier that nothing arrives on; the bounded wait runs
// out, records the timeout and the kernel returns.
__global__ void k_selftest_bounded_wait(int *err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait_bounded(&bar, 0, &abort_flag, err, limit_ns);
}
}  // namespace

cudaError_t launch_selftest_bounded_wait(uint64_t timeout_ns, cudaStream_t st) {
    int *err = device_error_ptr();
    if (!err) return cudaErrorInvalidSymbol;
    k_selftest_bounded_wait<<<1, 32, 0, st>>>(err, timeout_ns);
    return cudaGetLastError();
}

}  // namespace eqat
