// fp32 contractions on the CUDA cores for layers stored in fp32 (the pages train
// each Block-AP block in fp32: modelfoundations note, "Paper vs. code").  bf16
// tensor-core operands would spend most of the 1e-3 budget of ds/dz on operand
// rounding, so this mode keeps every operand in fp32.
//
// D[GM, GN] = sum_k A(m, k) B(n, k) with 64x64 output tiles, 16-deep k slices
// staged in shared memory and a 4x4 register block per thread.  Non-store
// epilogues run as a second pass over D kept in fp32 scratch.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "eqat_internal.h"
#include "eqat_qmath.cuh"

namespace eqat {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

// A(m, k) = A[m * a_sm + k * a_sk]; B(n, k) = B[n * b_sn + k * b_sk].
__global__ void __launch_bounds__(256)
    k_gemm_f32(const float *__restrict__ A, int64_t a_sm, int64_t a_sk, const float *__restrict__ B,
               int64_t b_sn, int64_t b_sk, float *__restrict__ C, int64_t ldc, int GM, int GN, int GK) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < GK; k0 += TK) {
        for (int i = tid; i < TK * TM; i += 256) {
            const int kk = i / TM, mm = i % TM;
            const int m = m0 + mm, k = k0 + kk;
            As[kk][mm] = (m < GM && k < GK) ? A[m * a_sm + k * a_sk] : 0.0f;
        }
        for (int i = tid; i < TK * TN; i += 256) {
            const int kk = i / TN, nn = i % TN;
            const int n = n0 + nn, k = k0 + kk;
            Bs[kk][nn] = (n < GN && k < GK) ? B[n * b_sn + k * b_sk] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= GM) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < GN) C[static_cast<int64_t>(m) * ldc + n] = acc[i][j];
        }
    }
}

// Block-AP straight-through epilogue over dW-hat [N, K] (fp32): one thread per
// group.  Same arithmetic as the fused tensor-core epilogue.
__global__ void k_ste_epilogue_f32(const float *__restrict__ W, const float *__restrict__ s,
                                   const float *__restrict__ z, const float *__restrict__ dwh,
                                   float *__restrict__ dW, float *__restrict__ ds,
                                   float *__restrict__ dz, int64_t n_groups, int group, float Q,
                                   bool clamp_pass) {
    const int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gi >= n_groups) return;
    const float sc = s[gi];
    const float rcp = __frcp_rn(sc);
    const float zr = rintf(z[gi]);
    float acc_s = 0.0f, acc_z = 0.0f;
    const int64_t e0 = gi * group;
    for (int i = 0; i < group; ++i) {
        const float d = dwh[e0 + i];
        const QuantElem e = quant_elem(W[e0 + i], sc, rcp, zr, Q);
        const bool keep = e.inside || clamp_pass;
        acc_s = fmaf(d, __fsub_rn(__fsub_rn(e.c, zr), keep ? e.u : 0.0f), acc_s);
        acc_z += keep ? 0.0f : d;
        if (dW) dW[e0 + i] = keep ? d : 0.0f;
    }
    if (ds) ds[gi] = acc_s;
    if (dz) dz[gi] = -sc * acc_z;
}

__device__ __forceinline__ uint32_t code_at(const uint8_t *codes, int64_t e, int bits) {
    if (bits == 2) return (codes[e / 4] >> (2 * (e % 4))) & 3u;
    if (bits == 4) return (codes[e / 2] >> (4 * (e % 2))) & 15u;
    return codes[e];
}

// E2E-QP epilogue: ds = sum_group dW-hat (W_q - zq), dz = -s sum_group dW-hat
// (both nullable; s fp32 or fp16, read for dz only); one thread per group.
__global__ void k_e2e_ds_epilogue_f32(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ zq,
                                      const float *__restrict__ dwh, float *__restrict__ ds,
                                      float *__restrict__ dz, const void *__restrict__ s, bool s_f16,
                                      int64_t n_groups, int group, int bits) {
    const int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gi >= n_groups) return;
    const float zf = static_cast<float>(zq[gi]);
    float acc = 0.0f, sum = 0.0f;
    const int64_t e0 = gi * group;
    for (int i = 0; i < group; ++i) {
        const float d = dwh[e0 + i];
        acc = fmaf(d, __fsub_rn(static_cast<float>(code_at(codes, e0 + i, bits)), zf), acc);
        sum += d;
    }
    if (ds) ds[gi] = acc;
    if (dz) {
        const float sc = s_f16 ? __half2float(static_cast<const __half *>(s)[gi]) : static_cast<const float *>(s)[gi];
        dz[gi] = -sc * sum;
    }
}

}  // namespace

cudaError_t launch_gemm_f32(const Operand &A, const Operand &B, int64_t GM, int64_t GN, int64_t GK,
                            const EpiArgs &epi, float *d_scratch, const DeviceInfo &dev,
                            cudaStream_t st) {
    (void)dev;
    if (GM <= 0 || GN <= 0 || GK <= 0) return cudaSuccess;
    if (GM > INT32_MAX || GN > INT32_MAX || GK > INT32_MAX) return cudaErrorInvalidValue;
    const int64_t a_sm = A.mn_major ? 1 : A.ld, a_sk = A.mn_major ? A.ld : 1;
    const int64_t b_sn = B.mn_major ? 1 : B.ld, b_sk = B.mn_major ? B.ld : 1;
    float *C;
    int64_t ldc;
    if (epi.kind == Epi::kStore) {
        if (!epi.out_f32) return cudaErrorInvalidValue;
        C = static_cast<float *>(epi.out);
        ldc = epi.ldo;
    } else {
        C = d_scratch;
        ldc = GN;
    }
    dim3 grid(static_cast<unsigned>((GN + TN - 1) / TN), static_cast<unsigned>((GM + TM - 1) / TM));
    if (grid.y > 65535u) return cudaErrorInvalidValue;
    k_gemm_f32<<<grid, 256, 0, st>>>(static_cast<const float *>(A.ptr), a_sm, a_sk,
                                     static_cast<const float *>(B.ptr), b_sn, b_sk, C, ldc,
                                     static_cast<int>(GM), static_cast<int>(GN), static_cast<int>(GK));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || epi.kind == Epi::kStore) return e;
    const int64_t n_groups = GM * (GN / epi.group);
    if (n_groups == 0) return cudaSuccess;
    const int threads = 128;
    const unsigned blocks = static_cast<unsigned>((n_groups + threads - 1) / threads);
    if (epi.kind == Epi::kFqGrad) {
        if (!epi.w_f32) return cudaErrorInvalidValue;
        k_ste_epilogue_f32<<<blocks, threads, 0, st>>>(
            static_cast<const float *>(epi.W), epi.s, epi.z, d_scratch, static_cast<float *>(epi.dW),
            epi.ds, epi.dz, n_groups, epi.group, static_cast<float>((1 << epi.bits) - 1), epi.clamp_pass);
    } else {
        k_e2e_ds_epilogue_f32<<<blocks, threads, 0, st>>>(epi.codes, epi.zq, d_scratch, epi.ds, epi.dz, epi.s_e2e,
                                                          epi.s_f16, n_groups, epi.group, epi.bits);
    }
    return cudaGetLastError();
}

}  // namespace eqat
