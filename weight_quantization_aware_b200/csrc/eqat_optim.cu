// The Block-AP parameter update: AdamW with decoupled weight decay over all
// tensors of a block in one launch (modelfoundations note, Phase 1 and "Paper vs.
// code": AdamW, the weights and the quantization parameters in separate
// learning-rate groups on cosine schedules), and the fp32 form of the
// reconstruction-loss gradient.
//
// AdamW is HBM-bound: per parameter it reads p, g, m, v and writes p, m, v (and a
// bf16 copy of W for the next forward), 28 bytes for a bf16-gradient weight.  One
// launch walks 4096-element chunks of every tensor; each thread moves four
// elements per step with 16-byte accesses.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "eqat_internal.h"

namespace eqat {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 4096;  // elements per block iteration: 256 threads x 4 x 4

struct AdamwParams {
    AdamwSeg seg[kAdamwMaxSegs];
    int64_t chunk_begin[kAdamwMaxSegs + 1];  // prefix sums of chunks per segment
    int nseg;
};

__device__ __forceinline__ void adamw_elem(const AdamwSeg &s, float g, float &p, float &m, float &v) {
    p = __fmul_rn(p, s.decay);
    m = fmaf(s.b1, m, __fmul_rn(s.omb1, g));
    v = fmaf(s.b2, v, __fmul_rn(__fmul_rn(s.omb2, g), g));
    const float denom = __fadd_rn(__fmul_rn(sqrtf(v), s.inv_sqrt_bc2), s.eps);
    p = __fsub_rn(p, __fmul_rn(s.step_size, __fdiv_rn(m, denom)));
}

__global__ void __launch_bounds__(kThreads) k_adamw(const __grid_constant__ AdamwParams P) {
    const int64_t total = P.chunk_begin[P.nseg];
    for (int64_t c = blockIdx.x; c < total; c += gridDim.x) {
        int si = 0;
        while (si + 1 < P.nseg && c >= P.chunk_begin[si + 1]) ++si;
        const AdamwSeg &s = P.seg[si];
        const int64_t base = (c - P.chunk_begin[si]) * kChunk;
#pragma unroll
        for (int r = 0; r < kChunk / (kThreads * 4); ++r) {
            const int64_t i = base + (static_cast<int64_t>(r) * kThreads + threadIdx.x) * 4;
            if (i + 4 <= s.n) {
                float4 p = *reinterpret_cast<const float4 *>(s.p + i);
                float4 m = *reinterpret_cast<const float4 *>(s.m + i);
                float4 v = *reinterpret_cast<const float4 *>(s.v + i);
                float g[4];
                if (s.g_bf16) {
                    const uint2 raw = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(s.g) + i);
                    const __nv_bfloat162 g01 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
                    const __nv_bfloat162 g23 = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
                    g[0] = __low2float(g01);
                    g[1] = __high2float(g01);
                    g[2] = __low2float(g23);
                    g[3] = __high2float(g23);
                } else {
                    const float4 gf = *reinterpret_cast<const float4 *>(static_cast<const float *>(s.g) + i);
                    g[0] = gf.x;
                    g[1] = gf.y;
                    g[2] = gf.z;
                    g[3] = gf.w;
                }
                adamw_elem(s, g[0], p.x, m.x, v.x);
                adamw_elem(s, g[1], p.y, m.y, v.y);
                adamw_elem(s, g[2], p.z, m.z, v.z);
                adamw_elem(s, g[3], p.w, m.w, v.w);
                *reinterpret_cast<float4 *>(s.p + i) = p;
                *reinterpret_cast<float4 *>(s.m + i) = m;
                *reinterpret_cast<float4 *>(s.v + i) = v;
                if (s.copy) {
                    if (s.copy_bf16) {
                        uint2 o;
                        const __nv_bfloat162 a = __floats2bfloat162_rn(p.x, p.y), b = __floats2bfloat162_rn(p.z, p.w);
                        o.x = *reinterpret_cast<const uint32_t *>(&a);
                        o.y = *reinterpret_cast<const uint32_t *>(&b);
                        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(s.copy) + i) = o;
                    } else {
                        *reinterpret_cast<float4 *>(static_cast<float *>(s.copy) + i) = p;
                    }
                }
            } else {
                for (int64_t j = i; j < s.n && j < i + 4; ++j) {
                    float p = s.p[j], m = s.m[j], v = s.v[j];
                    const float g = s.g_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(s.g)[j])
                                             : static_cast<const float *>(s.g)[j];
                    adamw_elem(s, g, p, m, v);
                    s.p[j] = p;
                    s.m[j] = m;
                    s.v[j] = v;
                    if (s.copy) {
                        if (s.copy_bf16)
                            static_cast<__nv_bfloat16 *>(s.copy)[j] = __float2bfloat16_rn(p);
                        else
                            static_cast<float *>(s.copy)[j] = p;
                    }
                }
            }
        }
    }
}

// dY = scale (dY - T) in place; the block's sum of (dY - T)^2 goes to *loss.
__global__ void __launch_bounds__(kThreads) k_mse_f32(float *__restrict__ dY, const float *__restrict__ T,
                                                      int64_t n, float scale, double *__restrict__ loss) {
    __shared__ double red[kThreads / 32];
    double acc = 0.0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const float d = __fsub_rn(dY[i], T[i]);
        acc += static_cast<double>(d) * d;
        dY[i] = __fmul_rn(d, scale);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) a += red[w];
        atomicAdd(loss, a * (0.5 * static_cast<double>(scale)));  // scale = 2 / n: the mean
    }
}

// Y = 0 (K == 0): dY = scale (0 - T) in bf16, *loss += sum T^2 scale / 2.
__global__ void __launch_bounds__(kThreads) k_mse_zero_bf16(__nv_bfloat16 *__restrict__ dY,
                                                            const __nv_bfloat16 *__restrict__ T, int64_t n,
                                                            float scale, double *__restrict__ loss) {
    double acc = 0.0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const float d = -__bfloat162float(T[i]);
        acc += static_cast<double>(d) * d;
        dY[i] = __float2bfloat16_rn(__fmul_rn(d, scale));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if ((threadIdx.x & 31) == 0) atomicAdd(loss, acc * (0.5 * static_cast<double>(scale)));
}

}  // namespace

cudaError_t launch_adamw(const AdamwSeg *segs, int nseg, const DeviceInfo &dev, cudaStream_t st) {
    if (nseg < 1 || nseg > kAdamwMaxSegs) return cudaErrorInvalidValue;
    AdamwParams P{};
    P.nseg = nseg;
    P.chunk_begin[0] = 0;
    for (int i = 0; i < nseg; ++i) {
        P.seg[i] = segs[i];
        P.chunk_begin[i + 1] = P.chunk_begin[i] + (segs[i].n + kChunk - 1) / kChunk;
    }
    const int64_t total = P.chunk_begin[nseg];
    if (total == 0) return cudaSuccess;
    const int grid = static_cast<int>(std::min<int64_t>(total, static_cast<int64_t>(dev.sm_count) * 8));
    k_adamw<<<grid, kThreads, 0, st>>>(P);
    return cudaGetLastError();
}

cudaError_t launch_mse_zero_bf16(void *dY, const void *target, int64_t n, float scale, double *loss,
                                 const DeviceInfo &dev, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int grid = static_cast<int>(std::min<int64_t>((n + kThreads - 1) / kThreads, dev.sm_count * 4));
    k_mse_zero_bf16<<<grid, kThreads, 0, st>>>(static_cast<__nv_bfloat16 *>(dY),
                                               static_cast<const __nv_bfloat16 *>(target), n, scale, loss);
    return cudaGetLastError();
}

cudaError_t launch_mse_f32(float *dY, const float *target, int64_t n, float scale, double *loss,
                           const DeviceInfo &dev, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int grid = static_cast<int>(std::min<int64_t>((n + kThreads - 1) / kThreads, dev.sm_count * 4));
    k_mse_f32<<<grid, kThreads, 0, st>>>(dY, target, n, scale, loss);
    return cudaGetLastError();
}

}  // namespace eqat
