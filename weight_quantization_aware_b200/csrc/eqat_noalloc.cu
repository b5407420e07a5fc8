// eqat_fq_linear_fwd_noalloc: the Block-AP forward for callers that cannot
// allocate device memory and cannot hand the library a workspace.
//
// Who needs it: code that only ever receives its input and output buffers from
// a host framework (custom-operator and plugin interfaces without a workspace
// hook), processes that must not call cudaMalloc once they are running (it can
// synchronise the whole device and stall latency-critical work), and callers
// whose device memory is owned by an allocator that the library cannot reach.
//
// The forward needs W-hat (the fake-quantized weight) between the quantizer
// prepass and the tensor-core contraction.  Here that scratch is a fixed array in
// device global memory that belongs to the library: it is created when the
// library's device code is loaded on a GPU and stays there until the process
// exits, on every GPU that loads the library.  The caller still passes X, W, s, z
// and Y.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/eqat.h"
#include "eqat_internal.h"

// Scratch for W-hat: EQAT_NOALLOC_SCRATCH_BYTES (32 MiB) = 16 Mi bf16 weights or
// 8 Mi fp32 weights, e.g. one 4096 x 4096 bf16 projection.  In host code this
// name is only a stand-in for the device array; kernels get the device address
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fq_fwd_scratch[EQAT_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (the first call on a device does this set-up).
cudaError_t scratch_address(int dev, void **addr) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_fq_fwd_scratch);
        if (e != cudaSuccess) return e;
        if (!p) return cudaErrorInvalidSymbol;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return cudaSuccess;
}

eqat_status reject(eqat_status st, const char *msg) {
    eqat::set_error_detail(msg);
    return st;
}

bool misaligned(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

extern "C" eqat_status eqat_fq_linear_fwd_noalloc(const void *X, const void *W, int dt, const float *s,
                                                  const float *z, void *Y, int64_t M, int64_t N, int64_t K,
                                                  int bits, int group, eqat_stream_t stream) {
    if (dt != EQAT_F32 && dt != EQAT_BF16) return reject(EQAT_ERR_DTYPE, "dtype must be EQAT_F32 or EQAT_BF16");
    if (bits != 2 && bits != 3 && bits != 4) return reject(EQAT_ERR_UNSUPPORTED, "bits must be 2, 3 or 4");
    if (group != 32 && group != 64 && group != 128)
        return reject(EQAT_ERR_UNSUPPORTED, "group must be 32, 64 or 128");
    if (M < 0 || N < 0 || K < 0) return reject(EQAT_ERR_SHAPE, "negative size");
    if (K % group != 0) return reject(EQAT_ERR_SHAPE, "K must be a multiple of group");
    if (N % 8 != 0) return reject(EQAT_ERR_SHAPE, "N must be a multiple of 8");
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || N >= lim || K >= lim) return reject(EQAT_ERR_SHAPE, "a dimension is 2^31 or more");
    const uint64_t esize = dt == EQAT_F32 ? 4 : 2;
    const uint64_t need = static_cast<uint64_t>(N) * static_cast<uint64_t>(K) * esize;
    if (need > EQAT_NOALLOC_SCRATCH_BYTES)
        return reject(EQAT_ERR_WORKSPACE,
                      "N*K*sizeof(dtype) exceeds the 32 MiB static scratch of eqat_fq_linear_fwd_noalloc; "
                      "use eqat_fq_linear_fwd with a caller workspace");
    if ((M > 0 && K > 0 && !X) || (N > 0 && K > 0 && !W) || (N > 0 && K > 0 && (!s || !z)) ||
        (M > 0 && N > 0 && !Y))
        return reject(EQAT_ERR_NULL, "a required pointer is NULL");
    if (misaligned(X) || misaligned(W) || misaligned(s) || misaligned(z) || misaligned(Y))
        return reject(EQAT_ERR_ALIGN, "a pointer is not 16-byte aligned");
    if (M == 0 || N == 0) return EQAT_OK;

    eqat::DeviceInfo dev;
    cudaError_t e = eqat::current_device_info(dev);
    if (e != cudaSuccess) return reject(EQAT_ERR_CUDA, cudaGetErrorString(e));
    if (dev.major != 10) return reject(EQAT_ERR_UNSUPPORTED, "needs an sm_100 (B200) device");
    if (dev.device < 0 || dev.device >= kMaxDevices) return reject(EQAT_ERR_CUDA, "device ordinal out of range");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool f32 = dt == EQAT_F32;
    if (K == 0) {
        e = cudaMemsetAsync(Y, 0, static_cast<size_t>(M * N) * esize, st);
        return e == cudaSuccess ? EQAT_OK : reject(EQAT_ERR_CUDA, cudaGetErrorString(e));
    }
    void *scratch = nullptr;
    e = scratch_address(dev.device, &scratch);
    if (e != cudaSuccess) return reject(EQAT_ERR_CUDA, cudaGetErrorString(e));

    // Same two launches as eqat_fq_linear_fwd, with W-hat in the static scratch.
    // Nothing there has to start at zero: the prepass writes every element the
    // contraction reads.
    e = eqat::launch_fake_quant(W, f32, s, z, N, K, bits, group, scratch, f32, nullptr, nullptr, dev, st);
    if (e != cudaSuccess) return reject(EQAT_ERR_CUDA, cudaGetErrorString(e));
    eqat::EpiArgs epi;
    epi.kind = eqat::Epi::kStore;
    epi.out = Y;
    epi.ldo = N;
    epi.out_f32 = f32;
    const eqat::Operand A{X, K, false};
    const eqat::Operand B{scratch, K, false};
    e = f32 ? eqat::launch_gemm_f32(A, B, M, N, K, epi, nullptr, dev, st)
            : eqat::launch_gemm_tc(A, B, M, N, K, epi, dev, st);
    if (e != cudaSuccess) return reject(EQAT_ERR_CUDA, cudaGetErrorString(e));
    return EQAT_OK;
}
