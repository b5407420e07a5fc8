// Host-side declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace eqat {

struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int major = 0;
    int minor = 0;
};

// Cached attributes of the current device (thread-safe, one query per device).
cudaError_t current_device_info(DeviceInfo &info);

// ---------------------------------------------------------------- HBM kernels
// All element counts are validated by the caller; every launch goes on `st`.

// One weight matrix of a multi-layer init or pack: W [N, K]; init writes s_out,
// z_out; pack reads s, z and writes codes, zq.
struct QuantLayerArgs {
    const void *W;
    const float *s, *z;
    float *s_out, *z_out;
    uint8_t *codes, *zq;
    int64_t N, K;
};
// Every layer of one call in one launch (up to eight per launch); empty layers
// are skipped.
cudaError_t launch_minmax_init_multi(const QuantLayerArgs *layers, int n, bool w_f32, int bits, int group,
                                     const DeviceInfo &dev, cudaStream_t st);
cudaError_t launch_pack_multi(const QuantLayerArgs *layers, int n, bool w_f32, int bits, int group,
                              const DeviceInfo &dev, cudaStream_t st);
cudaError_t launch_minmax_init(const void *W, bool w_f32, int64_t N, int64_t K, int bits, int group,
                               float *s, float *z, const DeviceInfo &dev, cudaStream_t st);
cudaError_t launch_fake_quant(const void *W, bool w_f32, const float *s, const float *z, int64_t N,
                              int64_t K, int bits, int group, void *W_hat, bool out_f32,
                              uint8_t *code, uint8_t *mask, const DeviceInfo &dev,
                              cudaStream_t st);
cudaError_t launch_pack(const void *W, bool w_f32, const float *s, const float *z, int64_t N,
                        int64_t K, int bits, int group, uint8_t *codes, uint8_t *zq,
                        const DeviceInfo &dev, cudaStream_t st);
// s is fp32, or fp16 when s_f16 (widened exactly before use).
cudaError_t launch_dequant(const uint8_t *codes, const uint8_t *zq, const void *s, bool s_f16, int64_t N,
                           int64_t K, int bits, int group, void *W_hat, bool out_f32,
                           const DeviceInfo &dev, cudaStream_t st);

// ---------------------------------------------------------------- contractions
// D[GM, GN] = sum_k A(m, k) B(n, k).  An operand is "K-major" when its reduction
// index is contiguous in memory (stored as [rows][GK]) and "MN-major" when its
// row index is ([GK][rows]).  `ld` is the row stride of the stored matrix in
// elements.
struct Operand {
    const void *ptr;
    int64_t ld;
    bool mn_major;
};

enum class Epi : int {
    kStore = 0,   // D -> out (bf16 or fp32), row stride ldo
    kFqGrad = 1,  // Block-AP straight-through: dW = D*mask, ds, dz per group
    kE2eDs = 2,   // E2E-QP: ds = sum_group D * (W_q - zq), dz = -s sum_group D
    kMse = 3,     // reconstruction MSE: out = mse_scale (D - target) (bf16), *loss += sum (D - target)^2
};

struct EpiArgs {
    Epi kind = Epi::kStore;
    void *out = nullptr;
    int64_t ldo = 0;
    bool out_f32 = false;
    // kFqGrad: quantizer inputs of the rows of D (D is [N, K] = dW-hat)
    const void *W = nullptr;
    bool w_f32 = false;
    const float *s = nullptr;
    const float *z = nullptr;
    void *dW = nullptr;
    float *ds = nullptr;
    float *dz = nullptr;
    bool clamp_pass = false;  // kFqGrad: clamp straight-through as well
    // kE2eDs (ds and dz nullable; s_e2e is read only for dz)
    const uint8_t *codes = nullptr;
    const uint8_t *zq = nullptr;
    const void *s_e2e = nullptr;
    bool s_f16 = false;
    // kMse (out, ldo: dY)
    const void *target = nullptr;  // [GM, GN] bf16, row stride ldo
    double *loss = nullptr;
    float mse_scale = 0.0f;
    int bits = 2;
    int group = 64;
};

// B made on load from packed codes (E2E-QP, Eq. 2): W-hat[w_rows, w_cols] =
// (W_q - zq) s, converted in shared memory inside the pair GEMM instead of being
// written to HBM first.  B.mn_major says how W-hat enters the contraction (K-major for
// the forward, MN-major for the input gradient); B.ptr and B.ld are ignored.
struct CvtArgs {
    bool on = false;
    const uint8_t *codes = nullptr;  // [w_rows, code_row_bytes(w_cols, bits)]
    const uint8_t *zq = nullptr;     // [w_rows, w_cols / group]
    const void *s = nullptr;         // [w_rows, w_cols / group], fp32 or fp16 (s_f16)
    bool s_f16 = false;
    int bits = 2;
    int group = 64;
    int64_t w_rows = 0, w_cols = 0;
};

struct GemmProblem {
    Operand A;
    Operand B;
    int64_t GM, GN, GK;
    EpiArgs epi;
    CvtArgs cvt = {};
};

// Whether the pair GEMM can make this W-hat from its codes on load: the code rows must
// be a whole number of 16-byte units for the tensor map (2-bit: w_cols % 64 == 0).
bool cvt_supported(int64_t w_rows, int64_t w_cols, int bits, int group);

// bf16 operands on tcgen05 tensor cores, fp32 accumulation in tensor memory.
// A grouped launch runs the tiles of up to two contractions in one persistent
// kernel (problem 0 first); problem 1, if present, must use the kStore epilogue.
cudaError_t launch_gemm_tc_group(const GemmProblem *probs, int nprob, const DeviceInfo &dev,
                                 cudaStream_t st);
cudaError_t launch_gemm_tc(const Operand &A, const Operand &B, int64_t GM, int64_t GN, int64_t GK,
                           const EpiArgs &epi, const DeviceInfo &dev, cudaStream_t st);

// fp32 operands on the CUDA cores; epilogues run as a separate pass over an
// fp32 D held in `d_scratch` (GM x GN floats) when epi.kind != kStore.
cudaError_t launch_gemm_f32(const Operand &A, const Operand &B, int64_t GM, int64_t GN, int64_t GK,
                            const EpiArgs &epi, float *d_scratch, const DeviceInfo &dev,
                            cudaStream_t st);

// Batch-1..8 inference: Y[M, N] = X[M, K] ((W_q - zq) s)^T straight from packed
// codes, bf16 X and Y, M in 1..8, group 64 or 128.  `ws` holds at least
// gemv_workspace_bytes(...) bytes (256-byte aligned): X's fragments, the group
// sums of X and the per-row-tile partials.
size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int group, int sm_count);
size_t gemv_workspace_bound(int64_t M, int64_t N, int64_t K, int bits, int group);  // any SM count
cudaError_t launch_dq_gemv(const void *X, const uint8_t *codes, const uint8_t *zq, const void *s, bool s_f16,
                           void *Y, int64_t M, int64_t N, int64_t K, int bits, int group, void *ws,
                           const DeviceInfo &dev, cudaStream_t st);

// Shared by the kernels that use TMA and bounded waits.
int *device_error_word();
cudaError_t encode_map_2d(CUtensorMap &map, CUtensorMapDataType type, const void *base, uint64_t inner,
                          uint64_t outer, uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swizzle);

// Multi-tensor AdamW (decoupled weight decay), fp32 math on fp32 state.
struct AdamwSeg {
    float *p;
    const void *g;
    float *m;
    float *v;
    void *copy;      // nullable: updated parameter in bf16 (copy_bf16) or fp32
    int64_t n;
    int g_bf16;
    int copy_bf16;
    float decay;     // 1 - lr wd
    float b1, b2;
    float omb1, omb2;  // 1 - b1, 1 - b2 (formed in double)
    float step_size; // lr / (1 - b1^t)
    float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
    float eps;
};
constexpr int kAdamwMaxSegs = 32;
cudaError_t launch_adamw(const AdamwSeg *segs, int nseg, const DeviceInfo &dev, cudaStream_t st);

// fp32 reconstruction MSE in place: dY = scale (dY - target), *loss += sum (dY - target)^2.
cudaError_t launch_mse_f32(float *dY, const float *target, int64_t n, float scale, double *loss,
                           const DeviceInfo &dev, cudaStream_t st);
// Y = 0 (K == 0), bf16: dY = scale (0 - T), *loss += sum T^2 scale / 2.
cudaError_t launch_mse_zero_bf16(void *dY, const void *target, int64_t n, float scale, double *loss,
                                 const DeviceInfo &dev, cudaStream_t st);

// Records the message that eqat_last_error_detail() returns on this thread.
void set_error_detail(const char *msg);

// Device error word (bounded waits): read-and-clear on the current device.
cudaError_t read_and_clear_device_error(int &value);
cudaError_t launch_selftest_bounded_wait(uint64_t timeout_ns, cudaStream_t st);

}  // namespace eqat
