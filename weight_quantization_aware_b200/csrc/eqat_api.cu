// extern "C" entry points of libeqat: argument validation on the host, then
// kernel launches on the caller's stream.  No entry point allocates memory,
// synchronises (except eqat_device_error) or falls back to another device.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/eqat.h"
#include "eqat_internal.h"

namespace eqat {

cudaError_t current_device_info(DeviceInfo &info) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev].device != dev) {
        DeviceInfo d;
        d.device = dev;
        if ((e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
        cache[dev] = d;
    }
    info = cache[dev];
    return cudaSuccess;
}

}  // namespace eqat

namespace {
thread_local char g_detail[256] = "";
}  // namespace

namespace eqat {
void set_error_detail(const char *msg) { std::snprintf(g_detail, sizeof(g_detail), "%s", msg); }
}  // namespace eqat

namespace {

using eqat::DeviceInfo;
using eqat::Epi;
using eqat::EpiArgs;
using eqat::Operand;

void set_detail(const char *msg) {
    std::snprintf(g_detail, sizeof(g_detail), "%s", msg);
}

eqat_status fail(eqat_status st, const char *msg) {
    set_detail(msg);
    return st;
}

eqat_status cuda_fail(cudaError_t e, const char *where) {
    std::snprintf(g_detail, sizeof(g_detail), "%s: %s", where, cudaGetErrorString(e));
    return EQAT_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Validates bits, group and sizes (no CUDA call).
eqat_status check_common(int64_t M, int64_t N, int64_t K, int bits, int group) {
    if (bits != 2 && bits != 3 && bits != 4) return fail(EQAT_ERR_UNSUPPORTED, "bits must be 2, 3 or 4");
    if (group != 32 && group != 64 && group != 128)
        return fail(EQAT_ERR_UNSUPPORTED, "group must be 32, 64 or 128");
    if (M < 0 || N < 0 || K < 0) return fail(EQAT_ERR_SHAPE, "negative size");
    if (K % group != 0) return fail(EQAT_ERR_SHAPE, "K must be a multiple of group");
    if (N % 8 != 0) return fail(EQAT_ERR_SHAPE, "N must be a multiple of 8");
    const int64_t lim = int64_t(1) << 31;
    if (M >= lim || N >= lim || K >= lim) return fail(EQAT_ERR_SHAPE, "a dimension is 2^31 or more");
    if ((N > 0 && K > (int64_t(1) << 60) / N) || (M > 0 && K > (int64_t(1) << 60) / M) ||
        (M > 0 && N > (int64_t(1) << 60) / M))
        return fail(EQAT_ERR_SHAPE, "size product overflows");
    return EQAT_OK;
}

// The current device must be an sm_100 part; fills dev.  Called after every
// argument check, right before the first launch.
eqat_status get_device(DeviceInfo &dev) {
    cudaError_t e = eqat::current_device_info(dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    if (dev.major != 10) return fail(EQAT_ERR_UNSUPPORTED, "needs an sm_100 (B200) device");
    return EQAT_OK;
}

// A pointer must be non-NULL when its buffer has elements, and 16-byte aligned.
eqat_status check_ptr(const void *p, int64_t elems, const char *name) {
    static thread_local char msg[128];
    if (elems > 0 && p == nullptr) {
        std::snprintf(msg, sizeof(msg), "%s is NULL", name);
        return fail(EQAT_ERR_NULL, msg);
    }
    if (p && !aligned(p, 16)) {
        std::snprintf(msg, sizeof(msg), "%s is not 16-byte aligned", name);
        return fail(EQAT_ERR_ALIGN, msg);
    }
    return EQAT_OK;
}

eqat_status check_dtype(int dt) {
    if (dt != EQAT_F32 && dt != EQAT_BF16) return fail(EQAT_ERR_DTYPE, "dtype must be EQAT_F32 or EQAT_BF16");
    return EQAT_OK;
}

// Step-size dtype of the E2E-QP entry points: fp32, or fp16 storage.
eqat_status check_sdtype(int sdt) {
    if (sdt != EQAT_F32 && sdt != EQAT_F16) return fail(EQAT_ERR_DTYPE, "sdt must be EQAT_F32 or EQAT_F16");
    return EQAT_OK;
}

size_t esize(int dt) { return dt == EQAT_F32 ? 4 : 2; }

// The decode-size path of eqat_dq_linear_fwd; EQAT_DQ_GEMV=0 turns it off
// (measurement aid: the dequant + GEMM path at the same sizes).
bool gemv_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("EQAT_DQ_GEMV");
        return !(v && v[0] == '0');
    }();
    return on;
}

// Dequantize on load in the E2E-QP contractions (bf16): the pair GEMM makes W-hat
// from the codes in shared memory instead of reading a W-hat that the dequantize
// kernel wrote to the workspace.  Each B tile is converted once per 256-row M tile,
// so the conversion work is M / 256 times the dequantize kernel's, while the HBM it
// saves (a 2-byte W-hat written and read back, 0.25-1 byte codes read instead) does
// not grow with M.  Measured on B200, forward alone: at M <= 256 it is 0.89-0.98x the
// time of dequantize + GEMM on 2-bit layers of 2^25 weights or more (13824 x 5120,
// 28672 x 8192), 1.03-1.26x on 3- and 4-bit layers and 1.3x on 4096 x 4096; at
// M >= 512 1.2-2.3x.  In the backward (dX = dY W-hat with W-hat made on load, an
// MN-major B) it is far slower: a forward + backward pair on the 70B gate at M = 64
// takes 777 us against 499 us when the forward dequantizes into the workspace and
// the backward reuses that W-hat.
// So: the forward makes W-hat on load only when the caller passes no workspace (a
// forward without one keeps nothing for a backward, and the dequantize path needs
// one); with a workspace it dequantizes into it.  The backward never makes W-hat on
// load.  EQAT_DQ_ONLOAD=1 uses it in both wherever the code layout allows,
// EQAT_DQ_ONLOAD=0 never (measurement aids and the tests' way to compare the paths).
int onload_mode() {
    static const int mode = [] {
        const char *v = std::getenv("EQAT_DQ_ONLOAD");
        if (v && v[0] == '0') return 0;
        if (v && v[0] == '1') return 1;
        return -1;  // by the rule above
    }();
    return mode;
}

bool fwd_onload(int64_t N, int64_t K, int bits, int group, bool have_ws) {
    if (!eqat::cvt_supported(N, K, bits, group)) return false;
    const int mode = onload_mode();
    if (mode >= 0) return mode == 1;
    return !have_ws;
}

bool bwd_onload(int64_t N, int64_t K, int bits, int group) {
    return eqat::cvt_supported(N, K, bits, group) && onload_mode() == 1;
}

eqat::CvtArgs cvt_args(const uint8_t *codes, const uint8_t *zq, const void *s, int sdt, int64_t N, int64_t K,
                       int bits, int group) {
    eqat::CvtArgs c;
    c.on = true;
    c.codes = codes;
    c.zq = zq;
    c.s = s;
    c.s_f16 = sdt == EQAT_F16;
    c.bits = bits;
    c.group = group;
    c.w_rows = N;
    c.w_cols = K;
    return c;
}

int64_t code_bytes(int64_t N, int64_t K, int bits) {
    return bits == 2 ? N * (K / 4) : bits == 4 ? N * (K / 2) : N * K;
}

size_t ws_need(int64_t N, int64_t K, int dt) {
    const size_t per = dt == EQAT_F32 ? 8 : 2;  // W-hat (+ fp32 dW-hat in fp32 mode)
    const size_t b = static_cast<size_t>(N) * static_cast<size_t>(K) * per;
    return (b + 255) & ~static_cast<size_t>(255);
}

eqat_status check_ws(const void *ws, size_t ws_bytes, int64_t N, int64_t K, int dt) {
    const size_t need = ws_need(N, K, dt);
    if (need == 0) return EQAT_OK;
    if (!ws || ws_bytes < need) return fail(EQAT_ERR_WORKSPACE, "workspace missing or smaller than eqat_workspace_bytes()");
    if (!aligned(ws, 256)) return fail(EQAT_ERR_ALIGN, "workspace is not 256-byte aligned");
    return EQAT_OK;
}

#define EQAT_TRY(expr)                       \
    do {                                     \
        eqat_status _s = (expr);             \
        if (_s != EQAT_OK) return _s;        \
    } while (0)

#define EQAT_CUDA(expr, where)                 \
    do {                                       \
        cudaError_t _e = (expr);               \
        if (_e != cudaSuccess) return cuda_fail(_e, where); \
    } while (0)

cudaError_t zero(void *p, size_t bytes, cudaStream_t st) {
    if (!p || bytes == 0) return cudaSuccess;
    return cudaMemsetAsync(p, 0, bytes, st);
}

// Y[GM, GN] = A . B^T with the dtype's engine.
cudaError_t contract(int dt, const Operand &A, const Operand &B, int64_t GM, int64_t GN, int64_t GK,
                     const EpiArgs &epi, float *f32_scratch, const DeviceInfo &dev, cudaStream_t st) {
    if (dt == EQAT_BF16) return eqat::launch_gemm_tc(A, B, GM, GN, GK, epi, dev, st);
    return eqat::launch_gemm_f32(A, B, GM, GN, GK, epi, f32_scratch, dev, st);
}

}  // namespace

extern "C" {

const char *eqat_status_string(int status) {
    switch (status) {
        case EQAT_OK: return "EQAT_OK";
        case EQAT_ERR_NULL: return "EQAT_ERR_NULL";
        case EQAT_ERR_SHAPE: return "EQAT_ERR_SHAPE";
        case EQAT_ERR_ALIGN: return "EQAT_ERR_ALIGN";
        case EQAT_ERR_DTYPE: return "EQAT_ERR_DTYPE";
        case EQAT_ERR_UNSUPPORTED: return "EQAT_ERR_UNSUPPORTED";
        case EQAT_ERR_WORKSPACE: return "EQAT_ERR_WORKSPACE";
        case EQAT_ERR_CUDA: return "EQAT_ERR_CUDA";
        case EQAT_ERR_TIMEOUT: return "EQAT_ERR_TIMEOUT";
        default: return "EQAT_ERR_UNKNOWN";
    }
}

const char *eqat_last_error_detail(void) { return g_detail; }

int eqat_version(void) { return EQAT_VERSION; }

size_t eqat_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int group, int dt) {
    if (N <= 0 || K <= 0 || (dt != EQAT_F32 && dt != EQAT_BF16)) return 0;
    size_t need = ws_need(N, K, dt);
    // the decode path (bf16, M <= 8) keeps its per-row-tile partial sums here
    if (dt == EQAT_BF16 && M >= 1 && M <= 8 && (group == 64 || group == 128) && bits >= 2 && bits <= 4)
        need = std::max(need, (eqat::gemv_workspace_bound(M, N, K, bits, group) + 255) & ~static_cast<size_t>(255));
    return need;
}

eqat_status eqat_minmax_init(const void *W, int wdt, int64_t N, int64_t K, int bits, int group, float *s,
                             float *z, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(wdt));
    EQAT_TRY(check_common(0, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(W, N * K, "W"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(z, ng, "z"));
    if (ng == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_minmax_init(W, wdt == EQAT_F32, N, K, bits, group, s, z, dev,
                                       reinterpret_cast<cudaStream_t>(stream)),
              "minmax_init");
    return EQAT_OK;
}

eqat_status eqat_fake_quant(const void *W, int wdt, const float *s, const float *z, int64_t N, int64_t K,
                            int bits, int group, void *W_hat, uint8_t *code, uint8_t *mask,
                            eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(wdt));
    EQAT_TRY(check_common(0, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(W, N * K, "W"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(z, ng, "z"));
    EQAT_TRY(check_ptr(W_hat, 0, "W_hat"));
    EQAT_TRY(check_ptr(code, 0, "code"));
    EQAT_TRY(check_ptr(mask, 0, "mask"));
    if (!W_hat && !code && !mask) return EQAT_OK;
    if (N * K == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_fake_quant(W, wdt == EQAT_F32, s, z, N, K, bits, group, W_hat, wdt == EQAT_F32,
                                      code, mask, dev, reinterpret_cast<cudaStream_t>(stream)),
              "fake_quant");
    return EQAT_OK;
}

eqat_status eqat_pack_codes(const void *W, int wdt, const float *s, const float *z, int64_t N, int64_t K,
                            int bits, int group, uint8_t *codes, uint8_t *zq, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(wdt));
    EQAT_TRY(check_common(0, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(W, N * K, "W"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(z, ng, "z"));
    EQAT_TRY(check_ptr(codes, code_bytes(N, K, bits), "codes"));
    EQAT_TRY(check_ptr(zq, ng, "zq"));
    if (N * K == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_pack(W, wdt == EQAT_F32, s, z, N, K, bits, group, codes, zq, dev,
                                reinterpret_cast<cudaStream_t>(stream)),
              "pack_codes");
    return EQAT_OK;
}

// n layers of one multi-layer call: at most EQAT_MAX_MULTI, host arrays present.
eqat_status check_multi(int n, const void *a, const void *b, const void *c) {
    if (n < 0 || n > EQAT_MAX_MULTI) return fail(EQAT_ERR_SHAPE, "layer count must be 0..EQAT_MAX_MULTI");
    if (n > 0 && (!a || !b || !c)) return fail(EQAT_ERR_NULL, "a layer array is NULL");
    return EQAT_OK;
}

eqat_status eqat_minmax_init_multi(int n, const void *const *W, int wdt, const int64_t *N, const int64_t *K,
                                   int bits, int group, float *const *s, float *const *z,
                                   eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(wdt));
    EQAT_TRY(check_multi(n, W, N, K));
    EQAT_TRY(check_multi(n, s, z, W));
    std::vector<eqat::QuantLayerArgs> layers(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) {
        EQAT_TRY(check_common(0, N[i], K[i], bits, group));
        const int64_t ng = N[i] * (K[i] / group);
        EQAT_TRY(check_ptr(W[i], N[i] * K[i], "W[i]"));
        EQAT_TRY(check_ptr(s[i], ng, "s[i]"));
        EQAT_TRY(check_ptr(z[i], ng, "z[i]"));
        eqat::QuantLayerArgs &a = layers[static_cast<size_t>(i)];
        a = eqat::QuantLayerArgs{};
        a.W = W[i];
        a.s_out = s[i];
        a.z_out = z[i];
        a.N = N[i];
        a.K = K[i];
    }
    int64_t total = 0;
    for (const auto &a : layers) total += a.N * a.K;
    if (total == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_minmax_init_multi(layers.data(), n, wdt == EQAT_F32, bits, group, dev,
                                             reinterpret_cast<cudaStream_t>(stream)),
              "minmax_init_multi");
    return EQAT_OK;
}

eqat_status eqat_pack_codes_multi(int n, const void *const *W, int wdt, const float *const *s,
                                  const float *const *z, const int64_t *N, const int64_t *K, int bits, int group,
                                  uint8_t *const *codes, uint8_t *const *zq, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(wdt));
    EQAT_TRY(check_multi(n, W, N, K));
    EQAT_TRY(check_multi(n, s, z, W));
    EQAT_TRY(check_multi(n, codes, zq, W));
    std::vector<eqat::QuantLayerArgs> layers(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) {
        EQAT_TRY(check_common(0, N[i], K[i], bits, group));
        const int64_t ng = N[i] * (K[i] / group);
        EQAT_TRY(check_ptr(W[i], N[i] * K[i], "W[i]"));
        EQAT_TRY(check_ptr(s[i], ng, "s[i]"));
        EQAT_TRY(check_ptr(z[i], ng, "z[i]"));
        EQAT_TRY(check_ptr(codes[i], code_bytes(N[i], K[i], bits), "codes[i]"));
        EQAT_TRY(check_ptr(zq[i], ng, "zq[i]"));
        eqat::QuantLayerArgs &a = layers[static_cast<size_t>(i)];
        a = eqat::QuantLayerArgs{};
        a.W = W[i];
        a.s = s[i];
        a.z = z[i];
        a.codes = codes[i];
        a.zq = zq[i];
        a.N = N[i];
        a.K = K[i];
    }
    int64_t total = 0;
    for (const auto &a : layers) total += a.N * a.K;
    if (total == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_pack_multi(layers.data(), n, wdt == EQAT_F32, bits, group, dev,
                                      reinterpret_cast<cudaStream_t>(stream)),
              "pack_codes_multi");
    return EQAT_OK;
}

eqat_status eqat_dequant_codes(const uint8_t *codes, const uint8_t *zq, const float *s, int64_t N, int64_t K,
                               int bits, int group, void *W_hat, int dt, eqat_stream_t stream) {
    return eqat_dequant_codes_ex(codes, zq, s, EQAT_F32, N, K, bits, group, W_hat, dt, stream);
}

eqat_status eqat_dequant_codes_ex(const uint8_t *codes, const uint8_t *zq, const void *s, int sdt, int64_t N,
                                  int64_t K, int bits, int group, void *W_hat, int dt, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(dt));
    EQAT_TRY(check_sdtype(sdt));
    EQAT_TRY(check_common(0, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(codes, code_bytes(N, K, bits), "codes"));
    EQAT_TRY(check_ptr(zq, ng, "zq"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(W_hat, N * K, "W_hat"));
    if (N * K == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_dequant(codes, zq, s, sdt == EQAT_F16, N, K, bits, group, W_hat, dt == EQAT_F32, dev,
                                   reinterpret_cast<cudaStream_t>(stream)),
              "dequant_codes");
    return EQAT_OK;
}

eqat_status eqat_fq_linear_fwd(const void *X, const void *W, int dt, const float *s, const float *z, void *Y,
                               int64_t M, int64_t N, int64_t K, int bits, int group, void *ws, size_t ws_bytes,
                               eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(dt));
    EQAT_TRY(check_common(M, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(X, M * K, "X"));
    EQAT_TRY(check_ptr(W, N * K, "W"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(z, ng, "z"));
    EQAT_TRY(check_ptr(Y, M * N, "Y"));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (M * N == 0) return EQAT_OK;
    if (K > 0) EQAT_TRY(check_ws(ws, ws_bytes, N, K, dt));
    EQAT_TRY(get_device(dev));
    if (K == 0) {
        EQAT_CUDA(zero(Y, static_cast<size_t>(M * N) * esize(dt), st), "memset Y");
        return EQAT_OK;
    }
    const bool f32 = dt == EQAT_F32;
    EQAT_CUDA(eqat::launch_fake_quant(W, f32, s, z, N, K, bits, group, ws, f32, nullptr, nullptr, dev, st),
              "fq prepass");
    EpiArgs epi;
    epi.kind = Epi::kStore;
    epi.out = Y;
    epi.ldo = N;
    epi.out_f32 = f32;
    EQAT_CUDA(contract(dt, Operand{X, K, false}, Operand{ws, K, false}, M, N, K, epi, nullptr, dev, st),
              "fq forward contraction");
    return EQAT_OK;
}

eqat_status eqat_fq_linear_bwd(const void *X, const void *W, int dt, const float *s, const float *z,
                               const void *dY, void *dX, void *dW, float *ds, float *dz, int64_t M, int64_t N,
                               int64_t K, int bits, int group, void *ws, size_t ws_bytes, int w_hat_in_ws,
                               eqat_stream_t stream) {
    return eqat_fq_linear_bwd_ex(X, W, dt, s, z, dY, dX, dW, ds, dz, M, N, K, bits, group, 0u, ws, ws_bytes,
                                 w_hat_in_ws, stream);
}

eqat_status eqat_fq_linear_bwd_ex(const void *X, const void *W, int dt, const float *s, const float *z,
                                  const void *dY, void *dX, void *dW, float *ds, float *dz, int64_t M, int64_t N,
                                  int64_t K, int bits, int group, uint32_t flags, void *ws, size_t ws_bytes,
                                  int w_hat_in_ws, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(dt));
    if (flags & ~EQAT_GRAD_CLAMP_PASS) return fail(EQAT_ERR_UNSUPPORTED, "unknown flag bits");
    EQAT_TRY(check_common(M, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(X, M * K, "X"));
    EQAT_TRY(check_ptr(W, N * K, "W"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(z, ng, "z"));
    EQAT_TRY(check_ptr(dY, M * N, "dY"));
    EQAT_TRY(check_ptr(dX, 0, "dX"));
    EQAT_TRY(check_ptr(dW, 0, "dW"));
    EQAT_TRY(check_ptr(ds, 0, "ds"));
    EQAT_TRY(check_ptr(dz, 0, "dz"));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool f32 = dt == EQAT_F32;
    const size_t es = esize(dt);
    const bool want_w = dW || ds || dz;
    if (!dX && !want_w) return EQAT_OK;
    if (N * K > 0) EQAT_TRY(check_ws(ws, ws_bytes, N, K, dt));
    EQAT_TRY(get_device(dev));

    // Contractions to run: the weight side dY^T X (fused straight-through
    // epilogue) and the input side dY W-hat.  On the tensor cores both run in one
    // grouped persistent launch.
    eqat::GemmProblem probs[2];
    int np = 0;
    if (want_w && N * K > 0) {
        if (M == 0) {
            EQAT_CUDA(zero(dW, static_cast<size_t>(N * K) * es, st), "memset dW");
            EQAT_CUDA(zero(ds, static_cast<size_t>(ng) * 4, st), "memset ds");
            EQAT_CUDA(zero(dz, static_cast<size_t>(ng) * 4, st), "memset dz");
        } else {
            EpiArgs epi;
            epi.kind = Epi::kFqGrad;
            epi.W = W;
            epi.w_f32 = f32;
            epi.s = s;
            epi.z = z;
            epi.dW = dW;
            epi.ds = ds;
            epi.dz = dz;
            epi.clamp_pass = (flags & EQAT_GRAD_CLAMP_PASS) != 0;
            epi.bits = bits;
            epi.group = group;
            probs[np++] = eqat::GemmProblem{Operand{dY, N, true}, Operand{X, K, true}, N, K, M, epi};
        }
    }
    if (dX && M * K > 0) {
        if (N == 0) {
            EQAT_CUDA(zero(dX, static_cast<size_t>(M * K) * es, st), "memset dX");
        } else {
            if (!w_hat_in_ws)
                EQAT_CUDA(eqat::launch_fake_quant(W, f32, s, z, N, K, bits, group, ws, f32, nullptr, nullptr, dev, st),
                          "fq prepass");
            EpiArgs epi;
            epi.kind = Epi::kStore;
            epi.out = dX;
            epi.ldo = K;
            epi.out_f32 = f32;
            probs[np++] = eqat::GemmProblem{Operand{dY, N, false}, Operand{ws, K, true}, M, K, N, epi};
        }
    }
    if (np == 0) return EQAT_OK;
    if (!f32) {
        EQAT_CUDA(eqat::launch_gemm_tc_group(probs, np, dev, st), "backward contractions");
    } else {
        float *scratch = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + static_cast<size_t>(N * K) * 4);
        for (int i = 0; i < np; ++i)
            EQAT_CUDA(eqat::launch_gemm_f32(probs[i].A, probs[i].B, probs[i].GM, probs[i].GN, probs[i].GK,
                                            probs[i].epi, scratch, dev, st),
                      "backward contraction (fp32)");
    }
    return EQAT_OK;
}

eqat_status eqat_dq_linear_fwd(const void *X, int dt, const uint8_t *codes, const uint8_t *zq, const float *s,
                               void *Y, int64_t M, int64_t N, int64_t K, int bits, int group, void *ws,
                               size_t ws_bytes, eqat_stream_t stream) {
    return eqat_dq_linear_fwd_ex(X, dt, codes, zq, s, EQAT_F32, Y, M, N, K, bits, group, ws, ws_bytes, stream);
}

eqat_status eqat_dq_linear_fwd_ex(const void *X, int dt, const uint8_t *codes, const uint8_t *zq, const void *s,
                                  int sdt, void *Y, int64_t M, int64_t N, int64_t K, int bits, int group, void *ws,
                                  size_t ws_bytes, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(dt));
    EQAT_TRY(check_sdtype(sdt));
    EQAT_TRY(check_common(M, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(X, M * K, "X"));
    EQAT_TRY(check_ptr(codes, code_bytes(N, K, bits), "codes"));
    EQAT_TRY(check_ptr(zq, ng, "zq"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(Y, M * N, "Y"));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (M * N == 0) return EQAT_OK;
    const bool f32 = dt == EQAT_F32;
    // no workspace: W-hat made on load (bf16, a code layout the converter takes)
    const bool onload = K > 0 && !f32 && fwd_onload(N, K, bits, group, ws != nullptr);
    if (K > 0 && !(onload && ws == nullptr)) EQAT_TRY(check_ws(ws, ws_bytes, N, K, dt));
    EQAT_TRY(get_device(dev));
    if (K == 0) {
        EQAT_CUDA(zero(Y, static_cast<size_t>(M * N) * esize(dt), st), "memset Y");
        return EQAT_OK;
    }
    if (ws && !f32 && M <= 8 && (group == 64 || group == 128) && gemv_enabled() &&
        eqat::gemv_workspace_bytes(M, N, K, bits, group, dev.sm_count) <= ws_bytes) {
        // decode sizes: stream the codes once, no W-hat in memory (the partials
        // take at most M N K / 128 bytes, inside any workspace check_ws accepts)
        EQAT_CUDA(eqat::launch_dq_gemv(X, codes, zq, s, sdt == EQAT_F16, Y, M, N, K, bits, group, ws, dev, st),
                  "dq GEMV");
        return EQAT_OK;
    }
    EpiArgs epi;
    epi.kind = Epi::kStore;
    epi.out = Y;
    epi.ldo = N;
    epi.out_f32 = f32;
    if (onload) {
        // W-hat made from the codes inside the contraction, never written to HBM
        eqat::GemmProblem g{Operand{X, K, false}, Operand{nullptr, K, false}, M, N, K, epi};
        g.cvt = cvt_args(codes, zq, s, sdt, N, K, bits, group);
        EQAT_CUDA(eqat::launch_gemm_tc_group(&g, 1, dev, st), "dq forward contraction (dequantize on load)");
        return EQAT_OK;
    }
    EQAT_CUDA(eqat::launch_dequant(codes, zq, s, sdt == EQAT_F16, N, K, bits, group, ws, f32, dev, st),
              "dequant prepass");
    EQAT_CUDA(contract(dt, Operand{X, K, false}, Operand{ws, K, false}, M, N, K, epi, nullptr, dev, st),
              "dq forward contraction");
    return EQAT_OK;
}

eqat_status eqat_dq_linear_bwd_s(const void *X, int dt, const uint8_t *codes, const uint8_t *zq, const float *s,
                                 const void *dY, void *dX, float *ds, int64_t M, int64_t N, int64_t K, int bits,
                                 int group, void *ws, size_t ws_bytes, int w_hat_in_ws, eqat_stream_t stream) {
    return eqat_dq_linear_bwd(X, dt, codes, zq, s, EQAT_F32, dY, dX, ds, nullptr, M, N, K, bits, group, ws,
                              ws_bytes, w_hat_in_ws, stream);
}

eqat_status eqat_dq_linear_bwd(const void *X, int dt, const uint8_t *codes, const uint8_t *zq, const void *s,
                               int sdt, const void *dY, void *dX, float *ds, float *dz, int64_t M, int64_t N,
                               int64_t K, int bits, int group, void *ws, size_t ws_bytes, int w_hat_in_ws,
                               eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(dt));
    EQAT_TRY(check_sdtype(sdt));
    EQAT_TRY(check_common(M, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(X, M * K, "X"));
    EQAT_TRY(check_ptr(codes, code_bytes(N, K, bits), "codes"));
    EQAT_TRY(check_ptr(zq, ng, "zq"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(dY, M * N, "dY"));
    EQAT_TRY(check_ptr(dX, 0, "dX"));
    EQAT_TRY(check_ptr(ds, 0, "ds"));
    EQAT_TRY(check_ptr(dz, 0, "dz"));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool f32 = dt == EQAT_F32;
    if (!dX && !ds && !dz) return EQAT_OK;
    if (N * K > 0) EQAT_TRY(check_ws(ws, ws_bytes, N, K, dt));
    EQAT_TRY(get_device(dev));

    eqat::GemmProblem probs[2];
    int np = 0;
    if ((ds || dz) && ng > 0) {
        if (M == 0) {
            EQAT_CUDA(zero(ds, static_cast<size_t>(ng) * 4, st), "memset ds");
            EQAT_CUDA(zero(dz, static_cast<size_t>(ng) * 4, st), "memset dz");
        } else {
            EpiArgs epi;
            epi.kind = Epi::kE2eDs;
            epi.codes = codes;
            epi.zq = zq;
            epi.ds = ds;
            epi.dz = dz;
            epi.s_e2e = s;
            epi.s_f16 = sdt == EQAT_F16;
            epi.bits = bits;
            epi.group = group;
            probs[np++] = eqat::GemmProblem{Operand{dY, N, true}, Operand{X, K, true}, N, K, M, epi};
        }
    }
    if (dX && M * K > 0) {
        if (N == 0) {
            EQAT_CUDA(zero(dX, static_cast<size_t>(M * K) * esize(dt), st), "memset dX");
        } else {
            const bool onload = !f32 && bwd_onload(N, K, bits, group);
            if (!w_hat_in_ws && !onload)
                EQAT_CUDA(eqat::launch_dequant(codes, zq, s, sdt == EQAT_F16, N, K, bits, group, ws, f32, dev, st),
                          "dequant prepass");
            EpiArgs epi;
            epi.kind = Epi::kStore;
            epi.out = dX;
            epi.ldo = K;
            epi.out_f32 = f32;
            probs[np] = eqat::GemmProblem{Operand{dY, N, false}, Operand{ws, K, true}, M, K, N, epi};
            // dX = dY W-hat with W-hat made from the codes on load (MN-major B)
            if (onload) probs[np].cvt = cvt_args(codes, zq, s, sdt, N, K, bits, group);
            ++np;
        }
    }
    if (np == 0) return EQAT_OK;
    if (!f32) {
        EQAT_CUDA(eqat::launch_gemm_tc_group(probs, np, dev, st), "E2E backward contractions");
    } else {
        float *scratch = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + static_cast<size_t>(N * K) * 4);
        for (int i = 0; i < np; ++i)
            EQAT_CUDA(eqat::launch_gemm_f32(probs[i].A, probs[i].B, probs[i].GM, probs[i].GN, probs[i].GK,
                                            probs[i].epi, scratch, dev, st),
                      "E2E backward contraction (fp32)");
    }
    return EQAT_OK;
}

eqat_status eqat_fq_linear_fwd_mse(const void *X, const void *W, int dt, const float *s, const float *z,
                                   const void *T, void *dY, double *loss, int64_t M, int64_t N, int64_t K,
                                   int bits, int group, void *ws, size_t ws_bytes, eqat_stream_t stream) {
    DeviceInfo dev;
    EQAT_TRY(check_dtype(dt));
    EQAT_TRY(check_common(M, N, K, bits, group));
    const int64_t ng = N * (K / group);
    EQAT_TRY(check_ptr(X, M * K, "X"));
    EQAT_TRY(check_ptr(W, N * K, "W"));
    EQAT_TRY(check_ptr(s, ng, "s"));
    EQAT_TRY(check_ptr(z, ng, "z"));
    EQAT_TRY(check_ptr(T, M * N, "T"));
    EQAT_TRY(check_ptr(dY, M * N, "dY"));
    if (!loss) return fail(EQAT_ERR_NULL, "loss is NULL");
    if (!aligned(loss, 8)) return fail(EQAT_ERR_ALIGN, "loss is not 8-byte aligned");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (M * N > 0 && K > 0) EQAT_TRY(check_ws(ws, ws_bytes, N, K, dt));
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(zero(loss, sizeof(double), st), "memset loss");
    if (M * N == 0) return EQAT_OK;
    const bool f32 = dt == EQAT_F32;
    const float scale = static_cast<float>(2.0 / (static_cast<double>(M) * static_cast<double>(N)));
    if (K == 0) {  // Y = 0
        if (f32) {
            EQAT_CUDA(zero(dY, static_cast<size_t>(M * N) * esize(dt), st), "memset dY");
            EQAT_CUDA(eqat::launch_mse_f32(static_cast<float *>(dY), static_cast<const float *>(T), M * N, scale, loss,
                                           dev, st),
                      "mse (fp32)");
            return EQAT_OK;
        }
        EQAT_CUDA(eqat::launch_mse_zero_bf16(dY, T, M * N, scale, loss, dev, st), "mse (K == 0)");
        return EQAT_OK;
    }
    EQAT_CUDA(eqat::launch_fake_quant(W, f32, s, z, N, K, bits, group, ws, f32, nullptr, nullptr, dev, st),
              "fq prepass");
    EpiArgs epi;
    if (f32) {
        epi.kind = Epi::kStore;
        epi.out = dY;
        epi.ldo = N;
        epi.out_f32 = true;
        EQAT_CUDA(contract(dt, Operand{X, K, false}, Operand{ws, K, false}, M, N, K, epi, nullptr, dev, st),
                  "fq forward contraction");
        EQAT_CUDA(eqat::launch_mse_f32(static_cast<float *>(dY), static_cast<const float *>(T), M * N, scale, loss,
                                       dev, st),
                  "mse (fp32)");
        return EQAT_OK;
    }
    epi.kind = Epi::kMse;
    epi.out = dY;
    epi.ldo = N;
    epi.target = T;
    epi.loss = loss;
    epi.mse_scale = scale;
    EQAT_CUDA(eqat::launch_gemm_tc(Operand{X, K, false}, Operand{ws, K, false}, M, N, K, epi, dev, st),
              "fq forward contraction with the MSE epilogue");
    return EQAT_OK;
}

eqat_status eqat_adamw_step(const eqat_adamw_tensor *tensors, int n_tensors, const eqat_adamw_group *groups,
                            int n_groups, int64_t step, eqat_stream_t stream) {
    DeviceInfo dev;
    if (!tensors || !groups) return fail(EQAT_ERR_NULL, "tensors or groups is NULL");
    if (n_tensors < 0 || n_tensors > EQAT_ADAMW_MAX_TENSORS || n_groups < 1)
        return fail(EQAT_ERR_SHAPE, "n_tensors must be 0..32 and n_groups >= 1");
    if (step < 1) return fail(EQAT_ERR_SHAPE, "step must be >= 1");
    for (int i = 0; i < n_groups; ++i) {
        const eqat_adamw_group &g = groups[i];
        if (!(g.beta1 >= 0.0 && g.beta1 < 1.0 && g.beta2 >= 0.0 && g.beta2 < 1.0 && g.eps > 0.0 && g.lr >= 0.0 &&
              g.weight_decay >= 0.0))
            return fail(EQAT_ERR_UNSUPPORTED, "AdamW hyperparameters out of range");
    }
    eqat::AdamwSeg segs[EQAT_ADAMW_MAX_TENSORS];
    int n = 0;
    for (int i = 0; i < n_tensors; ++i) {
        const eqat_adamw_tensor &t = tensors[i];
        if (t.numel < 0) return fail(EQAT_ERR_SHAPE, "numel < 0");
        if (t.group < 0 || t.group >= n_groups) return fail(EQAT_ERR_SHAPE, "group index out of range");
        if (t.grad_dtype != EQAT_F32 && t.grad_dtype != EQAT_BF16) return fail(EQAT_ERR_DTYPE, "grad_dtype");
        if (t.param_copy && t.copy_dtype != EQAT_F32 && t.copy_dtype != EQAT_BF16) return fail(EQAT_ERR_DTYPE, "copy_dtype");
        EQAT_TRY(check_ptr(t.param, t.numel, "param"));
        EQAT_TRY(check_ptr(t.grad, t.numel, "grad"));
        EQAT_TRY(check_ptr(t.exp_avg, t.numel, "exp_avg"));
        EQAT_TRY(check_ptr(t.exp_avg_sq, t.numel, "exp_avg_sq"));
        EQAT_TRY(check_ptr(t.param_copy, 0, "param_copy"));
        if (t.numel == 0) continue;
        const eqat_adamw_group &g = groups[t.group];
        const double bc1 = 1.0 - std::pow(g.beta1, static_cast<double>(step));
        const double bc2 = 1.0 - std::pow(g.beta2, static_cast<double>(step));
        eqat::AdamwSeg &sg = segs[n++];
        sg.p = t.param;
        sg.g = t.grad;
        sg.m = t.exp_avg;
        sg.v = t.exp_avg_sq;
        sg.copy = t.param_copy;
        sg.n = t.numel;
        sg.g_bf16 = t.grad_dtype == EQAT_BF16;
        sg.copy_bf16 = t.copy_dtype == EQAT_BF16;
        sg.decay = static_cast<float>(1.0 - g.lr * g.weight_decay);
        sg.b1 = static_cast<float>(g.beta1);
        sg.b2 = static_cast<float>(g.beta2);
        sg.omb1 = static_cast<float>(1.0 - g.beta1);
        sg.omb2 = static_cast<float>(1.0 - g.beta2);
        sg.step_size = static_cast<float>(g.lr / bc1);
        sg.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
        sg.eps = static_cast<float>(g.eps);
    }
    if (n == 0) return EQAT_OK;
    EQAT_TRY(get_device(dev));
    EQAT_CUDA(eqat::launch_adamw(segs, n, dev, reinterpret_cast<cudaStream_t>(stream)), "adamw");
    return EQAT_OK;
}

double eqat_cosine_lr(double lr0, double lr_min, int64_t step, int64_t total) {
    if (total <= 0) return lr0;
    const double pi = 3.14159265358979323846;
    return lr_min + (lr0 - lr_min) * (1.0 + std::cos(pi * static_cast<double>(step) / static_cast<double>(total))) / 2.0;
}

eqat_status eqat_device_error(int *where, eqat_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int v = 0;
    e = eqat::read_and_clear_device_error(v);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (where) *where = v;
    if (v != 0) return fail(EQAT_ERR_TIMEOUT, "a bounded on-chip wait ran out");
    return EQAT_OK;
}

eqat_status eqat_selftest_bounded_wait(int64_t timeout_ns, eqat_stream_t stream) {
    if (timeout_ns < 100000 || timeout_ns > 10000000000ll)
        return fail(EQAT_ERR_SHAPE, "timeout_ns must be within 1e5 .. 1e10");
    DeviceInfo dev;
    cudaError_t e = eqat::current_device_info(dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    if (dev.major != 10) return fail(EQAT_ERR_UNSUPPORTED, "needs an sm_100 (B200) device");
    EQAT_CUDA(eqat::launch_selftest_bounded_wait(static_cast<uint64_t>(timeout_ns),
                                                 reinterpret_cast<cudaStream_t>(stream)),
              "selftest launch");
    return EQAT_OK;
}

}  // extern "C"
