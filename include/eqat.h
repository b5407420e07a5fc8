/*
 * eqat.h: C ABI of the B200 (sm_100a) fake-quantized linear layer of
 * EfficientQAT (Efficient Quantization-Aware Training for LLMs, arXiv 2407.11062).
 *
 * The layer quantizes each group of g consecutive in-features of an output row
 * with a step s and a zero point z (paperlayer.ai summary, appendix D):
 *   W_int = clamp(round(W / s) + z, 0, 2^b - 1)        (Eq. 1)
 *   W-hat = (W_int - z) * s                            (Eq. 2)
 * (zhaoyang97 ACL2025 notes, "Block-AP"), initialised per group by min-max
 * (modelfoundations.com note "EfficientQAT, low-bit training on a single GPU",
 * Phase 1), trained with a straight-through backward in Block-AP (paperlayer
 * appendix A) and, on frozen packed codes, with the exact scale gradient
 * dW-hat/ds = W_q - z in E2E-QP (modelfoundations Phase 2).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout: all matrices are dense, row-major and contiguous.
 *   X, dX      [M, K]  tokens x in-features
 *   W, dW, W-hat [N, K] out-features x in-features
 *   Y, dY      [M, N]
 *   s, z, ds, dz, zq [N, G], G = K / group  (group j of row n covers columns
 *              j*group .. j*group + group - 1)
 *   codes      [N, K/4] bytes for 2-bit (code of column k in bits 2*(k%4)),
 *              [N, K/2] for 4-bit (bits 4*(k%2)), [N, K] for 3-bit (one code
 *              per byte, unpacked).
 * Dtypes: X, W, Y, dY, dX, dW, W-hat share `dt` (EQAT_BF16 or EQAT_F32); s, z, ds,
 *   dz are fp32; codes and zq are uint8.  In EQAT_BF16 mode the contractions run
 *   on tcgen05 tensor cores with bf16 operands (W-hat rounded to bf16 to nearest
 *   even) and fp32 accumulation; in EQAT_F32 mode they run in fp32 on the CUDA
 *   cores.  The quantizer's element arithmetic is IEEE fp32 in both modes:
 *   W / s is a correctly rounded division and round() is half-to-even.
 * Quantizer readings (the pages leave these open): z is a float that every
 *   forward rounds (zr = round(z)); s = (xmax - xmin) / (2^b - 1) is floored at
 *   EQAT_S_MIN; the straight-through backward gives round an identity gradient
 *   and lets clamp pass the gradient only where 0 <= round(W/s) + zr <= 2^b - 1
 *   (bounds included).
 * Supported: bits in {2, 3, 4}; group in {32, 64, 128}; K % group == 0;
 *   N % 8 == 0; M, N, K >= 0 (empty problems are valid and write only what has
 *   a defined value, e.g. zero gradients when M == 0).
 * Pointers: device memory (cudaMalloc / PyTorch CUDA tensors) of the current
 *   device, 16-byte aligned, not overlapping one another.  The caller owns every
 *   buffer; the library allocates nothing and keeps no state beyond cached
 *   device attributes.  Outputs are overwritten (gradients are not accumulated).
 *   NULL optional outputs skip their work.
 * Workspace: entry points that take (ws, ws_bytes) need at least
 *   eqat_workspace_bytes(...) bytes of device scratch, 256-byte aligned; it
 *   holds W-hat between the quantizer prepass and the contractions.
 * Streams: every call enqueues its kernels on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream) and returns without synchronising.
 * Errors: argument errors are detected on the host before anything is launched
 *   and return EQAT_ERR_NULL / _SHAPE / _ALIGN / _DTYPE / _UNSUPPORTED /
 *   _WORKSPACE.  A launch failure returns EQAT_ERR_CUDA.  Kernels that wait on
 *   on-chip barriers bound every wait; a wait that runs out records
 *   EQAT_ERR_TIMEOUT in a device error word, the kernel releases what it holds
 *   and returns, and eqat_device_error() reports it.  No call aborts the process
 *   or lets an exception escape.
 */
#ifndef EQAT_H
#define EQAT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EQAT_VERSION 1
#define EQAT_S_MIN 1e-5f

typedef struct CUstream_st *eqat_stream_t; /* same type as cudaStream_t */

typedef enum {
    EQAT_OK = 0,
    EQAT_ERR_NULL = 1,        /* a required pointer is NULL */
    EQAT_ERR_SHAPE = 2,       /* negative size, K % group, N % 8, size overflow */
    EQAT_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned (ws: 256) */
    EQAT_ERR_DTYPE = 4,       /* unknown eqat_dtype */
    EQAT_ERR_UNSUPPORTED = 5, /* bits or group outside the supported set; no sm_100 device */
    EQAT_ERR_WORKSPACE = 6,   /* ws NULL or smaller than eqat_workspace_bytes() */
    EQAT_ERR_CUDA = 7,        /* a CUDA runtime / launch error */
    EQAT_ERR_TIMEOUT = 8      /* a bounded on-chip wait ran out (see eqat_device_error) */
} eqat_status;

/* EQAT_F16 is accepted only for the step size s of the E2E-QP entry points
 * that take an `sdt` argument (the pages' fp16 step-size storage). */
typedef enum { EQAT_F32 = 0, EQAT_BF16 = 1, EQAT_F16 = 2 } eqat_dtype;

/* Flags of eqat_fq_linear_bwd_ex. */
#define EQAT_GRAD_CLAMP_PASS 1u /* clamp straight-through too: dW = dY^T X, dz = 0,
                                   ds = sum_group (dY^T X) ((code - zr) - u) */

/* Human-readable name of a status; never NULL. */
const char *eqat_status_string(int status);

/* Detail of the last error returned on the calling thread (empty if none). */
const char *eqat_last_error_detail(void);

/* Library ABI version (EQAT_VERSION). */
int eqat_version(void);

/* Bytes of device workspace that the linear entry points need for this shape
 * (0 when none): W-hat (N K elements of dt; fp32 mode also an fp32 N K scratch),
 * and for eqat_dq_linear_fwd at decode sizes (bf16, 1 <= M <= 8, group 64 or
 * 128) the larger of that and the decode path's scratch (per-row-tile partial
 * sums, at most M N K / 128 bytes, which a W-hat-sized workspace always holds;
 * a smaller one makes the call dequantize W-hat and run the GEMM instead). */
size_t eqat_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int group, int dt);

/* a1. Per-group min-max initialisation (modelfoundations note, Phase 1):
 *   s[n,j] = max((xmax - xmin) / (2^b - 1), EQAT_S_MIN)   fp32, IEEE division
 *   z[n,j] = round(-xmin / s[n,j])                        fp32, integer-valued
 * W [N,K] of dtype wdt (bf16 or fp32); s, z [N,G] fp32 outputs. */
eqat_status eqat_minmax_init(const void *W, int wdt, int64_t N, int64_t K, int bits, int group,
                             float *s, float *z, eqat_stream_t stream);

/* a2. The quantizer prepass on its own (Eq. 1 with round(z), Eq. 2):
 *   u = W/s, q = round(u) + round(z), code = clamp(q, 0, 2^b-1),
 *   mask = [0 <= q <= 2^b-1], W_hat = (code - round(z)) * s.
 * W_hat [N,K] has dtype wdt (bf16: rounded to nearest even); code and mask
 * [N,K] uint8 are optional (NULL skips).  W_hat may be NULL too. */
eqat_status eqat_fake_quant(const void *W, int wdt, const float *s, const float *z, int64_t N,
                            int64_t K, int bits, int group, void *W_hat, uint8_t *code,
                            uint8_t *mask, eqat_stream_t stream);

/* a7. Pack to low-bit integers (modelfoundations note, "Paper vs. code": z is
 * hard-rounded at pack time; Phase 2: the weights become real integers):
 *   zq = clamp(round(z), 0, 2^b-1) (uint8 [N,G]),
 *   codes = clamp(round(W/s) + zq, 0, 2^b-1) packed as described above. */
eqat_status eqat_pack_codes(const void *W, int wdt, const float *s, const float *z, int64_t N,
                            int64_t K, int bits, int group, uint8_t *codes, uint8_t *zq,
                            eqat_stream_t stream);

/* a1 and a7 over the weight matrices of a whole block in one launch per eight
 * layers (the 70B Block-AP sweep initialises and packs all seven linears of a
 * decoder block together; small layers then share the waves of large ones
 * instead of paying a launch ramp and tail each).  Layer i has W[i] [N[i], K[i]]
 * and the outputs of eqat_minmax_init / eqat_pack_codes for it; results equal n
 * single calls, bit for bit.  W, N, K, s, z, codes, zq are HOST arrays of n
 * entries (0 <= n <= EQAT_MAX_MULTI) holding device pointers and sizes; every
 * layer has dtype wdt and the same bits and group.  The layers' buffers must not
 * overlap.  Arguments are checked layer by layer before any launch; an error
 * launches nothing. */
#define EQAT_MAX_MULTI 64
eqat_status eqat_minmax_init_multi(int n, const void *const *W, int wdt, const int64_t *N, const int64_t *K,
                                   int bits, int group, float *const *s, float *const *z,
                                   eqat_stream_t stream);
eqat_status eqat_pack_codes_multi(int n, const void *const *W, int wdt, const float *const *s,
                                  const float *const *z, const int64_t *N, const int64_t *K, int bits,
                                  int group, uint8_t *const *codes, uint8_t *const *zq,
                                  eqat_stream_t stream);

/* a3 (E2E-QP). Eq. 2 on frozen codes: W_hat = (W_q - zq) * s, dtype dt. */
eqat_status eqat_dequant_codes(const uint8_t *codes, const uint8_t *zq, const float *s, int64_t N,
                               int64_t K, int bits, int group, void *W_hat, int dt,
                               eqat_stream_t stream);

/* a2-a4. Block-AP forward: Y = X W_hat^T with W_hat from (W, s, z) as in
 * eqat_fake_quant (paperlayer section 3: quantization and dequantization sit
 * inside the computation graph).  Y [M,N] of dtype dt. */
eqat_status eqat_fq_linear_fwd(const void *X, const void *W, int dt, const float *s,
                               const float *z, void *Y, int64_t M, int64_t N, int64_t K,
                               int bits, int group, void *ws, size_t ws_bytes,
                               eqat_stream_t stream);

/* a5-a6. Block-AP straight-through backward (paperlayer appendix A):
 *   dX = dY W_hat                                   [M,K], dtype dt   (nullable)
 *   dW = (dY^T X) * mask                            [N,K], dtype dt   (nullable)
 *   ds = sum_group (dY^T X) ((code - zr) - mask*u)  [N,G], fp32       (nullable)
 *   dz = sum_group (dY^T X) s (mask - 1)            [N,G], fp32       (nullable)
 * with u, code, mask, zr as in eqat_fake_quant.  dY^T X is formed in fp32 on
 * chip and never stored; the mask, ds and dz reductions run in the epilogue of
 * that contraction.  In EQAT_BF16 mode both contractions run in one grouped
 * persistent launch.  w_hat_in_ws != 0 promises that ws already holds W_hat for
 * these (W, s, z, bits, group), as eqat_fq_linear_fwd leaves it on the same
 * stream, and skips the quantizer prepass (training: forward, then backward with
 * the same workspace). */
eqat_status eqat_fq_linear_bwd(const void *X, const void *W, int dt, const float *s,
                               const float *z, const void *dY, void *dX, void *dW, float *ds,
                               float *dz, int64_t M, int64_t N, int64_t K, int bits, int group,
                               void *ws, size_t ws_bytes, int w_hat_in_ws, eqat_stream_t stream);

/* a8. E2E-QP forward on frozen codes (modelfoundations Phase 2: only
 * dequantization in the graph): Y = X ((W_q - zq) s)^T.  With a workspace, W-hat
 * is dequantized into it first and stays there for eqat_dq_linear_bwd_s
 * (w_hat_in_ws = 1).  In bf16 mode ws may be NULL (ws_bytes 0): W-hat is then made
 * from the codes inside the contraction and kept nowhere (forward-only use; a
 * backward after it takes w_hat_in_ws = 0).  That needs rows of codes a multiple of
 * 16 bytes (K * bits / 8, or K for 3-bit codes); otherwise a NULL workspace is
 * EQAT_ERR_WORKSPACE.  At decode sizes (bf16, 1 <= M <= 8, group 64 or 128, with a
 * workspace) the codes are streamed once and W-hat is never written: the inference
 * GEMV of the packed model. */
eqat_status eqat_dq_linear_fwd(const void *X, int dt, const uint8_t *codes, const uint8_t *zq,
                               const float *s, void *Y, int64_t M, int64_t N, int64_t K, int bits,
                               int group, void *ws, size_t ws_bytes, eqat_stream_t stream);

/* a9. E2E-QP backward, scales only (modelfoundations Phase 2; zhaoyang97 notes,
 * E2E-QP: dW-hat/ds = w_q - z, no straight-through estimator):
 *   dX = dY W_hat (nullable),  ds = sum_group (dY^T X) (W_q - zq).
 * w_hat_in_ws as for eqat_fq_linear_bwd (ws holds W_hat from eqat_dq_linear_fwd). */
eqat_status eqat_dq_linear_bwd_s(const void *X, int dt, const uint8_t *codes, const uint8_t *zq,
                                 const float *s, const void *dY, void *dX, float *ds, int64_t M,
                                 int64_t N, int64_t K, int bits, int group, void *ws,
                                 size_t ws_bytes, int w_hat_in_ws, eqat_stream_t stream);

/* Quantizer variants (the pages leave these open or mention them in passing).
 *
 * eqat_fq_linear_bwd_ex: eqat_fq_linear_bwd with `flags`.  flags == 0 is
 * eqat_fq_linear_bwd.  EQAT_GRAD_CLAMP_PASS gives the clamp an identity
 * gradient as well (the all-pass clamp_ste of the modelfoundations note, "Paper
 * vs. code"): dW = dY^T X, ds = sum_group (dY^T X) ((code - zr) - u), dz = 0.
 * Unknown flag bits return EQAT_ERR_UNSUPPORTED. */
eqat_status eqat_fq_linear_bwd_ex(const void *X, const void *W, int dt, const float *s,
                                  const float *z, const void *dY, void *dX, void *dW, float *ds,
                                  float *dz, int64_t M, int64_t N, int64_t K, int bits, int group,
                                  uint32_t flags, void *ws, size_t ws_bytes, int w_hat_in_ws,
                                  eqat_stream_t stream);

/* eqat_dequant_codes / eqat_dq_linear_fwd with the step size s of dtype sdt:
 * EQAT_F32 or EQAT_F16 (paperlayer appendix D: a shared FP16 step size per
 * group).  An fp16 s is widened exactly to fp32 before any arithmetic. */
eqat_status eqat_dequant_codes_ex(const uint8_t *codes, const uint8_t *zq, const void *s, int sdt,
                                  int64_t N, int64_t K, int bits, int group, void *W_hat, int dt,
                                  eqat_stream_t stream);
eqat_status eqat_dq_linear_fwd_ex(const void *X, int dt, const uint8_t *codes, const uint8_t *zq,
                                  const void *s, int sdt, void *Y, int64_t M, int64_t N, int64_t K,
                                  int bits, int group, void *ws, size_t ws_bytes,
                                  eqat_stream_t stream);

/* E2E-QP backward with the zero point trained as well (z a float evaluated at
 * the frozen zq): W_hat = (W_q - z) s gives
 *   dX = dY W_hat                          (nullable)
 *   ds = sum_group (dY^T X) (W_q - zq)     (nullable)
 *   dz = -s * sum_group (dY^T X)           (nullable)
 * s of dtype sdt (EQAT_F32 or EQAT_F16); ds and dz fp32.  With dz == NULL and
 * sdt == EQAT_F32 this is eqat_dq_linear_bwd_s. */
eqat_status eqat_dq_linear_bwd(const void *X, int dt, const uint8_t *codes, const uint8_t *zq,
                               const void *s, int sdt, const void *dY, void *dX, float *ds,
                               float *dz, int64_t M, int64_t N, int64_t K, int bits, int group,
                               void *ws, size_t ws_bytes, int w_hat_in_ws, eqat_stream_t stream);

/* Block-AP step (modelfoundations note, Phase 1: each block is trained against the
 * full-precision block's outputs with an MSE loss, by AdamW with the weights and
 * the quantization parameters in separate learning-rate groups on cosine
 * schedules).
 *
 * eqat_fq_linear_fwd_mse: the forward of eqat_fq_linear_fwd against a target T
 * (the full-precision output, [M,N] of dtype dt), without storing Y:
 *   dY = 2 (Y - T) / (M N)   [M,N], dtype dt (the loss gradient, input of eqat_fq_linear_bwd)
 *   *loss = sum (Y - T)^2 / (M N)   one fp64 value in device memory, 8-byte aligned (overwritten)
 * In EQAT_BF16 mode the subtraction runs on Y's fp32 accumulator in the GEMM
 * epilogue; the loss is summed with atomics, so its last bits depend on order. */
eqat_status eqat_fq_linear_fwd_mse(const void *X, const void *W, int dt, const float *s, const float *z,
                                   const void *T, void *dY, double *loss, int64_t M, int64_t N, int64_t K,
                                   int bits, int group, void *ws, size_t ws_bytes, eqat_stream_t stream);

/* One AdamW step (decoupled weight decay, Loshchilov & Hutter; the pages print
 * no formula) over up to 32 tensors in one launch, step >= 1:
 *   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
 *   p <- p - lr / (1 - b1^step) * m / (sqrt(v) / sqrt(1 - b2^step) + eps)
 * in fp32.  param, exp_avg, exp_avg_sq are fp32 device arrays updated in place;
 * grad is EQAT_F32 or EQAT_BF16; param_copy (nullable) receives the updated
 * parameter in copy_dtype (EQAT_BF16 for the weights the next forward reads, or
 * EQAT_F32).  All pointers 16-byte aligned.  Hyperparameters come from
 * groups[tensor.group] (double: 1 - beta2 is formed before rounding to the
 * kernel's fp32 constants); the bias corrections are computed here in double. */
typedef struct {
    float *param;
    const void *grad;
    int grad_dtype;
    float *exp_avg;
    float *exp_avg_sq;
    void *param_copy;
    int copy_dtype;
    int group;
    int64_t numel;
} eqat_adamw_tensor;

typedef struct {
    double lr;
    double beta1;
    double beta2;
    double eps;
    double weight_decay;
} eqat_adamw_group;

#define EQAT_ADAMW_MAX_TENSORS 32
eqat_status eqat_adamw_step(const eqat_adamw_tensor *tensors, int n_tensors, const eqat_adamw_group *groups,
                            int n_groups, int64_t step, eqat_stream_t stream);

/* Cosine annealing (host): lr_min + (lr0 - lr_min) (1 + cos(pi step / total)) / 2,
 * step in [0, total]; the learning rate of step `step` of a schedule of `total`. */
double eqat_cosine_lr(double lr0, double lr_min, int64_t step, int64_t total);

/* Block-AP forward (as eqat_fq_linear_fwd) that allocates nothing and takes no
 * workspace: the paper has no counterpart; this entry point exists for callers of
 * the library that cannot allocate device memory or pass a scratch buffer (a
 * plugin or custom-operator interface that hands over only inputs and outputs, a
 * process that must not call cudaMalloc once running because it can stall the
 * whole device, memory owned by an allocator the library cannot reach).
 * W_hat lives in a static device array of EQAT_NOALLOC_SCRATCH_BYTES (32 MiB)
 * that the library holds on every GPU that loads it, until the process exits.
 * Limit: N * K * sizeof(dtype) <= EQAT_NOALLOC_SCRATCH_BYTES (16 Mi bf16 or 8 Mi
 * fp32 weights); larger layers are rejected with EQAT_ERR_WORKSPACE before
 * anything is launched.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress), so make that first call before any stream
 * capture.  That address is cached per device for the life of the process, so a
 * cudaDeviceReset (or any reset of the primary context) is not supported once
 * this entry point has run on that device: later calls would use the stale
 * address.  Every call shares the one array: calls whose kernels overlap on the
 * GPU (other streams, other host threads) race on it and must be serialised by
 * the caller.  Arguments, layout and the result are those of eqat_fq_linear_fwd. */
#define EQAT_NOALLOC_SCRATCH_BYTES 33554432u
eqat_status eqat_fq_linear_fwd_noalloc(const void *X, const void *W, int dt, const float *s,
                                       const float *z, void *Y, int64_t M, int64_t N, int64_t K,
                                       int bits, int group, eqat_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns EQAT_OK, EQAT_ERR_TIMEOUT if a bounded wait ran out
 * since the last call, or EQAT_ERR_CUDA if the synchronisation failed.  If
 * where != NULL it receives the raw error word (0 when clean). */
eqat_status eqat_device_error(int *where, eqat_stream_t stream);

/* Failure-detection self-test: launches one block whose single thread waits on
 * an on-chip barrier that nothing arrives on, with a bound of timeout_ns
 * nanoseconds (1e5 .. 1e10).  The wait runs out, records EQAT_ERR_TIMEOUT in
 * the device error word and the kernel returns normally; the context stays
 * usable.  Used by the tests of the bounded-wait path. */
eqat_status eqat_selftest_bounded_wait(int64_t timeout_ns, eqat_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EQAT_H */
