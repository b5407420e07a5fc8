/*
 * EfficientQAT fake-quantized linear layer: plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may include,
 * link, load or call this file; it exists so that tests, the smoke check and the
 * CPU baseline of bench.py can check the CUDA path against a slow, obviously
 * correct restatement of what the pages define.  It shares no code, header,
 * constant or helper with the CUDA sources.
 *
 * Sources (web pages on EfficientQAT, arXiv 2407.11062):
 *   [MF]  modelfoundations.com note "EfficientQAT, low-bit training on a single
 *         GPU": Phase 1 (Block-AP, min-max init), Phase 2 (E2E-QP, exact
 *         dW-hat/ds = W_int - z), "Paper vs. code" (round_ste on z every forward,
 *         hard-rounded z at pack time).
 *   [PL]  paperlayer.ai summary "EfficientQAT: Efficient Quantization-Aware
 *         Training for Large Language Models": section 3 (quant/dequant inside
 *         the graph), appendix A (straight-through estimator through rounding for
 *         s, z and W), appendix D (groups of g weights share a step size and an
 *         N-bit zero point).
 *   [ZN]  zhaoyang97 ACL2025 paper notes "EfficientQAT": Block-AP Eq. 1
 *         W_int = clamp(round(W/s) + z, 0, 2^N - 1), Eq. 2 W-hat = (W_int - z) s;
 *         E2E-QP gradient dW-hat/ds = w_q - z.
 *
 * Precision: the quantizer's element math is IEEE fp32 (round-to-nearest
 * division, round-half-even rintf), compiled with -ffp-contract=off and without
 * fast-math so that no step is fused or reassociated.  Contractions and
 * reductions accumulate in fp64 (fp32 x fp32 products are exact in fp64).
 *
 * Readings where the pages are silent:
 *   round()            = round-half-to-even (rintf under the default mode);
 *   W / s              = one correctly rounded fp32 division (never x * (1/s));
 *   s                  = (xmax - xmin) / (2^N - 1) in fp32, then max(s, 1e-5);
 *   z during Block-AP  = a float that is rounded (zr = rint(z)) in every forward;
 *   clamp gradient     = passes only where 0 <= round(W/s) + zr <= 2^N - 1
 *                        (inclusive bounds); round has identity gradient;
 *                        orc_ste_grads_clamp_pass is the all-pass variant;
 *   E2E zero point     = dz of W-hat = (W_q - z) s at z = zq (z as a float);
 *   fp16 step storage  = s widened exactly to fp32 before any arithmetic;
 *   pack               = zq = clamp(rint(z), 0, Q) as uint8, codes recomputed
 *                        with zr := zq; 2-bit: 4 codes per byte, code k at bits
 *                        2*(k%4); 4-bit: 2 per byte at bits 4*(k%2); 3-bit: one
 *                        code per byte; packed along K, row-major.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORC_S_MIN 1e-5f

static float orc_qmax(int bits) { return (float)((1 << bits) - 1); }

/* [MF] Phase 1 "Initialization": per-group min-max,
 * s = (xmax - xmin) / (2^N - 1), z = round(-xmin / s).  Groups are g consecutive
 * in-features of one output row ([PL] appendix D). */
void orc_minmax_init(const float *W, int64_t N, int64_t K, int bits, int group,
                     float *s, float *z)
{
    const int64_t G = K / group;
    const float Q = orc_qmax(bits);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < G; ++j) {
            const float *w = W + n * K + j * group;
            float xmin = w[0], xmax = w[0];
            for (int i = 1; i < group; ++i) {
                if (w[i] < xmin) xmin = w[i];
                if (w[i] > xmax) xmax = w[i];
            }
            float range = xmax - xmin;
            float sc = range / Q;
            if (!(sc >= ORC_S_MIN)) sc = ORC_S_MIN;
            float neg = -xmin;
            float zz = rintf(neg / sc);
            s[n * G + j] = sc;
            z[n * G + j] = zz;
        }
    }
}

/* [ZN] Eq. 1 and Eq. 2 with [MF] "round_ste on z every forward":
 *   zr = round(z); u = W/s; q = round(u) + zr; W_int = clamp(q, 0, Q);
 *   mask = [0 <= q <= Q]; W-hat = (W_int - zr) * s.
 * Any output pointer may be NULL. */
void orc_fake_quant(const float *W, const float *s, const float *z, int64_t N,
                    int64_t K, int bits, int group, float *What, uint8_t *code,
                    uint8_t *mask, float *u_out)
{
    const int64_t G = K / group;
    const float Q = orc_qmax(bits);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            const int64_t gi = n * G + k / group;
            const float sc = s[gi];
            const float zr = rintf(z[gi]);
            const float w = W[n * K + k];
            const float u = w / sc;
            const float r = rintf(u);
            const float q = r + zr;
            float c = q;
            if (c < 0.0f) c = 0.0f;
            if (c > Q) c = Q;
            const int inside = (q >= 0.0f) && (q <= Q);
            const float diff = c - zr;
            const float wh = diff * sc;
            if (What) What[n * K + k] = wh;
            if (code) code[n * K + k] = (uint8_t)c;
            if (mask) mask[n * K + k] = (uint8_t)inside;
            if (u_out) u_out[n * K + k] = u;
        }
    }
}

/* [MF] "Paper vs. code": z is hard-rounded at pack time; [MF] Phase 2: "pack the
 * weights into real integers"; [PL] appendix D: N-bit zero point per group.
 * Bytes per row: K/4 (2-bit), K/2 (4-bit), K (3-bit, one code per byte). */
void orc_pack(const float *W, const float *s, const float *z, int64_t N, int64_t K,
              int bits, int group, uint8_t *packed, uint8_t *zq)
{
    const int64_t G = K / group;
    const float Q = orc_qmax(bits);
    const int per_byte = (bits == 2) ? 4 : (bits == 4) ? 2 : 1;
    const int64_t row_bytes = K / per_byte;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < G; ++j) {
            float zr = rintf(z[n * G + j]);
            if (zr < 0.0f) zr = 0.0f;
            if (zr > Q) zr = Q;
            zq[n * G + j] = (uint8_t)zr;
        }
        memset(packed + n * row_bytes, 0, (size_t)row_bytes);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t gi = n * G + k / group;
            const float sc = s[gi];
            const float zr = (float)zq[gi];
            const float u = W[n * K + k] / sc;
            float c = rintf(u) + zr;
            if (c < 0.0f) c = 0.0f;
            if (c > Q) c = Q;
            const unsigned code = (unsigned)c;
            if (per_byte == 1) {
                packed[n * row_bytes + k] = (uint8_t)code;
            } else {
                const int shift = bits * (int)(k % per_byte);
                packed[n * row_bytes + k / per_byte] |= (uint8_t)(code << shift);
            }
        }
    }
}

/* Reads code (n, k) back out of the packed layout defined for orc_pack. */
static unsigned orc_code_at(const uint8_t *packed, int64_t K, int bits, int64_t n, int64_t k)
{
    const int per_byte = (bits == 2) ? 4 : (bits == 4) ? 2 : 1;
    const int64_t row_bytes = K / per_byte;
    const uint8_t byte = packed[n * row_bytes + k / per_byte];
    if (per_byte == 1) return byte;
    const int shift = bits * (int)(k % per_byte);
    return (byte >> shift) & ((1u << bits) - 1u);
}

/* [MF] Phase 2 / [ZN] Eq. 2 on frozen integers: W-hat = (W_q - z) * s. */
void orc_dequant_packed(const uint8_t *packed, const uint8_t *zq, const float *s,
                        int64_t N, int64_t K, int bits, int group, float *What)
{
    const int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            const int64_t gi = n * G + k / group;
            const float c = (float)orc_code_at(packed, K, bits, n, k);
            const float diff = c - (float)zq[gi];
            What[n * K + k] = diff * s[gi];
        }
    }
}

/* Forward Y = X W-hat^T ([PL] section 3: the dequantized weight feeds the
 * layer), for the token rows listed in `rows` (all rows when rows == NULL).
 * Y is [nrows, N], fp64. */
void orc_linear_fwd(const float *X, const float *What, int64_t M, int64_t N, int64_t K,
                    const int64_t *rows, int64_t nrows, double *Y)
{
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t m = rows ? rows[r] : r;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += (double)X[m * K + k] * (double)What[n * K + k];
            Y[r * N + n] = acc;
        }
    }
}

/* Chain rule on Y = X W-hat^T: dX = dY W-hat (W-hat does not depend on X).
 * dX is [nrows, K], fp64. */
void orc_linear_dx(const float *dY, const float *What, int64_t M, int64_t N, int64_t K,
                   const int64_t *rows, int64_t nrows, double *dX)
{
    if (!rows) nrows = M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t m = rows ? rows[r] : r;
        double *out = dX + r * K;
        for (int64_t k = 0; k < K; ++k) out[k] = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double g = (double)dY[m * N + n];
            for (int64_t k = 0; k < K; ++k)
                out[k] += g * (double)What[n * K + k];
        }
    }
}

/* Chain rule on Y = X W-hat^T: dW-hat = dY^T X, for the weight rows listed in
 * `wrows` (all when NULL).  dWhat is [nw, K], fp64. */
void orc_linear_dwhat(const float *dY, const float *X, int64_t M, int64_t N, int64_t K,
                      const int64_t *wrows, int64_t nw, double *dWhat)
{
    if (!wrows) nw = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nw; ++r) {
        const int64_t n = wrows ? wrows[r] : r;
        double *out = dWhat + r * K;
        for (int64_t k = 0; k < K; ++k) out[k] = 0.0;
        for (int64_t m = 0; m < M; ++m) {
            const double g = (double)dY[m * N + n];
            for (int64_t k = 0; k < K; ++k)
                out[k] += g * (double)X[m * K + k];
        }
    }
}

/* Block-AP straight-through backward ([PL] appendix A: gradients of W, s and z
 * through the rounding by the straight-through estimator; [MF] round_ste on z).
 * With round's gradient taken as identity and clamp passing the gradient only
 * inside [0, Q]:
 *   dW-hat/dW  = mask
 *   dW-hat/ds  = (W_int - zr) - mask * W/s
 *   dW-hat/dzr = s * (mask - 1),   dzr/dz = 1
 * so, per weight row n (listed in wrows) and group j,
 *   dW[n,k] = dWhat[n,k] * mask[n,k]
 *   ds[n,j] = sum_{k in j} dWhat[n,k] * ((W_int - zr) - mask * u)
 *   dz[n,j] = sum_{k in j} dWhat[n,k] * s * (mask - 1).
 * dWhat rows follow wrows; dW is [nw, K], ds and dz are [nw, G], all fp64. */
void orc_ste_grads(const float *W, const float *s, const float *z, const double *dWhat,
                   const int64_t *wrows, int64_t nw, int64_t N, int64_t K, int bits,
                   int group, double *dW, double *ds, double *dz)
{
    const int64_t G = K / group;
    const float Q = orc_qmax(bits);
    if (!wrows) nw = N;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nw; ++r) {
        const int64_t n = wrows ? wrows[r] : r;
        for (int64_t j = 0; j < G; ++j) {
            const float sc = s[n * G + j];
            const float zr = rintf(z[n * G + j]);
            double acc_s = 0.0, acc_z = 0.0;
            for (int i = 0; i < group; ++i) {
                const int64_t k = j * group + i;
                const float u = W[n * K + k] / sc;
                const float q = rintf(u) + zr;
                float c = q;
                if (c < 0.0f) c = 0.0f;
                if (c > Q) c = Q;
                const int inside = (q >= 0.0f) && (q <= Q);
                const double g = dWhat[r * K + k];
                if (dW) dW[r * K + k] = inside ? g : 0.0;
                const double dwds = (double)(c - zr) - (inside ? (double)u : 0.0);
                acc_s += g * dwds;
                acc_z += g * (double)sc * (double)(inside - 1);
            }
            if (ds) ds[r * G + j] = acc_s;
            if (dz) dz[r * G + j] = acc_z;
        }
    }
}

/* E2E-QP scale gradient ([MF] Phase 2, [ZN] E2E-QP): W-hat is linear in s with
 * dW-hat/ds = W_q - z exactly, so ds[n,j] = sum_{k in j} dWhat[n,k] * (W_q - z). */
void orc_e2e_ds(const uint8_t *packed, const uint8_t *zq, const double *dWhat,
                const int64_t *wrows, int64_t nw, int64_t N, int64_t K, int bits,
                int group, double *ds)
{
    const int64_t G = K / group;
    if (!wrows) nw = N;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nw; ++r) {
        const int64_t n = wrows ? wrows[r] : r;
        for (int64_t j = 0; j < G; ++j) {
            double acc = 0.0;
            for (int i = 0; i < group; ++i) {
                const int64_t k = j * group + i;
                const double diff = (double)orc_code_at(packed, K, bits, n, k) - (double)zq[n * G + j];
                acc += dWhat[r * K + k] * diff;
            }
            ds[r * G + j] = acc;
        }
    }
}

/* Variant of orc_ste_grads in which the clamp is straight-through as well (the
 * all-pass clamp_ste that [MF] "Paper vs. code" finds defined in the quantizer
 * but whose use the pages leave unstated).  With round and clamp both identity
 * in the backward pass, W-hat = (clamp(round(W/s) + zr, 0, Q) - zr) s gives
 *   dW-hat/dW  = (1/s) s                  = 1,
 *   dW-hat/ds  = (c - zr) + s (-W / s^2)  = (c - zr) - u,
 *   dW-hat/dzr = s (1 - 1)                = 0,
 * for every element, clamped or not. */
void orc_ste_grads_clamp_pass(const float *W, const float *s, const float *z, const double *dWhat,
                              const int64_t *wrows, int64_t nw, int64_t N, int64_t K, int bits,
                              int group, double *dW, double *ds, double *dz)
{
    const int64_t G = K / group;
    const float Q = orc_qmax(bits);
    if (!wrows) nw = N;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nw; ++r) {
        const int64_t n = wrows ? wrows[r] : r;
        for (int64_t j = 0; j < G; ++j) {
            const float sc = s[n * G + j];
            const float zr = rintf(z[n * G + j]);
            double acc_s = 0.0;
            for (int i = 0; i < group; ++i) {
                const int64_t k = j * group + i;
                const float u = W[n * K + k] / sc;
                float c = rintf(u) + zr;
                if (c < 0.0f) c = 0.0f;
                if (c > Q) c = Q;
                const double g = dWhat[r * K + k];
                if (dW) dW[r * K + k] = g;
                acc_s += g * ((double)(c - zr) - (double)u);
            }
            if (ds) ds[r * G + j] = acc_s;
            if (dz) dz[r * G + j] = 0.0;
        }
    }
}

/* E2E-QP with the zero point trained too (a float z evaluated at the frozen zq):
 * W-hat = (W_q - z) s ([ZN] Eq. 2, [MF] Phase 2) is linear in z with
 * dW-hat/dz = -s, so dz[n,j] = -s[n,j] * sum_{k in j} dWhat[n,k]. */
void orc_e2e_dz(const float *s, const double *dWhat, const int64_t *wrows, int64_t nw, int64_t N,
                int64_t K, int group, double *dz)
{
    const int64_t G = K / group;
    if (!wrows) nw = N;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nw; ++r) {
        const int64_t n = wrows ? wrows[r] : r;
        for (int64_t j = 0; j < G; ++j) {
            double acc = 0.0;
            for (int i = 0; i < group; ++i) acc += dWhat[r * K + j * group + i];
            dz[r * G + j] = -(double)s[n * G + j] * acc;
        }
    }
}

/* One AdamW step (decoupled weight decay) at step t >= 1 over n parameters, for
 * the Block-AP update of W, s and z ([MF] Phase 1 and "Paper vs. code": AdamW,
 * weights and quantization parameters in separate learning-rate groups).  The
 * pages print no formula; this is the textbook algorithm of Loshchilov & Hutter
 * as PyTorch's AdamW states it:
 *   p <- p (1 - lr wd)
 *   m <- b1 m + (1 - b1) g,   v <- b2 v + (1 - b2) g^2
 *   p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * in fp64 on fp32 state, each stored value rounded to fp32 once. */
void orc_adamw(float *p, const float *g, float *m, float *v, int64_t n, double lr, double b1, double b2,
               double eps, double wd, int64_t t)
{
    const double bc1 = 1.0 - pow(b1, (double)t);
    const double bc2 = 1.0 - pow(b2, (double)t);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const double gi = (double)g[i];
        double pi = (double)p[i] * (1.0 - lr * wd);
        const double mi = b1 * (double)m[i] + (1.0 - b1) * gi;
        const double vi = b2 * (double)v[i] + (1.0 - b2) * gi * gi;
        const float m32 = (float)mi, v32 = (float)vi;
        pi -= lr * ((double)m32 / bc1) / (sqrt((double)v32 / bc2) + eps);
        m[i] = m32;
        v[i] = v32;
        p[i] = (float)pi;
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
