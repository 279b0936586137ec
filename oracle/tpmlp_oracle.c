/*
 * fp64 CPU oracle for the tensor-parallel Transformer MLP block.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the bench's CPU
 * baseline use it. It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes (page "Megatron", zzmblog.top, section
 * "张量并行 / 数学原理" and "Transformer层的张量并行实现"): the MLP's first
 * linear layer is Y = X·A with A (h × 4h) split by columns, A = [A_1 … A_p];
 * the second is Z = Y·B with B (4h × h) split by rows, Z = Σ_i Y_i·B_i. The
 * column split gives Y = [X·A_1, …, X·A_p] exactly and the row split's sum is
 * exactly Y·B, so the unsplit definition is the oracle:
 *
 *   H = X·A + 1·aᵀ        (T × F)      pre-activation, kept for the backward
 *   Y = GeLU(H)                        GeLU(x) = x·Φ(x) = ½·x·(1 + erf(x/√2))
 *   Z = Y·B + 1·bᵀ        (T × h)
 *
 * and, for an upstream gradient dZ, the chain rule:
 *
 *   db = 1ᵀ·dZ,  dB = Yᵀ·dZ,  dY = dZ·Bᵀ,
 *   dH = dY ⊙ GeLU′(H),  GeLU′(x) = Φ(x) + x·φ(x),  φ(x) = exp(−x²/2)/√(2π)
 *   da = 1ᵀ·dH,  dA = Xᵀ·dH,  dX = dH·Aᵀ
 *
 * The activation is "gelu" (page "Megatron", section "实战使用 / 基础训练示例",
 * the TransformerConfig of the training script); the pages give no formula,
 * and the exact-erf form is the plain reading. The biases a (length F, split
 * with A's columns) and b (length h, added once after the shard sum) are not
 * on the pages' equations; they follow the block Z = GeLU(X·A + a)·B + b.
 *
 * Every matrix is row-major. Every sum runs over its index in ascending
 * order in double precision; the only parallelism is over independent output
 * rows (OpenMP), which does not change any sum's order.
 *
 * The tpo_*_sharded functions follow the pages' partition literally
 * (per-shard products concatenated or summed over i = 1..p) and exist so the
 * tests can check the pages' two identities against the unsplit functions.
 *
 * Each path function has an _act form whose last argument selects the
 * activation: 0 = the exact GeLU above, 1 = the tanh approximation
 * (tpo_gelu_tanh). The form without the suffix is act = 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TPO_SQRT1_2 0.70710678118654752440 /* 1/√2 */
#define TPO_INV_SQRT_2PI 0.39894228040143267794 /* 1/√(2π) */

void tpo_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int tpo_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Φ(x), the standard normal distribution function, via the C library erf. */
double tpo_normal_cdf(double x) { return 0.5 * (1.0 + erf(x * TPO_SQRT1_2)); }

/* φ(x), the standard normal density. */
double tpo_normal_pdf(double x) { return TPO_INV_SQRT_2PI * exp(-0.5 * x * x); }

/* GeLU(x) = x·Φ(x). */
double tpo_gelu(double x) { return x * tpo_normal_cdf(x); }

/* d/dx [x·Φ(x)] = Φ(x) + x·φ(x). */
double tpo_gelu_grad(double x) { return tpo_normal_cdf(x) + x * tpo_normal_pdf(x); }

/* The tanh approximation of GeLU (Hendrycks & Gimpel, "Gaussian Error Linear
 * Units", 2016): ½·x·(1 + tanh(u)), u = √(2/π)·(x + 0.044715·x³). Offered as
 * a variant; the exact form above is the reading of the pages' "gelu". */
#define TPO_SQRT_2_OVER_PI 0.79788456080286535588 /* √(2/π) */
#define TPO_GELU_TANH_C 0.044715

double tpo_gelu_tanh(double x) {
    const double u = TPO_SQRT_2_OVER_PI * (x + TPO_GELU_TANH_C * x * x * x);
    return 0.5 * x * (1.0 + tanh(u));
}

/* d/dx of the tanh form: ½(1 + tanh u) + ½·x·(1 − tanh² u)·du/dx,
 * du/dx = √(2/π)·(1 + 3·0.044715·x²). */
double tpo_gelu_tanh_grad(double x) {
    const double u = TPO_SQRT_2_OVER_PI * (x + TPO_GELU_TANH_C * x * x * x);
    const double th = tanh(u);
    const double du = TPO_SQRT_2_OVER_PI * (1.0 + 3.0 * TPO_GELU_TANH_C * x * x);
    return 0.5 * (1.0 + th) + 0.5 * x * (1.0 - th * th) * du;
}

/* Activation selector: 0 = exact GeLU, 1 = tanh approximation. */
static double tpo_act(int act, double x) { return act ? tpo_gelu_tanh(x) : tpo_gelu(x); }
static double tpo_act_grad(int act, double x) {
    return act ? tpo_gelu_tanh_grad(x) : tpo_gelu_grad(x);
}

/* C[m, n] (+)= Σ_k P[m, k]·Q[k, n] for P (M × K), Q (K × N), row-major.
 * The k loop is the middle loop so each C row is updated with Q's rows in
 * ascending k: every C[m, n] is still the sum over k in ascending order. */
static void mm_nn(int64_t M, int64_t N, int64_t K, const double* P, const double* Q,
                  double* C, int accumulate) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double* c = C + m * N;
        if (!accumulate) memset(c, 0, (size_t)N * sizeof(double));
        for (int64_t k = 0; k < K; ++k) {
            const double pk = P[m * K + k];
            const double* q = Q + k * N;
            for (int64_t n = 0; n < N; ++n) c[n] += pk * q[n];
        }
    }
}

/* C[m, n] = Σ_k P[m, k]·Q[n, k]: a product with the second operand transposed
 * (P: M × K, Q: N × K), each entry a dot product in ascending k. */
static void mm_nt(int64_t M, int64_t N, int64_t K, const double* P, const double* Q,
                  double* C) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const double* p = P + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const double* q = Q + n * K;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += p[k] * q[k];
            C[m * N + n] = s;
        }
    }
}

/* C[m, n] = Σ_t P[t, m]·Q[t, n]: a product with the first operand transposed
 * (P: K × M, Q: K × N). Each thread owns rows m of C and walks t upward. */
static void mm_tn(int64_t M, int64_t N, int64_t K, const double* P, const double* Q,
                  double* C) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double* c = C + m * N;
        memset(c, 0, (size_t)N * sizeof(double));
        for (int64_t t = 0; t < K; ++t) {
            const double pt = P[t * M + m];
            const double* q = Q + t * N;
            for (int64_t n = 0; n < N; ++n) c[n] += pt * q[n];
        }
    }
}

/* out[n] = Σ_t Mat[t, n] over t ascending (a column sum, 1ᵀ·Mat). */
void tpo_colsum(int64_t T, int64_t N, const double* Mat, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t) s += Mat[t * N + n];
        out[n] = s;
    }
}

/* Forward of the unsplit block. */
void tpo_forward_act(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
                 const double* a, const double* B, const double* b, double* H, double* Y,
                 double* Z, int act) {
    mm_nn(T, F, h, X, A, H, 0);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t f = 0; f < F; ++f) {
            H[t * F + f] += a[f];
            Y[t * F + f] = tpo_act(act, H[t * F + f]);
        }
    mm_nn(T, h, F, Y, B, Z, 0);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < h; ++j) Z[t * h + j] += b[j];
}

void tpo_forward(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
                 const double* a, const double* B, const double* b, double* H, double* Y,
                 double* Z) {
    tpo_forward_act(T, h, F, X, A, a, B, b, H, Y, Z, 0);
}

/* Backward of the unsplit block, given the forward's H and Y. */
void tpo_backward_act(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
                  const double* B, const double* H, const double* Y, const double* dZ,
                  double* dH, double* dX, double* dA, double* da, double* dB,
                  double* db, int act) {
    tpo_colsum(T, h, dZ, db);
    mm_tn(F, h, T, Y, dZ, dB);
    mm_nt(T, F, h, dZ, B, dH); /* dH holds dY = dZ·Bᵀ here */
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t f = 0; f < F; ++f) dH[t * F + f] *= tpo_act_grad(act, H[t * F + f]);
    tpo_colsum(T, F, dH, da);
    mm_tn(h, F, T, X, dH, dA);
    mm_nt(T, h, F, dH, A, dX);
}

void tpo_backward(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
                  const double* B, const double* H, const double* Y, const double* dZ,
                  double* dH, double* dX, double* dA, double* da, double* dB,
                  double* db) {
    tpo_backward_act(T, h, F, X, A, B, H, Y, dZ, dH, dX, dA, da, dB, db, 0);
}

/* Copy the column block [c0, c0 + nc) of a row-major R × C matrix. */
static double* col_block(int64_t R, int64_t C, const double* M, int64_t c0, int64_t nc) {
    double* out = (double*)malloc((size_t)(R * nc) * sizeof(double));
    for (int64_t r = 0; r < R; ++r) memcpy(out + r * nc, M + r * C + c0, (size_t)nc * sizeof(double));
    return out;
}

/* Forward through the pages' partition. Shard i holds A_i = A[:, i·Fp:(i+1)·Fp],
 * a_i and B_i = B[i·Fp:(i+1)·Fp, :]. Column-parallel: H_i = X·A_i + a_i and
 * Y_i = GeLU(H_i), written side by side into H and Y. Row-parallel: the p
 * partial products P_i = Y_i·B_i are formed separately and summed over
 * i = 1..p in order (the all-reduce), then b is added once. Returns 0, or -1
 * if p does not divide F. */
int tpo_forward_sharded_act(int64_t T, int64_t h, int64_t F, int p, const double* X,
                        const double* A, const double* a, const double* B, const double* b,
                        double* H, double* Y, double* Z, int act) {
    if (p < 1 || F % p != 0) return -1;
    const int64_t Fp = F / p;
    double* Hi = (double*)malloc((size_t)(T * Fp) * sizeof(double));
    double* Pi = (double*)malloc((size_t)(T * h) * sizeof(double));
    memset(Z, 0, (size_t)(T * h) * sizeof(double));
    for (int i = 0; i < p; ++i) {
        double* Ai = col_block(h, F, A, i * Fp, Fp);
        double* Yi = (double*)malloc((size_t)(T * Fp) * sizeof(double));
        mm_nn(T, Fp, h, X, Ai, Hi, 0);
        for (int64_t t = 0; t < T; ++t)
            for (int64_t f = 0; f < Fp; ++f) {
                double v = Hi[t * Fp + f] + a[i * Fp + f];
                H[t * F + i * Fp + f] = v;
                Yi[t * Fp + f] = tpo_act(act, v);
                Y[t * F + i * Fp + f] = Yi[t * Fp + f];
            }
        mm_nn(T, h, Fp, Yi, B + (int64_t)i * Fp * h, Pi, 0);
        for (int64_t e = 0; e < T * h; ++e) Z[e] += Pi[e];
        free(Ai);
        free(Yi);
    }
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < h; ++j) Z[t * h + j] += b[j];
    free(Hi);
    free(Pi);
    return 0;
}

int tpo_forward_sharded(int64_t T, int64_t h, int64_t F, int p, const double* X,
                        const double* A, const double* a, const double* B, const double* b,
                        double* H, double* Y, double* Z) {
    return tpo_forward_sharded_act(T, h, F, p, X, A, a, B, b, H, Y, Z, 0);
}

/* Backward through the partition. Per shard, with no exchange:
 * dY_i = dZ·B_iᵀ, dH_i = dY_i ⊙ GeLU′(H_i), dA_i = Xᵀ·dH_i, da_i = 1ᵀ·dH_i,
 * dB_i = Y_iᵀ·dZ. X is replicated, so its gradient is the sum over shards of
 * dH_i·A_iᵀ, taken in order i = 1..p. db = 1ᵀ·dZ. */
int tpo_backward_sharded_act(int64_t T, int64_t h, int64_t F, int p, const double* X,
                         const double* A, const double* B, const double* H, const double* Y,
                         const double* dZ, double* dH, double* dX, double* dA, double* da,
                         double* dB, double* db, int act) {
    if (p < 1 || F % p != 0) return -1;
    const int64_t Fp = F / p;
    double* Pi = (double*)malloc((size_t)(T * h) * sizeof(double));
    memset(dX, 0, (size_t)(T * h) * sizeof(double));
    tpo_colsum(T, h, dZ, db);
    for (int i = 0; i < p; ++i) {
        double* Ai = col_block(h, F, A, i * Fp, Fp);
        double* Hi = col_block(T, F, H, i * Fp, Fp);
        double* Yi = col_block(T, F, Y, i * Fp, Fp);
        const double* Bi = B + (int64_t)i * Fp * h;
        double* dHi = (double*)malloc((size_t)(T * Fp) * sizeof(double));
        double* dAi = (double*)malloc((size_t)(h * Fp) * sizeof(double));
        mm_nt(T, Fp, h, dZ, Bi, dHi);
        for (int64_t e = 0; e < T * Fp; ++e) dHi[e] *= tpo_act_grad(act, Hi[e]);
        mm_tn(h, Fp, T, X, dHi, dAi);
        mm_tn(Fp, h, T, Yi, dZ, dB + (int64_t)i * Fp * h);
        tpo_colsum(T, Fp, dHi, da + i * Fp);
        mm_nt(T, h, Fp, dHi, Ai, Pi);
        for (int64_t e = 0; e < T * h; ++e) dX[e] += Pi[e];
        for (int64_t t = 0; t < T; ++t)
            memcpy(dH + t * F + i * Fp, dHi + t * Fp, (size_t)Fp * sizeof(double));
        for (int64_t k = 0; k < h; ++k)
            memcpy(dA + k * F + i * Fp, dAi + k * Fp, (size_t)Fp * sizeof(double));
        free(Ai);
        free(Hi);
        free(Yi);
        free(dHi);
        free(dAi);
    }
    free(Pi);
    return 0;
}

int tpo_backward_sharded(int64_t T, int64_t h, int64_t F, int p, const double* X,
                         const double* A, const double* B, const double* H, const double* Y,
                         const double* dZ, double* dH, double* dX, double* dA, double* da,
                         double* dB, double* db) {
    return tpo_backward_sharded_act(T, h, F, p, X, A, B, H, Y, dZ, dH, dX, dA, da, dB, db, 0);
}

/* The forward and backward restricted to the token rows R (nR of them).
 * Outputs are nR-row matrices: H_R, Y_R, dH_R (nR × F) and Z_R, dX_R (nR × h).
 * Each needs only its own rows: H[r, :] = X[r, :]·A + a, Z[r, :] = Y[r, :]·B + b,
 * dH[r, :] = (dZ[r, :]·Bᵀ) ⊙ GeLU′(H[r, :]), dX[r, :] = dH[r, :]·Aᵀ. */
void tpo_rows_act(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
              const double* a, const double* B, const double* b, const double* dZ,
              int64_t nR, const int64_t* R, double* H_R, double* Y_R, double* Z_R,
              double* dH_R, double* dX_R, int act) {
    (void)T;
    double* XR = (double*)malloc((size_t)(nR * h) * sizeof(double));
    double* dZR = (double*)malloc((size_t)(nR * h) * sizeof(double));
    for (int64_t r = 0; r < nR; ++r) {
        memcpy(XR + r * h, X + R[r] * h, (size_t)h * sizeof(double));
        memcpy(dZR + r * h, dZ + R[r] * h, (size_t)h * sizeof(double));
    }
    mm_nn(nR, F, h, XR, A, H_R, 0);
    for (int64_t r = 0; r < nR; ++r)
        for (int64_t f = 0; f < F; ++f) {
            H_R[r * F + f] += a[f];
            Y_R[r * F + f] = tpo_act(act, H_R[r * F + f]);
        }
    mm_nn(nR, h, F, Y_R, B, Z_R, 0);
    for (int64_t r = 0; r < nR; ++r)
        for (int64_t j = 0; j < h; ++j) Z_R[r * h + j] += b[j];
    mm_nt(nR, F, h, dZR, B, dH_R);
    for (int64_t e = 0; e < nR * F; ++e) dH_R[e] *= tpo_act_grad(act, H_R[e]);
    mm_nt(nR, h, F, dH_R, A, dX_R);
    free(XR);
    free(dZR);
}

void tpo_rows(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
              const double* a, const double* B, const double* b, const double* dZ,
              int64_t nR, const int64_t* R, double* H_R, double* Y_R, double* Z_R,
              double* dH_R, double* dX_R) {
    tpo_rows_act(T, h, F, X, A, a, B, b, dZ, nR, R, H_R, Y_R, Z_R, dH_R, dX_R, 0);
}

/* The forward and backward restricted to the hidden columns J of F (nJ of
 * them). Outputs: H_J, Y_J, dH_J (T × nJ), dA_J (h × nJ), da_J (nJ),
 * dB_J (nJ × h). Column f needs only A[:, f], a[f] and B[f, :]:
 * H[:, f] = X·A[:, f] + a[f], dY[:, f] = dZ·B[f, :]ᵀ, dH[:, f] = dY[:, f] ⊙
 * GeLU′(H[:, f]), dA[:, f] = Xᵀ·dH[:, f], da[f] = 1ᵀ·dH[:, f],
 * dB[f, :] = Y[:, f]ᵀ·dZ. */
void tpo_cols_act(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
              const double* a, const double* B, const double* dZ, int64_t nJ,
              const int64_t* J, double* H_J, double* Y_J, double* dH_J, double* dA_J,
              double* da_J, double* dB_J, int act) {
    double* AJ = (double*)malloc((size_t)(h * nJ) * sizeof(double)); /* h × nJ */
    double* BJ = (double*)malloc((size_t)(nJ * h) * sizeof(double)); /* nJ × h */
    for (int64_t k = 0; k < h; ++k)
        for (int64_t c = 0; c < nJ; ++c) AJ[k * nJ + c] = A[k * F + J[c]];
    for (int64_t c = 0; c < nJ; ++c) memcpy(BJ + c * h, B + J[c] * h, (size_t)h * sizeof(double));
    mm_nn(T, nJ, h, X, AJ, H_J, 0);
    for (int64_t t = 0; t < T; ++t)
        for (int64_t c = 0; c < nJ; ++c) {
            H_J[t * nJ + c] += a[J[c]];
            Y_J[t * nJ + c] = tpo_act(act, H_J[t * nJ + c]);
        }
    mm_nt(T, nJ, h, dZ, BJ, dH_J);
    for (int64_t e = 0; e < T * nJ; ++e) dH_J[e] *= tpo_act_grad(act, H_J[e]);
    mm_tn(h, nJ, T, X, dH_J, dA_J);
    tpo_colsum(T, nJ, dH_J, da_J);
    mm_tn(nJ, h, T, Y_J, dZ, dB_J);
    free(AJ);
    free(BJ);
}

void tpo_cols(int64_t T, int64_t h, int64_t F, const double* X, const double* A,
              const double* a, const double* B, const double* dZ, int64_t nJ,
              const int64_t* J, double* H_J, double* Y_J, double* dH_J, double* dA_J,
              double* da_J, double* dB_J) {
    tpo_cols_act(T, h, F, X, A, a, B, dZ, nJ, J, H_J, Y_J, dH_J, dA_J, da_J, dB_J, 0);
}

/* ---------------------------------------------------------------------------
 * Tensor-parallel linear layers (page "Megatron", section "张量并行 / 数学原理"
 * for the two splits, section "Transformer层的张量并行实现" for their use in the
 * attention layer: the QKV projection is split by columns, the output
 * projection by rows). Unsplit, both compute
 *
 *   Y = X·W + 1·biasᵀ      X: T × K, W: K × N, Y: T × N
 *   dbias = 1ᵀ·dY,  dW = Xᵀ·dY,  dX = dY·Wᵀ
 *
 * The _sharded forms follow the partition literally. Column split: shard i
 * holds W_i = W[:, i·N/p : (i+1)·N/p] and bias_i; Y_i = X·W_i + bias_i side
 * by side (no exchange); backward dW_i = Xᵀ·dY_i, dbias_i = 1ᵀ·dY_i and, X
 * being replicated, dX = Σ_i dY_i·W_iᵀ over i = 1..p in order. Row split:
 * shard i holds W_i = W[i·K/p : (i+1)·K/p, :] and the matching columns X_i
 * of X; Y = Σ_i X_i·W_i (in order) + bias; backward dX_i = dY·W_iᵀ (no
 * exchange), dW_i = X_iᵀ·dY, dbias = 1ᵀ·dY.
 * ------------------------------------------------------------------------- */

void tpo_linear_forward(int64_t T, int64_t K, int64_t N, const double* X, const double* W,
                        const double* bias, double* Y) {
    mm_nn(T, N, K, X, W, Y, 0);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) Y[t * N + n] += bias[n];
}

void tpo_linear_backward(int64_t T, int64_t K, int64_t N, const double* X, const double* W,
                         const double* dY, double* dX, double* dW, double* dbias) {
    tpo_colsum(T, N, dY, dbias);
    mm_tn(K, N, T, X, dY, dW);
    mm_nt(T, K, N, dY, W, dX);
}

/* split: 0 = columns, 1 = rows. Returns -1 if p does not divide the split
 * dimension (N for columns, K for rows). */
int tpo_linear_forward_sharded(int64_t T, int64_t K, int64_t N, int p, int split, const double* X,
                               const double* W, const double* bias, double* Y) {
    if (p < 1) return -1;
    if (split == 0) {
        if (N % p != 0) return -1;
        const int64_t Np = N / p;
        double* Yi = (double*)malloc((size_t)(T * Np) * sizeof(double));
        for (int i = 0; i < p; ++i) {
            double* Wi = col_block(K, N, W, i * Np, Np);
            mm_nn(T, Np, K, X, Wi, Yi, 0);
            for (int64_t t = 0; t < T; ++t)
                for (int64_t n = 0; n < Np; ++n) Y[t * N + i * Np + n] = Yi[t * Np + n] + bias[i * Np + n];
            free(Wi);
        }
        free(Yi);
        return 0;
    }
    if (K % p != 0) return -1;
    const int64_t Kp = K / p;
    double* Pi = (double*)malloc((size_t)(T * N) * sizeof(double));
    memset(Y, 0, (size_t)(T * N) * sizeof(double));
    for (int i = 0; i < p; ++i) {
        double* Xi = col_block(T, K, X, i * Kp, Kp);
        mm_nn(T, N, Kp, Xi, W + (int64_t)i * Kp * N, Pi, 0);
        for (int64_t e = 0; e < T * N; ++e) Y[e] += Pi[e];
        free(Xi);
    }
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) Y[t * N + n] += bias[n];
    free(Pi);
    return 0;
}

int tpo_linear_backward_sharded(int64_t T, int64_t K, int64_t N, int p, int split, const double* X,
                                const double* W, const double* dY, double* dX, double* dW,
                                double* dbias) {
    if (p < 1) return -1;
    tpo_colsum(T, N, dY, dbias);
    if (split == 0) {
        if (N % p != 0) return -1;
        const int64_t Np = N / p;
        double* Pi = (double*)malloc((size_t)(T * K) * sizeof(double));
        double* dWi = (double*)malloc((size_t)(K * Np) * sizeof(double));
        memset(dX, 0, (size_t)(T * K) * sizeof(double));
        for (int i = 0; i < p; ++i) {
            double* Wi = col_block(K, N, W, i * Np, Np);
            double* dYi = col_block(T, N, dY, i * Np, Np);
            mm_tn(K, Np, T, X, dYi, dWi);
            for (int64_t k = 0; k < K; ++k)
                memcpy(dW + k * N + i * Np, dWi + k * Np, (size_t)Np * sizeof(double));
            mm_nt(T, K, Np, dYi, Wi, Pi);
            for (int64_t e = 0; e < T * K; ++e) dX[e] += Pi[e];
            free(Wi);
            free(dYi);
        }
        free(Pi);
        free(dWi);
        return 0;
    }
    if (K % p != 0) return -1;
    const int64_t Kp = K / p;
    double* dXi = (double*)malloc((size_t)(T * Kp) * sizeof(double));
    for (int i = 0; i < p; ++i) {
        const double* Wi = W + (int64_t)i * Kp * N;
        double* Xi = col_block(T, K, X, i * Kp, Kp);
        mm_nt(T, Kp, N, dY, Wi, dXi);
        for (int64_t t = 0; t < T; ++t)
            memcpy(dX + t * K + i * Kp, dXi + t * Kp, (size_t)Kp * sizeof(double));
        mm_tn(Kp, N, T, Xi, dY, dW + (int64_t)i * Kp * N);
        free(Xi);
    }
    free(dXi);
    return 0;
}
