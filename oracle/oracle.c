/*
 * Packed LoRA forward/backward oracle: plain fp64 loops on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the definition the CUDA path is
 * checked against.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load it; the library never calls it, and it shares no
 * code, header or constant with the library.
 *
 * What it computes (one frozen base projection shared by N adapters, adapter
 * i owning the contiguous token rows [off[i], off[i+1]) of the packed buffer):
 *
 *   Y_i  = X_i W + s_i (X_i A_i) B_i                 (forward)
 *   dX_i = dY_i W^T + s_i (dY_i B_i^T) A_i^T         (input gradient)
 *   dB_i = s_i (X_i A_i)^T dY_i                      (reduces over the tokens)
 *   dA_i = X_i^T (s_i dY_i B_i^T)                    (reduces over the tokens)
 *
 * Sources:
 *  - LoRA layer: frozen W plus a trainable low-rank branch A (d -> r) then
 *    B (r -> d), outputs added, branch scaled by alpha/r, A Gaussian-init and
 *    B zero-init: "LLM+LoRA微调加速技术原理解析" (m.youleyou.com),
 *    section 深入理解LoRA：基本原理与PEFT实现.
 *  - Only A and B receive gradients, through the chain rule; W stays frozen:
 *    "LoRA加速集成方案" (cloud.baidu.com), 四、工作原理 › 3. 反向传播阶段.
 *  - Many adapters packed over one shared frozen base, operators batching the
 *    adapters over the concatenated LoRA tensors, covering the forward and the
 *    backward gradient cases: PLoRA summary (gist.science, arXiv 2508.02932),
 *    技术摘要 › 方法论 › 2. LoRA 执行引擎 › 打包 LoRA 算子 / 算子设计.
 *
 * Storage is row-major in the PyTorch/PEFT module layouts:
 *   X[T][d_in], W_store[d_out][d_in] (= W^T), A_store_i[r_i][d_in] (= A_i^T),
 *   B_store_i[d_out][r_i] (= B_i^T), dY[T][d_out]; dA_i, dB_i are stored like
 *   A_store_i, B_store_i.  Inputs are bf16 bit patterns (dtype 0) or fp32
 *   (dtype 1), widened exactly to double; every sum is accumulated in double
 *   in index order.  No blocking, no fusion, no reordering.
 *
 * Parallelism (nthreads > 1) only splits independent output elements across
 * OpenMP threads; the arithmetic of each element is unchanged.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BF16 0
#define ORACLE_FP32 1

static double ld(const void* base, int dtype, int64_t idx) {
    if (dtype == ORACLE_BF16) {
        uint32_t u = ((uint32_t)((const uint16_t*)base)[idx]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float*)base)[idx];
}

static int adapter_of_row(int32_t n, const int64_t* off, int64_t t) {
    for (int32_t i = 0; i < n; ++i)
        if (t >= off[i] && t < off[i + 1]) return i;
    return -1;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    omp_set_num_threads(nthreads > 0 ? nthreads : 1);
#else
    (void)nthreads;
#endif
}

int oracle_num_procs(void) {
#ifdef _OPENMP
    return omp_get_num_procs();
#else
    return 1;
#endif
}

/* H[t][k] = sum_j X[t][j] * A_i[j][k], with A_i[j][k] = A_store_i[k][j]. */
static double h_elem(int dtype, int64_t d_in, const void* X, const void* Ai, int64_t t, int k) {
    double acc = 0.0;
    for (int64_t j = 0; j < d_in; ++j)
        acc += ld(X, dtype, t * d_in + j) * ld(Ai, dtype, (int64_t)k * d_in + j);
    return acc;
}

/* G[t][k] = s_i * sum_c dY[t][c] * B_i[k][c], with B_i[k][c] = B_store_i[c][k]. */
static double g_elem(int dtype, int64_t d_out, int r, double s, const void* dY, const void* Bi,
                     int64_t t, int k) {
    double acc = 0.0;
    for (int64_t c = 0; c < d_out; ++c)
        acc += ld(dY, dtype, t * d_out + c) * ld(Bi, dtype, c * r + k);
    return s * acc;
}

/*
 * Forward.  For each requested row t (all T rows if rows == NULL):
 *   Y[t][c] = sum_j X[t][j] W[j][c] + s_i sum_k H[t][k] B_i[k][c]
 * Y_out is [n_rows][d_out] (n_rows = T when rows == NULL).
 * H_out, if not NULL, receives H[t][k] for k < r_i in a [n_rows][h_ld] array
 * (unused columns are left as they are).
 * Returns 0, or -1 if a requested row lies outside every segment.
 */
int oracle_forward(int dtype, int64_t d_in, int64_t d_out, int32_t n, const int64_t* off,
                   const int32_t* rank, const float* scale, const void* X, const void* W,
                   const void* const* A, const void* const* B, int64_t n_rows, const int64_t* rows,
                   double* Y_out, double* H_out, int64_t h_ld, int nthreads) {
    const int64_t T = off[n];
    const int64_t R = rows ? n_rows : T;
    for (int64_t q = 0; q < R; ++q)
        if (adapter_of_row(n, off, rows ? rows[q] : q) < 0) return -1;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < R; ++q) {
        const int64_t t = rows ? rows[q] : q;
        const int i = adapter_of_row(n, off, t);
        const int r = rank[i];
        const double s = (double)scale[i];
        double* H = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
        for (int k = 0; k < r; ++k) H[k] = h_elem(dtype, d_in, X, A[i], t, k);
        if (H_out)
            for (int k = 0; k < r; ++k) H_out[q * h_ld + k] = H[k];
        for (int64_t c = 0; c < d_out; ++c) {
            double base = 0.0;
            for (int64_t j = 0; j < d_in; ++j)
                base += ld(X, dtype, t * d_in + j) * ld(W, dtype, c * d_in + j);
            double lora = 0.0;
            for (int k = 0; k < r; ++k) lora += H[k] * ld(B[i], dtype, c * r + k);
            Y_out[q * d_out + c] = base + s * lora;
        }
        free(H);
    }
    return 0;
}

/*
 * Input gradient.  For each requested row t:
 *   dX[t][j] = sum_c dY[t][c] W[j][c] + sum_k G[t][k] A_i[j][k]
 * dX_out is [n_rows][d_in].  G_out, if not NULL, receives G[t][k] (k < r_i)
 * in a [n_rows][g_ld] array.
 */
int oracle_input_grad(int dtype, int64_t d_in, int64_t d_out, int32_t n, const int64_t* off,
                      const int32_t* rank, const float* scale, const void* W,
                      const void* const* A, const void* const* B, const void* dY,
                      int64_t n_rows, const int64_t* rows, double* dX_out, double* G_out,
                      int64_t g_ld, int nthreads) {
    const int64_t T = off[n];
    const int64_t R = rows ? n_rows : T;
    for (int64_t q = 0; q < R; ++q)
        if (adapter_of_row(n, off, rows ? rows[q] : q) < 0) return -1;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < R; ++q) {
        const int64_t t = rows ? rows[q] : q;
        const int i = adapter_of_row(n, off, t);
        const int r = rank[i];
        const double s = (double)scale[i];
        double* G = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
        for (int k = 0; k < r; ++k) G[k] = g_elem(dtype, d_out, r, s, dY, B[i], t, k);
        if (G_out)
            for (int k = 0; k < r; ++k) G_out[q * g_ld + k] = G[k];
        for (int64_t j = 0; j < d_in; ++j) {
            double base = 0.0;
            for (int64_t c = 0; c < d_out; ++c)
                base += ld(dY, dtype, t * d_out + c) * ld(W, dtype, c * d_in + j);
            double lora = 0.0;
            for (int k = 0; k < r; ++k) lora += G[k] * ld(A[i], dtype, (int64_t)k * d_in + j);
            dX_out[q * d_in + j] = base + lora;
        }
        free(G);
    }
    return 0;
}

/*
 * Weight gradients of every adapter, each a sum over that adapter's tokens:
 *   dB_i[k][c] = s_i sum_{t in seg i} H[t][k] dY[t][c]   stored dB_store_i[c][k]
 *   dA_i[j][k] =     sum_{t in seg i} X[t][j] G[t][k]    stored dA_store_i[k][j]
 * An adapter with no tokens gets zeros.  dA[i] is [r_i][d_in], dB[i] is
 * [d_out][r_i], both double.  If n_cols_a > 0, only the hidden columns
 * j = cols_a[0..n_cols_a) of dA are computed (the others are left as they
 * are); likewise cols_b for the rows c of dB.
 */
int oracle_weight_grads(int dtype, int64_t d_in, int64_t d_out, int32_t n, const int64_t* off,
                        const int32_t* rank, const float* scale, const void* X,
                        const void* const* A, const void* const* B, const void* dY,
                        double* const* dA, double* const* dB, int64_t n_cols_a,
                        const int64_t* cols_a, int64_t n_cols_b, const int64_t* cols_b,
                        int nthreads) {
    set_threads(nthreads);
    const int64_t na = n_cols_a > 0 ? n_cols_a : d_in;
    const int64_t nb = n_cols_b > 0 ? n_cols_b : d_out;
    for (int32_t i = 0; i < n; ++i) {
        const int64_t t0 = off[i], nt = off[i + 1] - off[i];
        const int r = rank[i];
        const double s = (double)scale[i];
        double* H = (double*)malloc(sizeof(double) * (size_t)(nt > 0 ? nt : 1) * (size_t)r);
        double* G = (double*)malloc(sizeof(double) * (size_t)(nt > 0 ? nt : 1) * (size_t)r);
#pragma omp parallel for schedule(static)
        for (int64_t u = 0; u < nt; ++u)
            for (int k = 0; k < r; ++k) {
                H[u * r + k] = h_elem(dtype, d_in, X, A[i], t0 + u, k);
                G[u * r + k] = g_elem(dtype, d_out, r, s, dY, B[i], t0 + u, k);
            }
#pragma omp parallel for schedule(static)
        for (int64_t q = 0; q < nb; ++q) {
            const int64_t c = n_cols_b > 0 ? cols_b[q] : q;
            for (int k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int64_t u = 0; u < nt; ++u) acc += H[u * r + k] * ld(dY, dtype, (t0 + u) * d_out + c);
                dB[i][c * r + k] = s * acc;
            }
        }
#pragma omp parallel for schedule(static)
        for (int64_t q = 0; q < na; ++q) {
            const int64_t j = n_cols_a > 0 ? cols_a[q] : q;
            for (int k = 0; k < r; ++k) {
                double acc = 0.0;
                for (int64_t u = 0; u < nt; ++u) acc += ld(X, dtype, (t0 + u) * d_in + j) * G[u * r + k];
                dA[i][(int64_t)k * d_in + j] = acc;
            }
        }
        free(H);
        free(G);
    }
    return 0;
}

/*
 * One AdamW step on n elements, in double (TEST INFRASTRUCTURE, like the rest of this file).
 * The LoRA fine-tuning loop on "LLM+LoRA微调加速技术原理解析" (m.youleyou.com, the PEFT example)
 * updates the adapters with torch.optim.AdamW; the pages print no formula, so this follows that
 * optimizer's documented algorithm (Adam with decoupled weight decay), in its order:
 *   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
 *   p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 */
void oracle_adamw(int64_t n, double* p, double* m, double* v, const double* g, double lr, double beta1,
                  double beta2, double eps, double weight_decay, int step) {
    const double bc1 = 1.0 - pow(beta1, (double)step);
    const double bc2 = 1.0 - pow(beta2, (double)step);
    for (int64_t e = 0; e < n; ++e) {
        p[e] = p[e] * (1.0 - lr * weight_decay);
        m[e] = beta1 * m[e] + (1.0 - beta1) * g[e];
        v[e] = beta2 * v[e] + (1.0 - beta2) * g[e] * g[e];
        const double denom = sqrt(v[e]) / sqrt(bc2) + eps;
        p[e] = p[e] - (lr / bc1) * m[e] / denom;
    }
}
