/*
 * lora_oracle_c.c — the LoRA-adapted linear layer, forward and backward, as
 * plain fp64 loops on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py load this library (through
 * oracle/lora_oracle_c.py).  It shares no code with the CUDA library and
 * includes none of its headers.
 *
 * What it computes (cited by page title and section):
 *  - "Liger-Kernel内核级优化：GPU利用率飙升至90%以上", section
 *    "为什么传统微调会“卡脖子”？": y = Wx + B(Ax), evaluated as the four calls
 *    ax = linear(x, A); bax = linear(ax, B); wx = linear(x, W); y = wx + bax.
 *    The branch is scaled by s = alpha / r (the pages give alpha and r only in
 *    configurations; the scale is the reading taken).
 *  - same page, section "内核融合：把“碎片化”变成“流水线”": the activation comes
 *    after the add (SiLU).
 *  - "Swift-All一文详解：如何用Liger-Kernel提升训练效率", 2.2 (2): SwiGLU,
 *    Y = SiLU(Z_gate) * Z_up, each of gate and up a LoRA linear with its own
 *    W, A, B.
 *  - the backward is the chain rule of that forward (the pages print no
 *    formula; "系统架构与工作流程" says only that it is fused, with
 *    recompute):  dZ = dY * act'(Z);  U = dZ B;  dX = dZ W + s U A;
 *    dA = s U^T X;  dB = s dZ^T T  with T = X A^T.
 *
 * Every number is an IEEE double; no product is blocked, fused or reordered
 * beyond the formulas.  Sums run in index order.  The only concession to
 * size is that independent output rows are shared out among POSIX threads.
 * sigma(z) = 1 / (1 + exp(-z)) with libm's exp.
 *
 * Build: gcc -O2 -fPIC -shared -pthread (oracle/build_oracle.py); no
 * -ffast-math, so the compiler keeps every operation as written.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ACT_IDENTITY = 0, ACT_SILU = 1, ACT_SWIGLU = 2 };

/* ------------------------------------------------------------------------ */
/* rows of an output shared out among threads                               */
/* ------------------------------------------------------------------------ */
typedef void (*row_fn)(void* ctx, int64_t row_begin, int64_t row_end);

typedef struct {
  row_fn fn;
  void* ctx;
  int64_t begin, end;
} job_t;

static void* run_job(void* p) {
  job_t* j = (job_t*)p;
  j->fn(j->ctx, j->begin, j->end);
  return NULL;
}

int oracle_threads(void) {
  const char* e = getenv("ORACLE_THREADS");
  long n = e ? strtol(e, NULL, 10) : sysconf(_SC_NPROCESSORS_ONLN);
  if (n < 1) n = 1;
  if (n > 256) n = 256;
  return (int)n;
}

static void par_rows(int64_t rows, row_fn fn, void* ctx) {
  int nt = oracle_threads();
  if (rows < 64 || nt == 1) {
    fn(ctx, 0, rows);
    return;
  }
  if (nt > rows) nt = (int)rows;
  pthread_t th[256];
  job_t jobs[256];
  int started = 0;
  for (int t = 0; t < nt; ++t) {
    jobs[t].fn = fn;
    jobs[t].ctx = ctx;
    jobs[t].begin = rows * t / nt;
    jobs[t].end = rows * (t + 1) / nt;
  }
  for (int t = 1; t < nt; ++t) {
    if (pthread_create(&th[t], NULL, run_job, &jobs[t]) != 0) break;
    started = t;
  }
  fn(ctx, jobs[0].begin, jobs[0].end);
  for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
  /* rows of threads that could not be started run here */
  for (int t = started + 1; t < nt; ++t) fn(ctx, jobs[t].begin, jobs[t].end);
}

/* ------------------------------------------------------------------------ */
/* the three products the layer uses                                        */
/* ------------------------------------------------------------------------ */
typedef struct {
  const double *a, *b;
  double* c;
  int64_t M, K, N;
} prod_t;

/* linear(x, w) without bias: C[m][n] = sum_k A[m][k] B[n][k]   (A M x K, B N x K) */
static void linear_rows(void* p, int64_t m0, int64_t m1) {
  const prod_t* q = (const prod_t*)p;
  for (int64_t m = m0; m < m1; ++m)
    for (int64_t n = 0; n < q->N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < q->K; ++k) acc += q->a[m * q->K + k] * q->b[n * q->K + k];
      q->c[m * q->N + n] = acc;
    }
}

/* C = A B:  C[m][n] = sum_k A[m][k] B[k][n]   (A M x K, B K x N), i-k-j order */
static void matmul_rows(void* p, int64_t m0, int64_t m1) {
  const prod_t* q = (const prod_t*)p;
  for (int64_t m = m0; m < m1; ++m) {
    double* c = q->c + m * q->N;
    for (int64_t n = 0; n < q->N; ++n) c[n] = 0.0;
    for (int64_t k = 0; k < q->K; ++k) {
      const double a = q->a[m * q->K + k];
      const double* b = q->b + k * q->N;
      for (int64_t n = 0; n < q->N; ++n) c[n] += a * b[n];
    }
  }
}

/* C = A^T B:  C[m][n] = sum_k A[k][m] B[k][n]   (A K x M, B K x N) */
static void matmul_tn_rows(void* p, int64_t m0, int64_t m1) {
  const prod_t* q = (const prod_t*)p;
  for (int64_t m = m0; m < m1; ++m) {
    double* c = q->c + m * q->N;
    for (int64_t n = 0; n < q->N; ++n) c[n] = 0.0;
    for (int64_t k = 0; k < q->K; ++k) {
      const double a = q->a[k * q->M + m];
      const double* b = q->b + k * q->N;
      for (int64_t n = 0; n < q->N; ++n) c[n] += a * b[n];
    }
  }
}

static void linear(const double* X, const double* W, double* Y, int64_t M, int64_t K, int64_t N) {
  prod_t q = {X, W, Y, M, K, N};
  par_rows(M, linear_rows, &q);
}

static void matmul(const double* A, const double* B, double* C, int64_t M, int64_t K, int64_t N) {
  prod_t q = {A, B, C, M, K, N};
  par_rows(M, matmul_rows, &q);
}

static void matmul_tn(const double* A, const double* B, double* C, int64_t K, int64_t M, int64_t N) {
  prod_t q = {A, B, C, M, K, N};
  par_rows(M, matmul_tn_rows, &q);
}

/* ------------------------------------------------------------------------ */
/* activations                                                              */
/* ------------------------------------------------------------------------ */
static double sigma(double z) { return 1.0 / (1.0 + exp(-z)); }
static double silu(double z) { return z * sigma(z); }
/* d SiLU / dz = sigma(z) (1 + z (1 - sigma(z))) */
static double silu_grad(double z) {
  const double g = sigma(z);
  return g * (1.0 + z * (1.0 - g));
}

void oracle_sigmoid(const double* z, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = sigma(z[i]);
}
void oracle_silu(const double* z, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu(z[i]);
}
void oracle_silu_grad(const double* z, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = silu_grad(z[i]);
}

/* ------------------------------------------------------------------------ */
/* forward                                                                  */
/* ------------------------------------------------------------------------ */
/* One LoRA linear without activation, the four calls in order:
 *   T (= ax)  = linear(X, A)          M x r
 *   bax       = linear(T, B)          M x d_out
 *   wx        = linear(X, W)          M x d_out
 *   Z         = wx + s * bax */
static int branch_forward(int64_t M, int64_t d_in, int64_t d_out, int64_t r, double s, const double* X,
                          const double* W, const double* A, const double* B, double* T, double* Z) {
  double* bax = (double*)malloc(sizeof(double) * (size_t)(M * d_out > 0 ? M * d_out : 1));
  if (!bax) return -1;
  linear(X, A, T, M, d_in, r);
  linear(T, B, bax, M, r, d_out);
  linear(X, W, Z, M, d_in, d_out);
  for (int64_t i = 0; i < M * d_out; ++i) Z[i] = Z[i] + s * bax[i];
  free(bax);
  return 0;
}

/* Y = act(Z): identity, SiLU(Z), or SiLU(Z_gate) * Z_up.  T_up, Z_up: the up
 * projection's (SwiGLU only). */
int oracle_lora_forward(int64_t M, int64_t d_in, int64_t d_out, int64_t r, double s, int act, const double* X,
                        const double* W, const double* A, const double* B, const double* W_up, const double* A_up,
                        const double* B_up, double* T, double* Z, double* Y, double* T_up, double* Z_up) {
  if (act < ACT_IDENTITY || act > ACT_SWIGLU) return -2;
  if (branch_forward(M, d_in, d_out, r, s, X, W, A, B, T, Z)) return -1;
  if (act == ACT_SWIGLU && branch_forward(M, d_in, d_out, r, s, X, W_up, A_up, B_up, T_up, Z_up)) return -1;
  for (int64_t i = 0; i < M * d_out; ++i) {
    if (act == ACT_IDENTITY) Y[i] = Z[i];
    else if (act == ACT_SILU) Y[i] = silu(Z[i]);
    else Y[i] = silu(Z[i]) * Z_up[i];
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* backward                                                                 */
/* ------------------------------------------------------------------------ */
/* Gradients of Z = X W^T + s (X A^T) B^T with W frozen, for a given dZ:
 *   U  = dZ B             M x r
 *   dX = dZ W + s U A     M x d_in     (accumulated into dX when add != 0)
 *   dA = s U^T X          r x d_in
 *   dB = s dZ^T T         d_out x r */
static int branch_backward(int64_t M, int64_t d_in, int64_t d_out, int64_t r, double s, const double* dZ,
                           const double* X, const double* W, const double* A, const double* B, const double* T,
                           double* U, double* dX, double* dA, double* dB, int add) {
  const size_t n_x = (size_t)(M * d_in > 0 ? M * d_in : 1);
  double* dzw = (double*)malloc(sizeof(double) * n_x);
  double* ua = (double*)malloc(sizeof(double) * n_x);
  if (!dzw || !ua) {
    free(dzw);
    free(ua);
    return -1;
  }
  matmul(dZ, B, U, M, d_out, r);
  matmul(dZ, W, dzw, M, d_out, d_in);
  matmul(U, A, ua, M, r, d_in);
  for (int64_t i = 0; i < M * d_in; ++i) {
    const double g = dzw[i] + s * ua[i];
    dX[i] = add ? dX[i] + g : g;
  }
  matmul_tn(U, X, dA, M, r, d_in);
  matmul_tn(dZ, T, dB, M, d_out, r);
  for (int64_t i = 0; i < r * d_in; ++i) dA[i] = s * dA[i];
  for (int64_t i = 0; i < d_out * r; ++i) dB[i] = s * dB[i];
  free(dzw);
  free(ua);
  return 0;
}

/* The backward recomputes the forward into T, Z, Y (and, for SwiGLU, T_up,
 * Z_up), forms dZ = dY * act'(Z) (SwiGLU: dZ_gate = dY Z_up SiLU'(Z_gate),
 * dZ_up = dY SiLU(Z_gate)) and applies the branch gradients; SwiGLU's dX is
 * the sum of both projections' input gradients. */
int oracle_lora_backward(int64_t M, int64_t d_in, int64_t d_out, int64_t r, double s, int act, const double* dY,
                         const double* X, const double* W, const double* A, const double* B, const double* W_up,
                         const double* A_up, const double* B_up, double* T, double* Z, double* Y, double* T_up,
                         double* Z_up, double* dZ, double* dZ_up, double* U, double* U_up, double* dX, double* dA,
                         double* dB, double* dA_up, double* dB_up) {
  if (act < ACT_IDENTITY || act > ACT_SWIGLU) return -2;
  const int sw = act == ACT_SWIGLU;
  if (oracle_lora_forward(M, d_in, d_out, r, s, act, X, W, A, B, W_up, A_up, B_up, T, Z, Y, T_up, Z_up)) return -1;
  for (int64_t i = 0; i < M * d_out; ++i) {
    if (act == ACT_IDENTITY) dZ[i] = dY[i];
    else if (act == ACT_SILU) dZ[i] = dY[i] * silu_grad(Z[i]);
    else {
      dZ[i] = dY[i] * Z_up[i] * silu_grad(Z[i]);
      dZ_up[i] = dY[i] * silu(Z[i]);
    }
  }
  if (branch_backward(M, d_in, d_out, r, s, dZ, X, W, A, B, T, U, dX, dA, dB, 0)) return -1;
  if (sw && branch_backward(M, d_in, d_out, r, s, dZ_up, X, W_up, A_up, B_up, T_up, U_up, dX, dA_up, dB_up, 1))
    return -1;
  return 0;
}

/* Adapter gradients of the identity layer without touching W (cheap at any
 * size): T = X A^T, U = dY B, dA = s U^T X, dB = s dY^T T. */
int oracle_adapter_grads_identity(int64_t M, int64_t d_in, int64_t d_out, int64_t r, double s, const double* dY,
                                  const double* X, const double* A, const double* B, double* T, double* U,
                                  double* dA, double* dB) {
  linear(X, A, T, M, d_in, r);
  matmul(dY, B, U, M, d_out, r);
  matmul_tn(U, X, dA, M, r, d_in);
  matmul_tn(dY, T, dB, M, d_out, r);
  for (int64_t i = 0; i < r * d_in; ++i) dA[i] = s * dA[i];
  for (int64_t i = 0; i < d_out * r; ++i) dB[i] = s * dB[i];
  return 0;
}

/* Exact value of bf16 bit patterns: the 16 bits are the upper half of an
 * IEEE binary32 whose lower half is zero. */
void oracle_bf16_to_f64(const uint16_t* bits, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    const uint32_t u = (uint32_t)bits[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    out[i] = (double)f;
  }
}
