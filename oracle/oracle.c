/*
 * oracle.c -- plain fp64 CPU oracle for the fused linear-layer GEMM + epilogue.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library. The product path never does, and
 * this file shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (and where the pages define it):
 *
 *   C[i][j] = sum_{k=0}^{K-1} a(r_i, k) * b(k, c_j)  (+ bias[c_j] if given)
 *   S[i][j] = sum_{k=0}^{K-1} |a(r_i, k) * b(k, c_j)|  (+ |bias[c_j]| if given)
 *
 * for a chosen list of rows r_i of A (R x K, row-major) and columns c_j of
 * B (K x C, row-major). Every product and partial sum is carried in IEEE
 * binary64, and each output element is summed in ascending k: this is the
 * plain definition of the matrix product with a bias broadcast over rows.
 *
 *  - Forward Z = X.W + b: "nvmath-python epilog fusion guide", section on
 *    MatmulEpilog.BIAS (bias broadcast onto the product), and the fused
 *    kernel of "AI inference compiler operator fusion", section 3.1
 *    (sum over K, then bias[col] added to that column).
 *  - Backward G = dY2.W2 (the product that DRELU_BGRAD masks):
 *    "nvmath-python fused epilog (itzkxy)", section on DRELU_BGRAD.
 *  - S is the error scale of the acceptance bound |err| <= 2e-3 * S.
 *
 * The epilogue steps (ReLU, mask bits, mask application, column sums) are
 * done in oracle/__init__.py on the fp64 results of this file.
 *
 * Inputs are raw 16-bit patterns (IEEE binary16 or bfloat16), decoded here
 * from the published bit layouts, so the oracle reads exactly the bytes the
 * GPU receives.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
 * bits. Exponent 0 encodes zero and subnormals (f * 2^-24); exponent 31
 * encodes infinities (f == 0) and NaNs. */
double oracle_half_to_double(uint16_t h) {
  int s = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 25); /* (1 + f/2^10) * 2^(e-15) */
  return s ? -v : v;
}

/* bfloat16: the upper half of an IEEE 754 binary32: 1 sign bit, 8 exponent
 * bits (bias 127), 7 fraction bits. Exponent 0 encodes zero and subnormals
 * (f * 2^-133); exponent 255 encodes infinities and NaNs. */
double oracle_bf16_to_double(uint16_t h) {
  int s = (h >> 15) & 1;
  int e = (h >> 7) & 0xff;
  int f = h & 0x7f;
  double v;
  if (e == 0)
    v = ldexp((double)f, -133);
  else if (e == 255)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(128 + f), e - 134); /* (1 + f/2^7) * 2^(e-127) */
  return s ? -v : v;
}

static double decode(uint16_t h, int dtype) {
  return dtype == ORACLE_BF16 ? oracle_bf16_to_double(h) : oracle_half_to_double(h);
}

typedef struct {
  const uint16_t* A;     /* R x K */
  const double* Bsel;    /* K x nc: B restricted to the chosen columns, decoded */
  const double* bsel;    /* nc or NULL */
  int dtype;
  int64_t K;
  const int64_t* rows;   /* nr entries, or NULL for rows 0..nr-1 */
  int64_t nc;
  int64_t row_begin, row_end; /* this worker's slice of the row list */
  double* C;             /* nr x nc */
  double* S;             /* nr x nc */
} job_t;

#define ROWS_PER_PASS 8

/* Rows are taken ROWS_PER_PASS at a time so that each decoded row of B is
 * read once per pass instead of once per row; every output element is still
 * its own binary64 sum, taken over k in ascending order. */
static void* worker(void* p) {
  job_t* j = (job_t*)p;
  const int64_t nc = j->nc;
  for (int64_t i0 = j->row_begin; i0 < j->row_end; i0 += ROWS_PER_PASS) {
    const int nrow = (int)(j->row_end - i0 < ROWS_PER_PASS ? j->row_end - i0 : ROWS_PER_PASS);
    const uint16_t* arow[ROWS_PER_PASS];
    double* c[ROWS_PER_PASS];
    double* s[ROWS_PER_PASS];
    for (int r = 0; r < nrow; ++r) {
      const int64_t i = i0 + r;
      const int64_t row = j->rows ? j->rows[i] : i;
      arow[r] = j->A + row * j->K;
      c[r] = j->C + i * nc;
      s[r] = j->S + i * nc;
      for (int64_t q = 0; q < nc; ++q) {
        c[r][q] = 0.0;
        s[r][q] = 0.0;
      }
    }
    for (int64_t k = 0; k < j->K; ++k) {
      const double* brow = j->Bsel + k * nc;
      for (int r = 0; r < nrow; ++r) {
        const double a = decode(arow[r][k], j->dtype);
        double* cr = c[r];
        double* sr = s[r];
        for (int64_t q = 0; q < nc; ++q) {
          const double prod = a * brow[q];
          cr[q] += prod;
          sr[q] += fabs(prod);
        }
      }
    }
    if (j->bsel) {
      for (int r = 0; r < nrow; ++r) {
        for (int64_t q = 0; q < nc; ++q) {
          c[r][q] += j->bsel[q];
          s[r][q] += fabs(j->bsel[q]);
        }
      }
    }
  }
  return NULL;
}

/*
 * oracle_matmul_bias: C, S as defined in the header comment.
 *   A     R x K row-major 16-bit patterns      B    K x Cn row-major
 *   bias  Cn patterns, or NULL (no bias term)
 *   rows  nr row indices into A, or NULL meaning rows 0..nr-1
 *   cols  nc column indices into B, or NULL meaning columns 0..nc-1
 *   C, S  nr x nc doubles, written
 * Returns 0, or -1 on a bad argument or allocation failure.
 */
int oracle_matmul_bias(const uint16_t* A, const uint16_t* B, const uint16_t* bias, int dtype,
                       int64_t R, int64_t Cn, int64_t K, const int64_t* rows, int64_t nr,
                       const int64_t* cols, int64_t nc, double* C, double* S, int nthreads) {
  if (!A || !B || !C || !S || R < 0 || Cn < 0 || K < 0 || nr < 0 || nc < 0) return -1;
  if (dtype != ORACLE_F16 && dtype != ORACLE_BF16) return -1;
  if (!rows && nr > R) return -1;
  if (!cols && nc > Cn) return -1;
  for (int64_t i = 0; rows && i < nr; ++i)
    if (rows[i] < 0 || rows[i] >= R) return -1;
  for (int64_t q = 0; cols && q < nc; ++q)
    if (cols[q] < 0 || cols[q] >= Cn) return -1;
  if (nr == 0 || nc == 0) return 0;

  double* Bsel = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * (size_t)nc);
  double* bsel = bias ? (double*)malloc(sizeof(double) * (size_t)nc) : NULL;
  if (!Bsel || (bias && !bsel)) {
    free(Bsel);
    free(bsel);
    return -1;
  }
  for (int64_t k = 0; k < K; ++k)
    for (int64_t q = 0; q < nc; ++q)
      Bsel[k * nc + q] = decode(B[k * Cn + (cols ? cols[q] : q)], dtype);
  for (int64_t q = 0; bias && q < nc; ++q) bsel[q] = decode(bias[cols ? cols[q] : q], dtype);

  if (nthreads < 1) nthreads = 1;
  if (nthreads > nr) nthreads = (int)nr;
  if (nthreads > 256) nthreads = 256;
  pthread_t tid[256];
  int spawned[256];
  job_t jobs[256];
  for (int t = 0; t < nthreads; ++t) {
    jobs[t].A = A;
    jobs[t].Bsel = Bsel;
    jobs[t].bsel = bsel;
    jobs[t].dtype = dtype;
    jobs[t].K = K;
    jobs[t].rows = rows;
    jobs[t].nc = nc;
    jobs[t].row_begin = nr * t / nthreads;
    jobs[t].row_end = nr * (t + 1) / nthreads;
    jobs[t].C = C;
    jobs[t].S = S;
  }
  /* worker 0 runs on the calling thread; a worker whose thread cannot be
   * created also runs on the calling thread */
  for (int t = 1; t < nthreads; ++t) spawned[t] = pthread_create(&tid[t], NULL, worker, &jobs[t]) == 0;
  worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) {
    if (spawned[t])
      pthread_join(tid[t], NULL);
    else
      worker(&jobs[t]);
  }
  free(Bsel);
  free(bsel);
  return 0;
}
