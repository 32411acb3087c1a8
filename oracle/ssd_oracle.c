/*
 * ssd_oracle.c -- float64 CPU oracle for the SSD (Mamba-2) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code with the CUDA library.
 *
 * What it computes is the plain definition of the scalar-times-identity
 * selective SSM, run as a sequential recurrence one token at a time
 * ("Transformers are SSMs", paperlayer.ai summary: §2.4 scalar-times-identity
 * structure; §3.4.1 the linear (recurrent) mode; App. B.2.1 sequential
 * recurrence).  For every document d and head h, with group g = h / (H/G):
 *
 *     delta_t = softplus(dt[t,h] + dt_bias[h])
 *     S_t     = exp(delta_t * A[h]) * S_{t-1} + delta_t * B[t,g,:]^T x[t,h,:]   (N x P)
 *     y[t,h]  = C[t,g,:] . S_t + D[h] * x[t,h,:]
 *
 * S_{start-1} is the document's initial state (zero when none is given), so
 * no information crosses a document boundary (§8.3 Variable Length: the
 * transition multiplier is zero at a boundary).  The final state of the
 * document is S at its last token.  There is no chunking here: the chunked
 * block decomposition (§6) reaches the same numbers in exact arithmetic.
 *
 * All arithmetic is float64.  Parallel over (document, head) with OpenMP only;
 * the loop over t is sequential.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(z) = log(1 + exp(z)), written so that exp never overflows. */
static double oracle_softplus(double z) {
  if (z > 0.0) return z + log1p(exp(-z));
  return log1p(exp(z));
}

/*
 * ssd_oracle_forward
 *   ntokens        total tokens T (all documents packed back to back)
 *   nheads H, headdim P, dstate N, ngroups G  (H % G == 0)
 *   ndocs          number of documents
 *   doc_offsets    int64[ndocs+1], 0 = off[0] <= off[1] <= ... <= off[ndocs] = T
 *   x   [T,H,P]   dt [T,H]   A [H]   B,C [T,G,N]   D [H] or NULL   dt_bias [H] or NULL
 *   init [ndocs,H,N,P] or NULL (zero)
 *   heads          int32 list of heads to compute, or NULL for all heads
 *   nheads_sel     length of that list (ignored when heads == NULL)
 *   y    [T,H,P]   only the selected heads' entries are written
 *   final_states [ndocs,H,N,P] or NULL; only the selected heads are written
 *   nthreads       OpenMP threads (<= 0: library default)
 * Returns 0, or -1 on an inconsistent argument (nothing is written then).
 */
int ssd_oracle_forward(int64_t ntokens, int nheads, int headdim, int dstate, int ngroups,
                       int ndocs, const int64_t* doc_offsets,
                       const double* x, const double* dt, const double* A,
                       const double* B, const double* C, const double* D,
                       const double* dt_bias, const double* init,
                       const int32_t* heads, int nheads_sel,
                       double* y, double* final_states, int nthreads) {
  const int H = nheads, P = headdim, N = dstate, G = ngroups;
  if (H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0 || ndocs < 0) return -1;
  if (doc_offsets == NULL || doc_offsets[0] != 0 || doc_offsets[ndocs] != ntokens) return -1;
  for (int d = 0; d < ndocs; ++d)
    if (doc_offsets[d + 1] < doc_offsets[d]) return -1;
  const int nsel = heads ? nheads_sel : H;
  if (heads)
    for (int i = 0; i < nsel; ++i)
      if (heads[i] < 0 || heads[i] >= H) return -1;
  const int heads_per_group = H / G;
  const int64_t npairs = (int64_t)ndocs * nsel;

#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif

#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * (size_t)N * (size_t)P);
#pragma omp for schedule(dynamic, 1)
    for (int64_t pair = 0; pair < npairs; ++pair) {
      const int d = (int)(pair / nsel);
      const int h = heads ? heads[pair % nsel] : (int)(pair % nsel);
      const int g = h / heads_per_group;
      const double bias = dt_bias ? dt_bias[h] : 0.0;
      const double skip = D ? D[h] : 0.0;
      const size_t state_off = ((size_t)d * H + h) * (size_t)N * P;
      if (init)
        memcpy(S, init + state_off, sizeof(double) * (size_t)N * P);
      else
        memset(S, 0, sizeof(double) * (size_t)N * P);

      for (int64_t t = doc_offsets[d]; t < doc_offsets[d + 1]; ++t) {
        const double delta = oracle_softplus(dt[t * H + h] + bias);
        const double decay = exp(delta * A[h]);
        const double* xt = x + ((size_t)t * H + h) * P;
        const double* Bt = B + ((size_t)t * G + g) * N;
        const double* Ct = C + ((size_t)t * G + g) * N;
        double* yt = y + ((size_t)t * H + h) * P;
        /* state update: S <- decay * S + delta * B_t (outer) x_t */
        for (int n = 0; n < N; ++n) {
          const double coef = delta * Bt[n];
          double* row = S + (size_t)n * P;
          for (int p = 0; p < P; ++p) row[p] = decay * row[p] + coef * xt[p];
        }
        /* readout: y_t = C_t . S + D x_t */
        for (int p = 0; p < P; ++p) yt[p] = skip * xt[p];
        for (int n = 0; n < N; ++n) {
          const double c = Ct[n];
          const double* row = S + (size_t)n * P;
          for (int p = 0; p < P; ++p) yt[p] += c * row[p];
        }
      }
      if (final_states)
        memcpy(final_states + state_off, S, sizeof(double) * (size_t)N * P);
    }
    free(S);
  }
  return 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int ssd_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
