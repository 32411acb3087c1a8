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

/*
 * ssd_oracle_backward -- the gradient of the same recurrence, by the chain rule
 * taken backwards through the tokens (reverse-mode differentiation of the
 * definition above; the pages give only its cost, "Transformers are SSMs",
 * paperlayer.ai summary, §6 and §3.4.1).  The loss is
 *     sum_t <dy_t, y_t> + <dfinal, final_state>
 * for given cotangents dy [T,H,P] and dfinal [ndocs,H,N,P] (NULL: zero).  With
 * Gm the cotangent of the state S_t, walking t from the document's last token
 * down to its first:
 *
 *     Gm      += C_t^T dy_t                       (y_t reads S_t)
 *     dC_t    += S_t dy_t                         dD      += <dy_t, x_t>
 *     gB       = Gm^T B_t                         dx_t     = delta_t gB + D dy_t
 *     dB_t    += delta_t Gm x_t
 *     ddelta_t = <x_t, gB> + A exp(delta_t A) <Gm, S_{t-1}>
 *     dA      += delta_t exp(delta_t A) <Gm, S_{t-1}>
 *     ddt_t    = ddelta_t sigmoid(dt_t + dt_bias)   ddt_bias += ddt_t
 *     Gm       = exp(delta_t A) Gm                (cotangent of S_{t-1})
 *
 * and the cotangent of the initial state is Gm after the first token.  The
 * states S_t of one (document, head) are kept from a forward sweep.  dB and dC
 * sum over the heads of a group; dA, dD and ddt_bias come out per (document,
 * head) in dA_part, dD_part, dbias_part [ndocs, H] (the caller sums over
 * documents).  With a head list, only those heads are differentiated (their
 * share of dB and dC; the other heads' entries of per-head outputs are left
 * untouched).  dB and dC must be zero on entry.  Parallel over (document,
 * group); the heads of a group run one after another.  Returns 0, or -1 on an
 * inconsistent argument, or -2 when memory runs out.
 */
int ssd_oracle_backward(int64_t ntokens, int nheads, int headdim, int dstate, int ngroups,
                        int ndocs, const int64_t* doc_offsets,
                        const double* x, const double* dt, const double* A,
                        const double* B, const double* C, const double* D,
                        const double* dt_bias, const double* init,
                        const double* dy, const double* dfinal,
                        const int32_t* heads, int nheads_sel,
                        double* dx, double* ddt, double* dA_part, double* dB, double* dC,
                        double* dD_part, double* dbias_part, double* dinit, int nthreads) {
  const int H = nheads, P = headdim, N = dstate, G = ngroups;
  if (H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0 || ndocs < 0) return -1;
  if (doc_offsets == NULL || doc_offsets[0] != 0 || doc_offsets[ndocs] != ntokens) return -1;
  for (int d = 0; d < ndocs; ++d)
    if (doc_offsets[d + 1] < doc_offsets[d]) return -1;
  char* sel = (char*)calloc((size_t)H, 1);
  if (!sel) return -2;
  if (heads) {
    for (int i = 0; i < nheads_sel; ++i) {
      if (heads[i] < 0 || heads[i] >= H) {
        free(sel);
        return -1;
      }
      sel[heads[i]] = 1;
    }
  } else {
    memset(sel, 1, (size_t)H);
  }
  const int hpg = H / G;
  const size_t NP = (size_t)N * P;
  const int64_t ntasks = (int64_t)ndocs * G;
  int failed = 0;

#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif

#pragma omp parallel
  {
    int64_t maxlen = 0;
    for (int d = 0; d < ndocs; ++d)
      if (doc_offsets[d + 1] - doc_offsets[d] > maxlen) maxlen = doc_offsets[d + 1] - doc_offsets[d];
    /* S[j] = state before token j of the document (S[0] = initial state) */
    double* S = (double*)malloc(sizeof(double) * NP * (size_t)(maxlen + 1));
    double* Gm = (double*)malloc(sizeof(double) * NP);
    double* gB = (double*)malloc(sizeof(double) * (size_t)P);
    if (!S || !Gm || !gB) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t task = 0; task < ntasks; ++task) {
      if (!S || !Gm || !gB) continue;
      const int d = (int)(task / G), g = (int)(task % G);
      const int64_t t0 = doc_offsets[d], len = doc_offsets[d + 1] - t0;
      for (int h = g * hpg; h < (g + 1) * hpg; ++h) {
        if (!sel[h]) continue;
        const double bias = dt_bias ? dt_bias[h] : 0.0;
        const double skip = D ? D[h] : 0.0;
        const size_t soff = ((size_t)d * H + h) * NP;
        /* forward sweep, keeping every state */
        if (init)
          memcpy(S, init + soff, sizeof(double) * NP);
        else
          memset(S, 0, sizeof(double) * NP);
        for (int64_t j = 0; j < len; ++j) {
          const int64_t t = t0 + j;
          const double delta = oracle_softplus(dt[t * H + h] + bias);
          const double decay = exp(delta * A[h]);
          const double* xt = x + ((size_t)t * H + h) * P;
          const double* Bt = B + ((size_t)t * G + g) * N;
          const double* prev = S + (size_t)j * NP;
          double* next = S + (size_t)(j + 1) * NP;
          for (int n = 0; n < N; ++n)
            for (int p = 0; p < P; ++p)
              next[(size_t)n * P + p] = decay * prev[(size_t)n * P + p] + delta * Bt[n] * xt[p];
        }
        /* backward sweep */
        if (dfinal)
          memcpy(Gm, dfinal + soff, sizeof(double) * NP);
        else
          memset(Gm, 0, sizeof(double) * NP);
        double dA_acc = 0.0, dD_acc = 0.0, db_acc = 0.0;
        for (int64_t j = len - 1; j >= 0; --j) {
          const int64_t t = t0 + j;
          const double z = dt[t * H + h] + bias;
          const double delta = oracle_softplus(z);
          const double decay = exp(delta * A[h]);
          const double* xt = x + ((size_t)t * H + h) * P;
          const double* dyt = dy + ((size_t)t * H + h) * P;
          const double* Bt = B + ((size_t)t * G + g) * N;
          const double* Ct = C + ((size_t)t * G + g) * N;
          const double* St = S + (size_t)(j + 1) * NP;   /* state after token t */
          const double* Sp = S + (size_t)j * NP;         /* state before token t */
          double* dBt = dB + ((size_t)t * G + g) * N;
          double* dCt = dC + ((size_t)t * G + g) * N;
          double* dxt = dx + ((size_t)t * H + h) * P;
          for (int n = 0; n < N; ++n)
            for (int p = 0; p < P; ++p) Gm[(size_t)n * P + p] += Ct[n] * dyt[p];
          for (int n = 0; n < N; ++n) {
            double s = 0.0;
            for (int p = 0; p < P; ++p) s += St[(size_t)n * P + p] * dyt[p];
            dCt[n] += s;
          }
          for (int p = 0; p < P; ++p) dD_acc += dyt[p] * xt[p];
          for (int p = 0; p < P; ++p) {
            double s = 0.0;
            for (int n = 0; n < N; ++n) s += Gm[(size_t)n * P + p] * Bt[n];
            gB[p] = s;
          }
          for (int p = 0; p < P; ++p) dxt[p] = delta * gB[p] + skip * dyt[p];
          for (int n = 0; n < N; ++n) {
            double s = 0.0;
            for (int p = 0; p < P; ++p) s += Gm[(size_t)n * P + p] * xt[p];
            dBt[n] += delta * s;
          }
          double inner = 0.0;
          for (size_t e = 0; e < NP; ++e) inner += Gm[e] * Sp[e];
          double xg = 0.0;
          for (int p = 0; p < P; ++p) xg += xt[p] * gB[p];
          const double ddelta = xg + A[h] * decay * inner;
          dA_acc += delta * decay * inner;
          const double g_dt = ddelta / (1.0 + exp(-z));
          ddt[t * H + h] = g_dt;
          db_acc += g_dt;
          for (size_t e = 0; e < NP; ++e) Gm[e] *= decay;
        }
        if (dinit) memcpy(dinit + soff, Gm, sizeof(double) * NP);
        dA_part[(size_t)d * H + h] = dA_acc;
        dD_part[(size_t)d * H + h] = dD_acc;
        dbias_part[(size_t)d * H + h] = db_acc;
      }
    }
    free(S);
    free(Gm);
    free(gB);
  }
  free(sel);
  return failed ? -2 : 0;
}
