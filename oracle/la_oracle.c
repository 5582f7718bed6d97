/*
 * la_oracle.c — fp64 CPU oracle of the Lightning Attention layer kernel.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg
 * may load this library.  It shares no code, header, table or constant with the CUDA path and
 * includes nothing from it.
 *
 * What it follows.
 *   - "Ling and Ring 2.6 Technical Report" (Chinese translation, garden.houmin.site), §4.1.1
 *     ("Context Parallel for Lightning Attention"): linear attention evaluated as an RNN-style
 *     recurrence over the sequence, O(N), with a per-head hidden state of shape [B,H,D,D].
 *   - §2.1, Fig. 2: the kernel sits between QK-Norm/RoPE and a grouped RMSNorm + sigmoid gate, so
 *     the kernel itself applies no normaliser, softmax or scale.
 *   - The decayed form of that recurrence is Lightning Attention's (TransNormerLLM, the report's
 *     reference 7).  The pages print neither the formula nor a decay schedule; the reading taken
 *     here is the plain one:
 *         S_t = lambda * S_{t-1} + k_t^T v_t,   o_t = q_t S_t,   lambda = exp(-slope)
 *     (diagonal term included, decay before adding the current token, read-out after the update).
 *
 * Arithmetic.  Inputs are upcast exactly from their stored bf16 or fp32 bits to double; lambda is
 * exp(-(double)slope); the state and every sum are double; loops run in a fixed order (i over the
 * key dimension outermost, j over the value dimension innermost, tokens in order).  Compile
 * without -ffast-math and with -ffp-contract=off.  OpenMP parallelises over independent heads
 * only, so the result does not depend on the thread count.
 *
 * Parity pins (tests/test_oracle.py): an O(N^2) brute-force decayed masked attention, the
 * lambda = 1 causal cumulative sum, the lambda -> 0 diagonal, N = 1, linearity in v and q,
 * prefix causality, and decode-after-prefill consistency.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_BF16 = 0, ORC_F32 = 1 };

/* Exact upcast of one stored element to double. */
static double orc_load(const void* base, int64_t idx, int dtype) {
  if (dtype == ORC_BF16) {
    uint16_t h = ((const uint16_t*)base)[idx];
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return (double)((const float*)base)[idx];
}

int orc_num_threads(int requested) {
#ifdef _OPENMP
  if (requested > 0) return requested;
  return omp_get_max_threads();
#else
  (void)requested;
  return 1;
#endif
}

/*
 * Prefill oracle: runs the recurrence over all N tokens of the selected heads.
 *
 *   B, N, H, d        shape of q, k, v: [B, N, H, d] contiguous, element type in_dtype
 *   slopes            float[H]
 *   heads, n_heads    flat head indices (b*H + h) to evaluate; heads == NULL means all B*H in order
 *   t_sel, n_t        sorted token indices whose outputs are recorded; t_sel == NULL means all N
 *   o                 double [n_sel_heads, n_t (or N), d]   (may be NULL)
 *   state             double [n_sel_heads, d, d]: final S   (may be NULL)
 *   state_in          double [n_sel_heads, d, d]: initial S (NULL = zero)
 *   nthreads          OpenMP threads (<= 0: default)
 * Returns 0, or -1 on a bad argument.
 */
int la_oracle_prefill(int64_t B, int64_t N, int64_t H, int64_t d, int in_dtype, const void* q,
                      const void* k, const void* v, const float* slopes, const int64_t* heads,
                      int64_t n_heads, const int64_t* t_sel, int64_t n_t, double* o,
                      double* state, const double* state_in, int nthreads) {
  if (B < 1 || N < 0 || H < 1 || d < 1 || !q || !k || !v || !slopes) return -1;
  if (in_dtype != ORC_BF16 && in_dtype != ORC_F32) return -1;
  const int64_t n_sel = heads ? n_heads : B * H;
  const int64_t n_out = t_sel ? n_t : N;
  int bad = 0;
  int nt = orc_num_threads(nthreads);

#pragma omp parallel for schedule(dynamic, 1) num_threads(nt) reduction(| : bad)
  for (int64_t sidx = 0; sidx < n_sel; ++sidx) {
    const int64_t flat = heads ? heads[sidx] : sidx;
    if (flat < 0 || flat >= B * H) { bad = 1; continue; }
    const int64_t b = flat / H, h = flat % H;
    const double lambda = exp(-(double)slopes[h]);
    double* S = (double*)malloc((size_t)(d * d) * sizeof(double));
    double* qt = (double*)malloc((size_t)d * sizeof(double));
    double* kt = (double*)malloc((size_t)d * sizeof(double));
    double* vt = (double*)malloc((size_t)d * sizeof(double));
    double* ot = (double*)malloc((size_t)d * sizeof(double));
    if (!S || !qt || !kt || !vt || !ot) {
      bad = 1;
      free(S); free(qt); free(kt); free(vt); free(ot);
      continue;
    }
    if (state_in) memcpy(S, state_in + sidx * d * d, (size_t)(d * d) * sizeof(double));
    else memset(S, 0, (size_t)(d * d) * sizeof(double));

    int64_t p = 0; /* next position in t_sel */
    for (int64_t t = 0; t < N; ++t) {
      const int64_t row = ((b * N + t) * H + h) * d;
      for (int64_t i = 0; i < d; ++i) {
        qt[i] = orc_load(q, row + i, in_dtype);
        kt[i] = orc_load(k, row + i, in_dtype);
        vt[i] = orc_load(v, row + i, in_dtype);
      }
      for (int64_t j = 0; j < d; ++j) ot[j] = 0.0;
      /* S <- lambda S + k^T v, then o = q S with the updated S. */
      for (int64_t i = 0; i < d; ++i) {
        double* Si = S + i * d;
        const double ki = kt[i], qi = qt[i];
        for (int64_t j = 0; j < d; ++j) {
          Si[j] = lambda * Si[j] + ki * vt[j];
          ot[j] += qi * Si[j];
        }
      }
      int record = 0;
      if (!t_sel) record = 1;
      else if (p < n_t && t_sel[p] == t) record = 1;
      if (record && o) {
        const int64_t pos = t_sel ? p : t;
        memcpy(o + (sidx * n_out + pos) * d, ot, (size_t)d * sizeof(double));
      }
      if (t_sel && p < n_t && t_sel[p] == t) ++p;
    }
    if (state) memcpy(state + sidx * d * d, S, (size_t)(d * d) * sizeof(double));
    free(S); free(qt); free(kt); free(vt); free(ot);
  }
  return bad ? -1 : 0;
}

/*
 * Decode oracle: one token for every (b, h), starting from the given state.
 *   q, k, v   [B, H, d], element type in_dtype
 *   state     double [B, H, d, d], updated in place: S <- lambda S + k^T v
 *   o         double [B, H, d]: o = q S (after the update)
 */
int la_oracle_decode(int64_t B, int64_t H, int64_t d, int in_dtype, const void* q, const void* k,
                     const void* v, const float* slopes, double* state, double* o,
                     int nthreads) {
  if (B < 1 || H < 1 || d < 1 || !q || !k || !v || !slopes || !state || !o) return -1;
  if (in_dtype != ORC_BF16 && in_dtype != ORC_F32) return -1;
  int nt = orc_num_threads(nthreads);
#pragma omp parallel for schedule(static) num_threads(nt)
  for (int64_t flat = 0; flat < B * H; ++flat) {
    const int64_t h = flat % H;
    const double lambda = exp(-(double)slopes[h]);
    double* S = state + flat * d * d;
    double* ot = o + flat * d;
    for (int64_t j = 0; j < d; ++j) ot[j] = 0.0;
    for (int64_t i = 0; i < d; ++i) {
      const double ki = orc_load(k, flat * d + i, in_dtype);
      const double qi = orc_load(q, flat * d + i, in_dtype);
      double* Si = S + i * d;
      for (int64_t j = 0; j < d; ++j) {
        const double vj = orc_load(v, flat * d + j, in_dtype);
        Si[j] = lambda * Si[j] + ki * vj;
        ot[j] += qi * Si[j];
      }
    }
  }
  return 0;
}
