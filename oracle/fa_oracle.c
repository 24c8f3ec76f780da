/*
 * fa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * The plain, slow, fp64 CPU definition of scaled-dot-product attention over
 * packed variable-length sequences. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call it; the product path never does.
 * It shares no code with the CUDA library.
 *
 * Sources on the pages:
 *  - "Mecanismo cu_seqlens en FlashAttention" (friki.work), sections
 *    "Estructuras de datos clave" and "Lógica de cálculo de longitud": the
 *    cumulative offsets have batch+1 entries, sequence b owns rows
 *    [cu[b], cu[b+1]), its length is cu[b+1] - cu[b]; section
 *    "Optimización de acceso a memoria": a sequence's first element sits at
 *    row cu[b] of the packed tensor.
 *  - "FlashAttention na inferência" (slavadubrov.com), section "Separar o
 *    armazenamento do cálculo": standard materialised attention scores every
 *    visible (query, key) pair, normalises the scores and multiplies by V.
 *  - "FlashAttention-2 GPU work partitioning" (iplexlaw.co.kr), section
 *    "Bloques pequeños, normalización global": the normalisation is global
 *    over the row, and the result is exact attention.
 *  - "Flash-Atención y Flash-Atención-2" (zepes.com), sections on the
 *    backward: the backward exists and recomputes probabilities; the
 *    gradient formulas themselves are not printed, so the backward here is
 *    the chain rule of the forward definition. Same page, FlashAttention-2
 *    section on multi-query and grouped-query attention: several query
 *    heads attend to one key/value head.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - causal alignment when lq != lk is bottom-right: key j is visible from
 *    query i iff j <= i + (lk - lq);
 *  - a row with no visible key has output 0 and logsumexp -inf, and adds
 *    nothing to any gradient;
 *  - logsumexp is the natural log of the sum of exp of the SCALED scores;
 *  - with H query heads and Hk key/value heads (H a multiple of Hk; Hk = H
 *    is ordinary multi-head attention, Hk = 1 multi-query), query head h
 *    uses key/value head h / (H / Hk): consecutive query heads share one.
 *    The key/value gradients of a shared head are the sums over its group.
 *
 * Layouts: q/dout/out/dq are [total_q, H, d]; k/v/dk/dv are [total_k, Hk, d];
 * lse is [H, total_q]. Element (row, h, c) of a tensor with H heads sits at
 * (row*H + h)*d + c.
 * Inputs are either fp64 or raw bf16 bit patterns (widened exactly).
 *
 * Each (sequence, head) unit is independent; OpenMP runs units in parallel.
 * Within a unit the rows are processed one by one (no online softmax, no
 * blocking of the key dimension).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define FA_ORACLE_IN_F64 0
#define FA_ORACLE_IN_BF16 1

static double load_in(const void* p, int64_t idx, int dtype) {
  if (dtype == FA_ORACLE_IN_F64) return ((const double*)p)[idx];
  uint32_t bits = ((uint32_t)((const uint16_t*)p)[idx]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Visibility of key j from query i in a sequence with lq queries, lk keys. */
static int key_visible(int64_t i, int64_t j, int64_t lq, int64_t lk, int causal) {
  if (j < 0 || j >= lk) return 0;
  if (!causal) return 1;
  return j <= i + (lk - lq);
}

/* Sequence lengths from cumulative offsets: len[b] = cu[b+1] - cu[b].
 * Returns 0 on success, -1 if the offsets do not start at 0 or decrease. */
int fa_oracle_seqlens(const int32_t* cu, int batch, int32_t* len) {
  if (batch < 0 || cu[0] != 0) return -1;
  for (int b = 0; b < batch; ++b) {
    len[b] = cu[b + 1] - cu[b];
    if (len[b] < 0) return -1;
  }
  return 0;
}

/* Element offset of (row r of sequence b, head h, channel 0) in a packed
 * [total, H, d] tensor: the sequence starts at packed row cu[b]. 64-bit. */
int64_t fa_oracle_elem_offset(const int32_t* cu, int b, int64_t r, int H, int h, int d) {
  return ((int64_t)cu[b] + r) * (int64_t)H * d + (int64_t)h * d;
}

/* Scores of query row i against every key of the unit, scaled; masked
 * entries are -inf. Returns the number of visible keys. */
static int64_t score_row(const void* q, const void* k, int dtype, int64_t qoff, const int64_t* koffs,
                         int64_t i, int64_t lq, int64_t lk, int d, double scale, int causal,
                         double* s) {
  int64_t nvis = 0;
  for (int64_t j = 0; j < lk; ++j) {
    if (!key_visible(i, j, lq, lk, causal)) {
      s[j] = -INFINITY;
      continue;
    }
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += load_in(q, qoff + c, dtype) * load_in(k, koffs[j] + c, dtype);
    s[j] = scale * acc;
    ++nvis;
  }
  return nvis;
}

/* Softmax of one score row in place (s becomes P) and its logsumexp. */
static double softmax_row(double* s, int64_t lk, int64_t nvis) {
  if (nvis == 0) {
    for (int64_t j = 0; j < lk; ++j) s[j] = 0.0;
    return -INFINITY;
  }
  double mx = -INFINITY;
  for (int64_t j = 0; j < lk; ++j)
    if (s[j] > mx) mx = s[j];
  double sum = 0.0;
  for (int64_t j = 0; j < lk; ++j) sum += (s[j] == -INFINITY) ? 0.0 : exp(s[j] - mx);
  double lse = mx + log(sum);
  for (int64_t j = 0; j < lk; ++j) s[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - lse);
  return lse;
}

/* units: n_units (b, h) pairs; NULL means every (b, h). */
static int64_t unit_count(int batch, int H, int n_units, const int32_t* units) {
  return units ? n_units : (int64_t)batch * H;
}
static void unit_at(int64_t u, int H, const int32_t* units, int* b, int* h) {
  if (units) {
    *b = units[2 * u];
    *h = units[2 * u + 1];
  } else {
    *b = (int)(u / H);
    *h = (int)(u % H);
  }
}

/* Forward: out = softmax(scale * Q K^T, masked) V per unit; lse per row.
 * row_step > 1 computes only query rows i with i % row_step == 0 (rows are
 * independent in the forward, so a sample of rows is exact). */
int fa_oracle_fwd(const void* q, const void* k, const void* v, int dtype,
                  const int32_t* cu_q, const int32_t* cu_k, int batch, int H, int Hk, int d,
                  double scale, int causal, int n_units, const int32_t* units, int row_step,
                  double* out, double* lse) {
  if (Hk < 1 || H % Hk != 0) return -2;
  const int g = H / Hk;  /* query heads per key/value head */
  const int64_t total_q = cu_q[batch];
  const int64_t nu = unit_count(batch, H, n_units, units);
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < nu; ++u) {
    int b, h;
    unit_at(u, H, units, &b, &h);
    const int64_t lq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
    double* s = (double*)malloc(sizeof(double) * (size_t)(lk > 0 ? lk : 1));
    int64_t* koffs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(lk > 0 ? lk : 1));
    if (!s || !koffs) {
      err = -1;
      free(s);
      free(koffs);
      continue;
    }
    const int hk = h / g;
    for (int64_t j = 0; j < lk; ++j) koffs[j] = fa_oracle_elem_offset(cu_k, b, j, Hk, hk, d);
    for (int64_t i = 0; i < lq; i += (row_step > 1 ? row_step : 1)) {
      const int64_t qoff = fa_oracle_elem_offset(cu_q, b, i, H, h, d);
      int64_t nvis = score_row(q, k, dtype, qoff, koffs, i, lq, lk, d, scale, causal, s);
      double l = softmax_row(s, lk, nvis);
      lse[(int64_t)h * total_q + cu_q[b] + i] = l;
      double* o = out + qoff;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      for (int64_t j = 0; j < lk; ++j) {
        if (s[j] == 0.0) continue;
        for (int c = 0; c < d; ++c) o[c] += s[j] * load_in(v, koffs[j] + c, dtype);
      }
    }
    free(s);
    free(koffs);
  }
  return err;
}

/* Backward of L = sum(out * dout), recomputed from the inputs alone:
 *   P = softmax(S), dV = P^T dO, dP = dO V^T, D_i = sum_j P_ij dP_ij,
 *   dS = P * (dP - D), dQ = scale dS K, dK = scale dS^T Q.
 * A unit here is (sequence, key/value head): its query heads are visited one
 * after the other and their rows one by one; dK and dV of the unit
 * accumulate over all of them. */
int fa_oracle_bwd(const void* q, const void* k, const void* v, const void* dout, int dtype,
                  const int32_t* cu_q, const int32_t* cu_k, int batch, int H, int Hk, int d,
                  double scale, int causal, int n_units, const int32_t* units,
                  double* dq, double* dk, double* dv) {
  if (Hk < 1 || H % Hk != 0) return -2;
  const int g = H / Hk;  /* query heads per key/value head */
  const int64_t nu = unit_count(batch, Hk, n_units, units);
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < nu; ++u) {
    int b, hk;
    unit_at(u, Hk, units, &b, &hk);
    const int64_t lq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
    const size_t nk = (size_t)(lk > 0 ? lk : 1);
    double* p = (double*)malloc(sizeof(double) * nk);
    double* dp = (double*)malloc(sizeof(double) * nk);
    int64_t* koffs = (int64_t*)malloc(sizeof(int64_t) * nk);
    if (!p || !dp || !koffs) {
      err = -1;
      free(p);
      free(dp);
      free(koffs);
      continue;
    }
    for (int64_t j = 0; j < lk; ++j) {
      koffs[j] = fa_oracle_elem_offset(cu_k, b, j, Hk, hk, d);
      for (int c = 0; c < d; ++c) {
        dk[koffs[j] + c] = 0.0;
        dv[koffs[j] + c] = 0.0;
      }
    }
    for (int h = hk * g; h < (hk + 1) * g; ++h)
    for (int64_t i = 0; i < lq; ++i) {
      const int64_t qoff = fa_oracle_elem_offset(cu_q, b, i, H, h, d);
      int64_t nvis = score_row(q, k, dtype, qoff, koffs, i, lq, lk, d, scale, causal, p);
      softmax_row(p, lk, nvis);
      double D = 0.0;
      for (int64_t j = 0; j < lk; ++j) {
        double acc = 0.0;
        if (p[j] != 0.0)
          for (int c = 0; c < d; ++c) acc += load_in(dout, qoff + c, dtype) * load_in(v, koffs[j] + c, dtype);
        dp[j] = acc;
        D += p[j] * acc;
      }
      double* dqi = dq + qoff;
      for (int c = 0; c < d; ++c) dqi[c] = 0.0;
      for (int64_t j = 0; j < lk; ++j) {
        if (p[j] == 0.0) continue;
        const double ds = p[j] * (dp[j] - D);
        for (int c = 0; c < d; ++c) {
          dqi[c] += scale * ds * load_in(k, koffs[j] + c, dtype);
          dk[koffs[j] + c] += scale * ds * load_in(q, qoff + c, dtype);
          dv[koffs[j] + c] += p[j] * load_in(dout, qoff + c, dtype);
        }
      }
    }
    free(p);
    free(dp);
    free(koffs);
  }
  return err;
}

/* Number of threads OpenMP will use (for reporting the CPU baseline). */
int fa_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
