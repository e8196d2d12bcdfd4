/*
 * dsa_oracle.c — plain, slow CPU definition of the DSA lightning indexer and
 * its MISA / MISA-dagger / HISA reductions.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path calls this code: only
 * the tests, the package's smoke check and the benchmark's CPU-baseline leg
 * load it.  It shares no code, header, table or constant with the CUDA library.
 *
 * Every quantity is the definition written out: operands are decoded to their
 * exact values, every dot product and head sum is accumulated in fp64 in
 * ascending index order, every selection is a full sort by the total order
 * (score descending, index ascending), and the final scores are rounded once
 * from fp64 to fp32 (nearest-even; -0.0 written as +0.0).  OpenMP only spreads
 * independent query rows over cores.
 *
 * Sources (page titles and sections):
 *  [DSA]  "PaperTrace 2.2.2 MISA, LISA and ResMiSA": the DSA score that opens
 *         the page (H_I heads share the history key k_s; query head q_{t,j}
 *         with weight w_{t,j}); section 2.2 "kernel boundary" (score, causal
 *         mask, top-k fused); section 2.3 "end-to-end acceptance" (explicit
 *         formula, causal mask, stable-sort top-k on small tensors).
 *  [MISA] "MISA: Mixture of Indexer Sparse Attention" summary, method steps
 *         1-6: pool the prefix into M = ceil(L/B) blocks, A_{t,j,b} =
 *         w_{t,j} ReLU(q_{t,j} . k~_b), E_{t,j} = (1/M) sum_b |A_{t,j,b}|,
 *         top-h heads, I^_{t,s} over the routed heads, top-k; MISA-dagger runs
 *         steps 4-5 twice, the second time with all H_I heads on k' candidates.
 *  [HISA] "PaperTrace 2.2.2", section 2.1 "HISA: filter blocks, then rerank
 *         tokens with the original formula"; "The new bottleneck of sparse
 *         attention", route one: HISA (mean-pooled block keys scored with the
 *         same indexer query, top blocks kept, DSA indexer run on their tokens).
 *  [LISA] "PaperTrace 2.2.2", section 3.1 "the shared key merges the linear
 *         term exactly": ReLU(x) = x + ReLU(-x), so
 *         I_{t,s} = g_t . k_s + sum_j w_{t,j} ReLU(-q_{t,j} . k_s) with the fused
 *         query g_t = sum_j w_{t,j} q_{t,j}; indexer LISA ranks tokens by the
 *         linear term l_{t,s} = g_t . k_s alone; LISA-dagger screens a pool by
 *         l and reranks it with every head.
 *  [RES]  "PaperTrace 2.2.2", section 3.2 "MISA-2 keeps the shared linear term
 *         and routes sparse residuals" (ResMiSA): per block b of the legal
 *         prefix and dimension c the key range [kmin_{b,c}, kmax_{b,c}];
 *         U^-_{t,b,j} = sum_c q+_c (-kmin_{b,c}) + q-_c kmax_{b,c} bounds
 *         -q_{t,j} . k over the block (q+ = max(q, 0), q- = max(-q, 0));
 *         S_{t,j} = |w_{t,j}| max_b ReLU(U^-_{t,b,j}); the top-r heads A_t;
 *         I^_{t,s} = l_{t,s} + sum_{j in A_t} w_{t,j} ReLU(-q_{t,j} . k_s).
 *  [BWD]  "PaperTrace 2.2.2", section 2.3 "why training gradients need
 *         recomputation": with z_{t,s,j} = q_{t,j} . k_s, m = 1[z > 0] (the ReLU
 *         derivative is 0 at 0) and an upstream gradient g_{t,s} on I_{t,s},
 *         the chain rule through I = sum_j w_j ReLU(z_j) gives
 *           dq_{t,j} = sum_s g_{t,s} w_{t,j} m_{t,s,j} k_s
 *           dk_s     = sum_t sum_j g_{t,s} w_{t,j} m_{t,s,j} q_{t,j}
 *           dw_{t,j} = sum_s g_{t,s} ReLU(z_{t,s,j})
 *         over the selected set S_t (the sparse stage recomputes only there).
 *  [DOSA] "The new bottleneck of sparse attention", route five (DoSA): a
 *         candidate whose upper bound lies below a lower bound of the k-th best
 *         score cannot enter the top-k, so skipping it leaves the top-k exact.
 *         The bound here is the library's reading: per block of 2^shift keys
 *         its per-dimension key range, hi / lo the largest / smallest q_j . k
 *         over that box, UB = sum_j (w_j > 0 ? w_j ReLU(hi_j) : w_j ReLU(lo_j))
 *         (ReLU is monotone), plus a rounding allowance 2^-12 sum_j |w_j|
 *         ||q_j||_1 max_c |k|_c.  DoSA's output is DSA's, which [DSA] defines.
 *  [SMLA] "PaperTrace 2.2.2", section 2.3 "end-to-end acceptance", second step:
 *         Sparse MLA on a fixed candidate set S_t, checked by logits, row
 *         maximum, softmax denominator and output against a naive gather
 *         attention; section 2.2: the selected positions feed Sparse MLA,
 *         which reads the latent KV at those positions.
 *  [FP8]  "PaperTrace 2.2.2", section 2.3 "from formula to FP8 cache":
 *         k^ = round(k/a), FP8 data plus scale, higher-precision accumulation.
 *         The e4m3 code follows the OCP 8-bit floating point specification
 *         (E4M3: bias 7, no infinities, S.1111.111 is NaN, max 448).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - The key is shared by all heads; the head subscript on k in the MISA
 *    summary's step 4 is read as a typo.
 *  - Query i of sequence b sits at position pos = q_pos0[b] + i; its legal
 *    keys are 0 <= s <= pos and s < k_len[b] (self-inclusive causal mask).
 *  - Rows with fewer than k legal keys return all of them, then (-1, -inf).
 *  - Ties: lower token index, lower head index, lower block index wins.
 *  - Blocks cover the legal prefix only; the block holding pos is the mean of
 *    its legal tokens.  A representative is the exact mean rounded once to the
 *    key storage type (bf16 or fp32).
 *  - MISA ranks heads by the un-normalised sum S_{t,j} = M_t E_{t,j}; the
 *    order is the same and E is reported as S / M_t.
 *  - HISA scores a block with the DSA formula on its representative
 *    (weights keep their sign, no absolute value).
 *  - Stacked MISA + HISA: the routed heads are used in both HISA stages.
 *  - LISA-dagger's pool is the exact top-min(M, |legal|) by the linear score
 *    (ties to the lower index): one fixed size inside the page's range
 *    [min(k, N_t), min(C, N_t)] for the pool; the page's sampling and
 *    histogram threshold estimate is not given, so the exact screen stands in.
 *  - ResMiSA's blocks are those of the MISA router (B tokens over the legal
 *    prefix, the boundary block holding only legal tokens); block extrema are
 *    of the key operand values; the routed residual heads are used in
 *    ascending head order; the reported score is I^.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Planted mistakes for the pin tests (tests/test_oracle_mutants.py): a build
 * with -DORC_MUTANT=n changes one step below; the default build (0) has none.
 * Each mutant is a plausible slip in writing the definitions down, and the pin
 * suite must reject every one of them. */
#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif
#define MUT(n) (ORC_MUTANT == (n))

/* ORC_F64: operands already decoded to fp64 values (the tests pass the split
 * query of orc_split_query this way); the CUDA library has no such type. */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2, ORC_F64 = 3 };
enum { ORC_OK = 0, ORC_ERR = -1 };

typedef struct {
  int32_t batch, n_q, n_k, heads, dim;
  int32_t q_dtype, k_dtype;
  const int32_t* q_pos0; /* [batch] or NULL: n_k - n_q */
  const int32_t* k_len;  /* [batch] or NULL: n_k */
  const void* q;         /* [batch,n_q,heads,dim] */
  const float* q_scale;  /* [batch,n_q] (e4m3 only) */
  const void* k;         /* [batch,n_k,dim] */
  const float* k_scale;  /* [batch,n_k] (e4m3 only) */
  const float* w;        /* [batch,n_q,heads] */
} orc_inputs;

/* ---------------------------------------------------------------- codecs -- */

/* OCP E4M3 decode: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN. */
double orc_e4m3_decode(uint8_t c) {
  int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, MUT(13) ? -10 : -9);
  else
    v = ldexp((double)(8 + m), e - 10);
  return sign ? -v : v;
}

/* Round-to-nearest-even, saturating OCP E4M3 encode of an fp32 value.
 * The representable magnitudes are m * 2^-9 (m = 0..7, subnormal) and
 * (8 + m) * 2^(e-10) for e = 1..15 (excluding e = 15, m = 7).  Values at or
 * beyond the largest finite magnitude 448 saturate to 448. */
uint8_t orc_e4m3_encode(float x) {
  double v = (double)x;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs(v);
  if (isnan(x)) return 0x7F;
  if (a >= 448.0) return sign | 0x7E;
  /* exponent e of the binade [2^(e-7), 2^(e-6)) holding a; subnormals use e = 1 spacing */
  int ex;
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) => binade exponent ex-1 */
  int E = ex - 1; /* a in [2^E, 2^(E+1)) */
  if (a == 0.0) return sign;
  if (E < -6) E = -6; /* subnormal range shares the spacing of the first binade */
  double ulp = ldexp(1.0, E - 3);
  double n = a / ulp; /* exact: scaling by a power of two */
  double fl = floor(n);
  double r = n - fl;
  double m_int = fl;
  if (!MUT(26) && (r > 0.5 || (r == 0.5 && (MUT(10) || fmod(fl, 2.0) != 0.0)))) m_int = fl + 1.0;
  double q = m_int * ulp; /* rounded magnitude */
  if (q >= 448.0) return sign | 0x7E;
  if (q == 0.0) return sign;
  /* re-derive the code from the rounded magnitude */
  frexp(q, &ex);
  E = ex - 1;
  if (E < -6) { /* subnormal */
    int mm = (int)(q / ldexp(1.0, -9));
    return sign | (uint8_t)mm;
  }
  int mm = (int)(q / ldexp(1.0, E - 3)) - 8;
  return sign | (uint8_t)(((E + 7) << 3) | mm);
}

/* Operand preparation: per-row scale a = amax / 448 in fp32 (amax == 0 gives
 * a = 1), code = e4m3(x / a) with the division in fp32.  [FP8] */
int orc_quantize_rows(const void* x, int32_t x_dtype, int64_t rows, int32_t cols, uint8_t* out,
                      float* out_scale) {
  if (x_dtype != ORC_F32 && x_dtype != ORC_BF16) return ORC_ERR;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    float amax = 0.0f;
    for (int32_t c = 0; c < cols; ++c) {
      float v;
      if (x_dtype == ORC_F32) {
        v = ((const float*)x)[r * cols + c];
      } else {
        uint32_t b = (uint32_t)((const uint16_t*)x)[r * cols + c] << 16;
        memcpy(&v, &b, 4);
      }
      float av = fabsf(v);
      if (av > amax) amax = av;
    }
    volatile float a = (amax > 0.0f) ? amax / (MUT(14) ? 240.0f : 448.0f) : 1.0f;
    out_scale[r] = a;
    for (int32_t c = 0; c < cols; ++c) {
      float v;
      if (x_dtype == ORC_F32) {
        v = ((const float*)x)[r * cols + c];
      } else {
        uint32_t b = (uint32_t)((const uint16_t*)x)[r * cols + c] << 16;
        memcpy(&v, &b, 4);
      }
      volatile float t = v / a;
      out[r * cols + c] = orc_e4m3_encode(t);
    }
  }
  return ORC_OK;
}

/* Query operand of the FP8-key path when the query arrives as bf16 / fp32:
 * the query is converted to the e4m3 compute type in two parts ([FP8]: the
 * query is converted to the compute type in registers, the dot products
 * accumulate in higher precision).  Reading: per (row, head) vector x of dim
 * values, s = amax|x| / 448 in fp32 (amax == 0 gives s = 1), v = x / s in fp32,
 * hi = e4m3(v), lo = e4m3(v - hi) with the subtraction in fp32; the operand
 * value is s * (hi + lo), written here exactly in fp64.
 *   x [vecs, dim] (F32 or BF16), out [vecs, dim] fp64. */
int orc_split_query(const void* x, int32_t x_dtype, int64_t vecs, int32_t dim, double* out) {
  if (x_dtype != ORC_F32 && x_dtype != ORC_BF16) return ORC_ERR;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < vecs; ++r) {
    float amax = 0.0f;
    for (int32_t c = 0; c < dim; ++c) {
      float v;
      if (x_dtype == ORC_F32) {
        v = ((const float*)x)[r * dim + c];
      } else {
        uint32_t b = (uint32_t)((const uint16_t*)x)[r * dim + c] << 16;
        memcpy(&v, &b, 4);
      }
      if (fabsf(v) > amax) amax = fabsf(v);
    }
    volatile float sc = (amax > 0.0f) ? amax / 448.0f : 1.0f;
    for (int32_t c = 0; c < dim; ++c) {
      float v;
      if (x_dtype == ORC_F32) {
        v = ((const float*)x)[r * dim + c];
      } else {
        uint32_t b = (uint32_t)((const uint16_t*)x)[r * dim + c] << 16;
        memcpy(&v, &b, 4);
      }
      volatile float t = v / sc;
      double hi = orc_e4m3_decode(orc_e4m3_encode(t));
      volatile float res = t - (float)hi;
      double lo = MUT(33) ? 0.0 : orc_e4m3_decode(orc_e4m3_encode(res));
      out[r * dim + c] = (double)sc * (hi + lo);
    }
  }
  return ORC_OK;
}

/* Nearest-even rounding of an exact fp64 value to bf16 (returned as double). */
static double round_to_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  double a = fabs(x);
  int ex;
  frexp(a, &ex);
  int E = ex - 1;
  if (E < -126) E = -126;              /* subnormal spacing 2^-133 */
  double ulp = ldexp(1.0, E - 7);      /* 8 significant bits */
  double n = a / ulp, fl = floor(n), r = n - fl, m = fl;
  if (r > 0.5 || (r == 0.5 && fmod(fl, 2.0) != 0.0)) m = fl + 1.0;
  double q = m * ulp;
  return x < 0 ? -q : q;
}

/* ------------------------------------------------------------- operands -- */

static double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << (MUT(25) ? 15 : 16);
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double q_val(const orc_inputs* in, int64_t row, int32_t j, int32_t c) {
  int64_t off = MUT(11) ? (row * in->dim + c) * (int64_t)in->heads + j
                        : (row * in->heads + j) * (int64_t)in->dim + c;
  switch (in->q_dtype) {
    case ORC_F32: return (double)((const float*)in->q)[off];
    case ORC_F64: return ((const double*)in->q)[off];
    case ORC_BF16: return bf16_value(((const uint16_t*)in->q)[off]);
    default: return (double)in->q_scale[row] * orc_e4m3_decode(((const uint8_t*)in->q)[off]);
  }
}

static double k_val(const orc_inputs* in, int32_t b, int64_t s, int32_t c) {
  int64_t kr = (int64_t)b * in->n_k + s;
  int64_t off = kr * in->dim + c;
  switch (in->k_dtype) {
    case ORC_F32: return (double)((const float*)in->k)[off];
    case ORC_F64: return ((const double*)in->k)[off];
    case ORC_BF16: return bf16_value(((const uint16_t*)in->k)[off]);
    default: return (double)in->k_scale[kr] * orc_e4m3_decode(((const uint8_t*)in->k)[off]);
  }
}

static int32_t row_pos(const orc_inputs* in, int64_t row) {
  int32_t b = (int32_t)(row / in->n_q), i = (int32_t)(row % in->n_q);
  int32_t p0 = in->q_pos0 ? in->q_pos0[b] : (MUT(21) ? 0 : in->n_k - in->n_q);
  return p0 + i;
}

/* Number of legal keys of a row: s <= pos and s < k_len. */
static int64_t row_legal(const orc_inputs* in, int64_t row) {
  int32_t b = (int32_t)(row / in->n_q);
  int64_t kl = (in->k_len && !MUT(5)) ? in->k_len[b] : in->n_k;
  int64_t n = (int64_t)row_pos(in, row) + (MUT(3) ? 0 : 1);
  if (n > kl) n = kl;
  return n < 0 ? 0 : n;
}

/* q_{t,j} . x for an explicit d-vector x (fp64). */
static double dot_q_vec(const orc_inputs* in, int64_t row, int32_t j, const double* x) {
  double acc = 0.0;
  for (int32_t c = 0; c < in->dim; ++c) acc += q_val(in, row, j, c) * x[c];
  return acc;
}

/* [DSA] I_{t,s} restricted to the listed heads (ascending): sum_j w_{t,j} max(q_{t,j}.k_s, 0).
 * The query row and the key are decoded to fp64 once; each head's dot product
 * runs over c ascending and the head sum over the listed order. */
static double score_heads(const orc_inputs* in, int64_t row, int64_t s, const int32_t* heads,
                          int32_t nh) {
  int32_t b = (int32_t)(row / in->n_q);
  double* kd = (double*)malloc(sizeof(double) * in->dim);
  for (int32_t c = 0; c < in->dim; ++c) kd[c] = k_val(in, b, s, c);
  double total = 0.0;
  for (int32_t a = 0; a < nh; ++a) {
    int32_t j = heads[a];
    double z = 0.0;
    for (int32_t c = 0; c < in->dim - (MUT(12) ? 1 : 0); ++c) z += q_val(in, row, j, c) * kd[c];
    total += (MUT(4) ? 1.0 : (double)in->w[row * in->heads + j]) * (MUT(1) ? z : (z > 0.0 ? z : 0.0));
  }
  free(kd);
  return total;
}

/* Decoded operands of one query row, reused across all its keys. */
typedef struct {
  double* q; /* [heads, dim] */
  double* kd; /* [dim] scratch */
} row_cache;

static row_cache row_cache_new(const orc_inputs* in, int64_t row) {
  row_cache rc;
  rc.q = (double*)malloc(sizeof(double) * (size_t)in->heads * in->dim);
  rc.kd = (double*)malloc(sizeof(double) * in->dim);
  for (int32_t j = 0; j < in->heads; ++j)
    for (int32_t c = 0; c < in->dim; ++c) rc.q[(size_t)j * in->dim + c] = q_val(in, row, j, c);
  return rc;
}

static void row_cache_free(row_cache* rc) {
  free(rc->q);
  free(rc->kd);
}

/* Same value as score_heads, reading the decoded query row from the cache. */
static double score_cached(const orc_inputs* in, row_cache* rc, int64_t row, int64_t s,
                           const int32_t* heads, int32_t nh) {
  int32_t b = (int32_t)(row / in->n_q);
  for (int32_t c = 0; c < in->dim; ++c) rc->kd[c] = k_val(in, b, s, c);
  double total = 0.0;
  for (int32_t a = 0; a < nh; ++a) {
    int32_t j = heads[a];
    const double* qj = rc->q + (size_t)j * in->dim;
    double z = 0.0;
    for (int32_t c = 0; c < in->dim - (MUT(12) ? 1 : 0); ++c) z += qj[c] * rc->kd[c];
    total += (MUT(4) ? 1.0 : (double)in->w[row * in->heads + j]) * (MUT(1) ? z : (z > 0.0 ? z : 0.0));
  }
  return total;
}

/* --------------------------------------------------------------- ranking -- */

typedef struct {
  double v;
  int64_t i;
} ranked;

/* Total order: value descending, index ascending ("stable sort", lower index wins). */
static int by_value_then_index(const void* a, const void* b) {
  const ranked* x = (const ranked*)a;
  const ranked* y = (const ranked*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  if (MUT(2)) return (x->i < y->i) - (x->i > y->i);
  return (x->i > y->i) - (x->i < y->i);
}

static float to_output_score(double v) {
  float f = (float)v;
  return f == 0.0f ? 0.0f : f; /* -0.0 -> +0.0 */
}

/* Write the first min(k, n) ranked entries then (-1, -inf) padding. */
static void emit_topk(const ranked* r, int64_t n, int32_t topk, int32_t* idx, float* sc,
                      double* sc64) {
  for (int32_t a = 0; a < topk; ++a) {
    if (a < n) {
      idx[a] = (int32_t)r[a].i;
      sc[a] = to_output_score(r[a].v);
      if (sc64) sc64[a] = r[a].v;
    } else {
      idx[a] = MUT(15) ? 0 : -1;
      sc[a] = -INFINITY;
      if (sc64) sc64[a] = -INFINITY;
    }
  }
}

/* ------------------------------------------------------------------ DSA -- */

/* [DSA] Exact top-k of I_{t,s} over the legal prefix, for the listed rows.
 * out_dots[r] = H * |legal| (the indexer's low-dimensional dot products). */
int orc_dsa_rows(const orc_inputs* in, int32_t topk, const int64_t* rows, int64_t n_rows,
                 int32_t* out_idx, float* out_score, double* out_score64, int64_t* out_dots) {
  int32_t* all = (int32_t*)malloc(sizeof(int32_t) * in->heads);
  for (int32_t j = 0; j < in->heads; ++j) all[j] = j;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t row = rows[r];
    int64_t n = row_legal(in, row);
    ranked* cand = (ranked*)malloc(sizeof(ranked) * (n > 0 ? n : 1));
    if (!cand) { err = 1; continue; }
    row_cache rc = row_cache_new(in, row);
    for (int64_t s = 0; s < n; ++s) {
      cand[s].v = score_cached(in, &rc, row, s, all, in->heads);
      cand[s].i = s;
    }
    row_cache_free(&rc);
    qsort(cand, (size_t)n, sizeof(ranked), by_value_then_index);
    emit_topk(cand, n, topk, out_idx + r * topk, out_score + r * topk,
              out_score64 ? out_score64 + r * topk : NULL);
    if (out_dots) out_dots[r] = (int64_t)in->heads * n;
    free(cand);
  }
  free(all);
  return err ? ORC_ERR : ORC_OK;
}

/* fp64 scores at explicit (row, s) pairs; heads == NULL means all heads,
 * otherwise heads is [n, nh] (one head list per pair). */
int orc_score_pairs(const orc_inputs* in, const int64_t* rows, const int64_t* s, int64_t n,
                    const int32_t* heads, int32_t nh, double* out) {
  int32_t* all = (int32_t*)malloc(sizeof(int32_t) * in->heads);
  for (int32_t j = 0; j < in->heads; ++j) all[j] = j;
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    if (heads)
      out[a] = score_heads(in, rows[a], s[a], heads + a * nh, nh);
    else
      out[a] = score_heads(in, rows[a], s[a], all, in->heads);
  }
  free(all);
  return ORC_OK;
}

/* Magnitude scale of a score at (row, s), the denominator of the relative
 * score tolerance: nu = sum_j |w_{t,j}| ||q_{t,j}|| ||k_s|| / sqrt(d), the
 * Cauchy-Schwarz bound on |q . k| (||q|| ||k||) scaled by 1/sqrt(d) to the size
 * a dot product of unaligned d-vectors typically has, weighted by |w| and
 * summed over the heads.  Norms are of the decoded operand values, in fp64.
 * heads == NULL means all heads, otherwise heads is [n, nh].  Test
 * infrastructure: the tolerance rule divides score differences by
 * max(|I|, nu). */
int orc_nu_pairs(const orc_inputs* in, const int64_t* rows, const int64_t* s, int64_t n,
                 const int32_t* heads, int32_t nh, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    int64_t row = rows[a];
    int32_t b = (int32_t)(row / in->n_q);
    int32_t cnt = heads ? nh : in->heads;
    double kk = 0.0;
    for (int32_t c = 0; c < in->dim; ++c) {
      double v = k_val(in, b, s[a], c);
      kk += v * v;
    }
    double knorm = MUT(32) ? kk : sqrt(kk);
    double acc = 0.0;
    for (int32_t x = 0; x < cnt; ++x) {
      int32_t j = heads ? heads[a * nh + x] : x;
      double qq = 0.0;
      for (int32_t c = 0; c < in->dim; ++c) {
        double v = q_val(in, row, j, c);
        qq += v * v;
      }
      double wj = (double)in->w[row * in->heads + j];
      acc += (MUT(30) ? wj : fabs(wj)) * sqrt(qq);
    }
    out[a] = acc * knorm / (MUT(31) ? 1.0 : sqrt((double)in->dim));
  }
  return ORC_OK;
}

/* -------------------------------------------------------------- pooling -- */

/* Mean of key rows [lo, hi) of sequence b, rounded once to the key storage
 * type (bf16 or fp32).  [MISA] step 1 / [HISA] block representatives. */
static void pooled_key(const orc_inputs* in, int32_t b, int64_t lo, int64_t hi, int32_t blk,
                       double* out) {
  for (int32_t c = 0; c < in->dim; ++c) {
    double sum = 0.0;
    for (int64_t s = lo; s < hi; ++s) sum += k_val(in, b, s, c);
    double mean = sum / (double)(MUT(6) ? blk : hi - lo);
    out[c] = MUT(16) ? mean : (in->k_dtype == ORC_BF16) ? round_to_bf16(mean) : (double)(float)mean;
  }
}

/* Representatives of the ceil(n/blk) blocks of the legal prefix [0, n). */
static double* block_representatives(const orc_inputs* in, int32_t b, int64_t n, int32_t blk,
                                     int64_t* n_blocks) {
  int64_t m = MUT(28) ? n / blk : (n + blk - 1) / blk;
  double* reps = (double*)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1) * in->dim);
  for (int64_t a = 0; a < m; ++a) {
    int64_t lo = a * blk, hi = lo + blk < n ? lo + blk : n;
    if (MUT(17)) hi = lo + blk < in->n_k ? lo + blk : in->n_k;
    pooled_key(in, b, lo, hi, blk, reps + a * in->dim);
  }
  *n_blocks = m;
  return reps;
}

/* Exported for tests: representatives of sequence b's prefix [0, n). */
int orc_pool(const orc_inputs* in, int32_t b, int64_t n, int32_t blk, double* out) {
  int64_t m;
  double* reps = block_representatives(in, b, n, blk, &m);
  memcpy(out, reps, sizeof(double) * (size_t)m * in->dim);
  free(reps);
  return ORC_OK;
}

/* [MISA] steps 1-3 for one row: S_{t,j} = sum_b |w_{t,j}| max(q_{t,j}.k~_b, 0)
 * over the M_t blocks of the legal prefix; the top-h heads by (S desc, j asc)
 * are returned in ascending head order. */
static void misa_route(const orc_inputs* in, int64_t row, int32_t blk, int32_t h, double* S,
                       int32_t* heads_out, int64_t* m_out) {
  int32_t b = (int32_t)(row / in->n_q);
  int64_t n = row_legal(in, row), m;
  double* reps = block_representatives(in, b, n, blk, &m);
  ranked* order = (ranked*)malloc(sizeof(ranked) * in->heads);
  for (int32_t j = 0; j < in->heads; ++j) {
    double s = 0.0;
    double aw = MUT(7) ? (double)in->w[row * in->heads + j] : fabs((double)in->w[row * in->heads + j]);
    for (int64_t a = 0; a < m; ++a) {
      double z = dot_q_vec(in, row, j, reps + a * in->dim);
      s += aw * (MUT(29) ? fabs(z) : (z > 0.0 ? z : 0.0));
    }
    S[j] = s;
    order[j].v = s;
    order[j].i = MUT(8) ? in->heads - 1 - j : j;
  }
  qsort(order, (size_t)in->heads, sizeof(ranked), by_value_then_index);
  if (MUT(8))
    for (int32_t j = 0; j < in->heads; ++j) order[j].i = in->heads - 1 - order[j].i;
  /* ascending head order of the selected set */
  char* chosen = (char*)calloc((size_t)in->heads, 1);
  for (int32_t a = 0; a < h; ++a) chosen[order[a].i] = 1;
  int32_t c = 0;
  for (int32_t j = 0; j < in->heads; ++j)
    if (chosen[j]) heads_out[c++] = j;
  free(chosen);
  free(order);
  free(reps);
  *m_out = m;
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* [MISA] MISA (k_prime == 0) and MISA-dagger (k_prime > 0) for the listed rows.
 *  forced_heads [n_rows, h]  : use these heads instead of the router's (conditional parity)
 *  forced_pool  [n_rows, k'] : use this first-pass pool (entries < 0 ignored)
 * Outputs (optional ones may be NULL):
 *  out_idx/out_score/out_score64 [n_rows, topk]; out_heads [n_rows, h] ascending;
 *  out_E [n_rows, H] = S / M_t; out_pool [n_rows, k'] (pool in rank order, -1 padded);
 *  out_dots [n_rows] = H*M_t + h*|legal| (+ H*min(k', |legal|) for MISA-dagger). */
int orc_misa_rows(const orc_inputs* in, int32_t topk, int32_t blk, int32_t h, int32_t k_prime,
                  const int64_t* rows, int64_t n_rows, const int32_t* forced_heads,
                  const int32_t* forced_pool, int32_t* out_idx, float* out_score,
                  double* out_score64, int32_t* out_heads, double* out_E, int32_t* out_pool,
                  int64_t* out_dots) {
  if (in->k_dtype == ORC_E4M3 || h < 1 || h > in->heads || blk < 1) return ORC_ERR;
  int32_t* all = (int32_t*)malloc(sizeof(int32_t) * in->heads);
  for (int32_t j = 0; j < in->heads; ++j) all[j] = j;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t row = rows[r];
    int64_t n = row_legal(in, row), m = 0;
    double* S = (double*)malloc(sizeof(double) * in->heads);
    int32_t* heads = (int32_t*)malloc(sizeof(int32_t) * h);
    misa_route(in, row, blk, h, S, heads, &m);
    if (forced_heads) {
      memcpy(heads, forced_heads + r * h, sizeof(int32_t) * h);
      qsort(heads, (size_t)h, sizeof(int32_t), cmp_i32);
    }
    if (out_heads) memcpy(out_heads + r * h, heads, sizeof(int32_t) * h);
    if (out_E)
      for (int32_t j = 0; j < in->heads; ++j)
        out_E[r * in->heads + j] = m > 0 ? S[j] / (double)(MUT(22) ? 1 : m) : 0.0;
    /* step 4: routed-head score over every legal token */
    ranked* cand = (ranked*)malloc(sizeof(ranked) * (n > 0 ? n : 1));
    row_cache rc = row_cache_new(in, row);
    for (int64_t s = 0; s < n; ++s) {
      cand[s].v = MUT(23) ? score_cached(in, &rc, row, s, all, in->heads)
                          : score_cached(in, &rc, row, s, heads, h);
      cand[s].i = s;
    }
    qsort(cand, (size_t)n, sizeof(ranked), by_value_then_index);
    int64_t dots = (int64_t)in->heads * m + (int64_t)h * n;
    if (k_prime <= 0) {
      emit_topk(cand, n, topk, out_idx + r * topk, out_score + r * topk,
                out_score64 ? out_score64 + r * topk : NULL);
    } else {
      /* MISA-dagger: keep k' by the routed score, rerank with all heads */
      int64_t np = n < k_prime ? n : k_prime - (MUT(18) ? 1 : 0);
      ranked* pool = (ranked*)malloc(sizeof(ranked) * (np > 0 ? np : 1));
      int64_t cnt = 0;
      if (forced_pool) {
        for (int32_t a = 0; a < k_prime; ++a) {
          int32_t s = forced_pool[r * k_prime + a];
          if (s >= 0 && cnt < np) pool[cnt++].i = s;
        }
      } else {
        for (int64_t a = 0; a < np; ++a) pool[cnt++].i = cand[a].i;
      }
      if (out_pool)
        for (int32_t a = 0; a < k_prime; ++a)
          out_pool[r * k_prime + a] = a < cnt ? (int32_t)pool[a].i : -1;
      for (int64_t a = 0; a < cnt; ++a)
        pool[a].v = MUT(24) ? score_cached(in, &rc, row, pool[a].i, heads, h)
                            : score_cached(in, &rc, row, pool[a].i, all, in->heads);
      qsort(pool, (size_t)cnt, sizeof(ranked), by_value_then_index);
      emit_topk(pool, cnt, topk, out_idx + r * topk, out_score + r * topk,
                out_score64 ? out_score64 + r * topk : NULL);
      dots += (int64_t)in->heads * cnt;
      free(pool);
    }
    if (out_dots) out_dots[r] = dots;
    row_cache_free(&rc);
    free(cand);
    free(heads);
    free(S);
  }
  free(all);
  return ORC_OK;
}

/* [HISA] (route_h == 0) and stacked MISA + HISA (route_h > 0) for the listed rows.
 *  1. (stacked) MISA router with block route_blk picks route_h heads;
 *  2. blocks of blk tokens over the legal prefix, representatives as in MISA;
 *     J_{t,b} = sum_{j in heads} w_{t,j} max(q_{t,j}.k~_b, 0);
 *  3. keep the top-r blocks by (J desc, b asc)  (or forced_blocks [n_rows, r]);
 *  4. score the legal tokens of the kept blocks with the same heads; top-k.
 *  out_blocks [n_rows, r] kept blocks in rank order (-1 padded); out_J [n_rows, r]
 *  their scores; out_dots = (H*M_t) + |heads|*M^b_t + |heads|*|candidates|. */
int orc_hisa_rows(const orc_inputs* in, int32_t topk, int32_t blk, int32_t r_keep,
                  int32_t route_h, int32_t route_blk, const int64_t* rows, int64_t n_rows,
                  const int32_t* forced_heads, const int32_t* forced_blocks, int32_t* out_idx,
                  float* out_score, double* out_score64, int32_t* out_blocks, double* out_J,
                  int32_t* out_heads, int64_t* out_dots) {
  if (in->k_dtype == ORC_E4M3 || blk < 1 || r_keep < 1) return ORC_ERR;
  if (route_h < 0 || route_h > in->heads) return ORC_ERR;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t row = rows[r];
    int32_t b = (int32_t)(row / in->n_q);
    int64_t n = row_legal(in, row);
    int32_t nh = route_h > 0 ? route_h : in->heads;
    int32_t* heads = (int32_t*)malloc(sizeof(int32_t) * nh);
    int64_t dots = 0;
    if (route_h > 0) {
      double* S = (double*)malloc(sizeof(double) * in->heads);
      int64_t m = 0;
      misa_route(in, row, route_blk, route_h, S, heads, &m);
      dots += (int64_t)in->heads * m;
      free(S);
      if (forced_heads) {
        memcpy(heads, forced_heads + r * nh, sizeof(int32_t) * nh);
        qsort(heads, (size_t)nh, sizeof(int32_t), cmp_i32);
      }
      if (out_heads) memcpy(out_heads + r * nh, heads, sizeof(int32_t) * nh);
    } else {
      for (int32_t j = 0; j < nh; ++j) heads[j] = j;
    }
    /* coarse stage: block scores */
    int64_t mb = 0;
    double* reps = block_representatives(in, b, n, blk, &mb);
    ranked* bl = (ranked*)malloc(sizeof(ranked) * (mb > 0 ? mb : 1));
    for (int64_t a = 0; a < mb; ++a) {
      double J = 0.0;
      for (int32_t x = 0; x < nh; ++x) {
        int32_t j = heads[x];
        double z = dot_q_vec(in, row, j, reps + a * in->dim);
        J += (MUT(9) ? 1.0 : (double)in->w[row * in->heads + j]) * (z > 0.0 ? z : 0.0);
      }
      bl[a].v = J;
      bl[a].i = a;
    }
    dots += (int64_t)nh * mb;
    qsort(bl, (size_t)mb, sizeof(ranked), by_value_then_index);
    int64_t kept = mb < r_keep ? mb : r_keep - (MUT(19) ? 1 : 0);
    char* keep = (char*)calloc((size_t)(mb > 0 ? mb : 1), 1);
    if (forced_blocks) {
      kept = 0;
      for (int32_t a = 0; a < r_keep; ++a) {
        int32_t x = forced_blocks[r * r_keep + a];
        if (x >= 0 && x < mb && !keep[x]) { keep[x] = 1; ++kept; }
      }
    } else {
      for (int64_t a = 0; a < kept; ++a) keep[bl[a].i] = 1;
    }
    if (out_blocks || out_J) {
      for (int32_t a = 0; a < r_keep; ++a) {
        int in_range = !forced_blocks && a < kept;
        if (out_blocks) out_blocks[r * r_keep + a] = in_range ? (int32_t)bl[a].i : -1;
        if (out_J) out_J[r * r_keep + a] = in_range ? bl[a].v : -INFINITY;
      }
    }
    /* fine stage: the DSA formula on the kept blocks' legal tokens */
    ranked* cand = (ranked*)malloc(sizeof(ranked) * (n > 0 ? n : 1));
    int64_t nc = 0;
    row_cache rc = row_cache_new(in, row);
    int32_t* allh = NULL;
    if (MUT(20)) {
      allh = (int32_t*)malloc(sizeof(int32_t) * in->heads);
      for (int32_t j = 0; j < in->heads; ++j) allh[j] = j;
    }
    for (int64_t s = 0; s < n; ++s) {
      if (!keep[s / blk]) continue;
      cand[nc].v = MUT(20) ? score_cached(in, &rc, row, s, allh, in->heads)
                           : score_cached(in, &rc, row, s, heads, nh);
      cand[nc].i = s;
      ++nc;
    }
    dots += (int64_t)nh * nc;
    qsort(cand, (size_t)nc, sizeof(ranked), by_value_then_index);
    emit_topk(cand, nc, topk, out_idx + r * topk, out_score + r * topk,
              out_score64 ? out_score64 + r * topk : NULL);
    if (out_dots) out_dots[r] = dots;
    row_cache_free(&rc);
    free(allh);
    free(cand);
    free(keep);
    free(bl);
    free(reps);
    free(heads);
  }
  return ORC_OK;
}

/* [HISA] coarse-stage scores of one row over every block of its legal prefix:
 * J_{t,a} = sum_{x} w_{t,heads[x]} max(q_{t,heads[x]} . k~_a, 0) (heads NULL: all),
 * the boundary block represented by the mean of its legal tokens.  Writes
 * out[0 .. M^b_t) and returns M^b_t.  Used by tests to judge near-ties at the
 * block cut-off. */
int64_t orc_block_scores(const orc_inputs* in, int64_t row, int32_t blk, const int32_t* heads,
                         int32_t nh, double* out) {
  int32_t b = (int32_t)(row / in->n_q);
  int64_t n = row_legal(in, row), m = 0;
  double* reps = block_representatives(in, b, n, blk, &m);
  for (int64_t a = 0; a < m; ++a) {
    double J = 0.0;
    int32_t cnt = heads ? nh : in->heads;
    for (int32_t x = 0; x < cnt; ++x) {
      int32_t j = heads ? heads[x] : x;
      double z = dot_q_vec(in, row, j, reps + a * in->dim);
      J += (double)in->w[row * in->heads + j] * (z > 0.0 ? z : 0.0);
    }
    out[a] = J;
  }
  free(reps);
  return m;
}

/* ------------------------------------------------------ LISA / ResMiSA -- */

/* [LISA] fused query g_t = sum_j w_{t,j} q_{t,j} (fp64, heads ascending). */
static void fused_query(const orc_inputs* in, int64_t row, double* g) {
  for (int32_t c = 0; c < in->dim; ++c) g[c] = 0.0;
  for (int32_t j = 0; j < in->heads; ++j) {
    double wj = (double)in->w[row * in->heads + j];
    for (int32_t c = 0; c < in->dim; ++c) g[c] += wj * q_val(in, row, j, c);
  }
}

/* [LISA] linear term l_{t,s} = g_t . k_s. */
static double linear_score(const orc_inputs* in, int64_t row, int64_t s, const double* g) {
  int32_t b = (int32_t)(row / in->n_q);
  double acc = 0.0;
  for (int32_t c = 0; c < in->dim; ++c) acc += g[c] * k_val(in, b, s, c);
  return acc;
}

/* [LISA] indexer LISA (pool_m == 0): top-k of l over the legal prefix, scores l.
 * LISA-dagger (pool_m > 0): pool = top-min(pool_m, |legal|) by l (or
 * forced_pool [n_rows, pool_m], entries < 0 ignored), reranked by the full I
 * over every head; top-k, scores I.
 * out_pool [n_rows, pool_m] (rank order, -1 padded); out_dots = |legal| key dots
 * (+ H * |pool| for the rerank). */
int orc_lisa_rows(const orc_inputs* in, int32_t topk, int32_t pool_m, const int64_t* rows,
                  int64_t n_rows, const int32_t* forced_pool, int32_t* out_idx, float* out_score,
                  double* out_score64, int32_t* out_pool, int64_t* out_dots) {
  if (pool_m < 0) return ORC_ERR;
  int32_t* all = (int32_t*)malloc(sizeof(int32_t) * in->heads);
  for (int32_t j = 0; j < in->heads; ++j) all[j] = j;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t row = rows[r];
    int64_t n = row_legal(in, row);
    double* g = (double*)malloc(sizeof(double) * in->dim);
    fused_query(in, row, g);
    ranked* cand = (ranked*)malloc(sizeof(ranked) * (n > 0 ? n : 1));
    row_cache rc = row_cache_new(in, row);
    for (int64_t s = 0; s < n; ++s) {
      cand[s].v = MUT(34) ? score_cached(in, &rc, row, s, all, in->heads)
                          : linear_score(in, row, s, g);
      cand[s].i = s;
    }
    qsort(cand, (size_t)n, sizeof(ranked), by_value_then_index);
    int64_t dots = n;
    if (pool_m == 0) {
      emit_topk(cand, n, topk, out_idx + r * topk, out_score + r * topk,
                out_score64 ? out_score64 + r * topk : NULL);
    } else {
      int64_t np = n < pool_m ? n : pool_m - (MUT(39) ? 1 : 0);
      ranked* pool = (ranked*)malloc(sizeof(ranked) * (np > 0 ? np : 1));
      int64_t cnt = 0;
      if (forced_pool) {
        for (int32_t a = 0; a < pool_m; ++a) {
          int32_t s = forced_pool[r * pool_m + a];
          if (s >= 0 && cnt < np) pool[cnt++].i = s;
        }
      } else {
        for (int64_t a = 0; a < np; ++a) pool[cnt++].i = cand[a].i;
      }
      if (out_pool)
        for (int32_t a = 0; a < pool_m; ++a)
          out_pool[r * pool_m + a] = a < cnt ? (int32_t)pool[a].i : -1;
      for (int64_t a = 0; a < cnt; ++a)
        pool[a].v = score_cached(in, &rc, row, pool[a].i, all, in->heads);
      qsort(pool, (size_t)cnt, sizeof(ranked), by_value_then_index);
      emit_topk(pool, cnt, topk, out_idx + r * topk, out_score + r * topk,
                out_score64 ? out_score64 + r * topk : NULL);
      dots += (int64_t)in->heads * cnt;
      free(pool);
    }
    if (out_dots) out_dots[r] = dots;
    row_cache_free(&rc);
    free(cand);
    free(g);
  }
  free(all);
  return ORC_OK;
}

/* [RES] residual bounds of one row: U^-_{t,a,j} for the M_t blocks a of the
 * legal prefix (blocks of blk tokens; the last holds only legal tokens) and
 * every head j, written to out [M_t, H]; returns M_t. */
static int64_t residual_bounds(const orc_inputs* in, int64_t row, int32_t blk, double* out) {
  int32_t b = (int32_t)(row / in->n_q);
  int64_t n = row_legal(in, row);
  if (MUT(38)) n = in->n_k;
  int64_t m = (n + blk - 1) / blk;
  double* kmin = (double*)malloc(sizeof(double) * in->dim);
  double* kmax = (double*)malloc(sizeof(double) * in->dim);
  for (int64_t a = 0; a < m; ++a) {
    int64_t lo = a * blk, hi = lo + blk < n ? lo + blk : n;
    for (int32_t c = 0; c < in->dim; ++c) {
      kmin[c] = INFINITY;
      kmax[c] = -INFINITY;
    }
    for (int64_t s = lo; s < hi; ++s)
      for (int32_t c = 0; c < in->dim; ++c) {
        double v = k_val(in, b, s, c);
        if (v < kmin[c]) kmin[c] = v;
        if (v > kmax[c]) kmax[c] = v;
      }
    for (int32_t j = 0; j < in->heads; ++j) {
      double u = 0.0;
      for (int32_t c = 0; c < in->dim; ++c) {
        double qc = q_val(in, row, j, c);
        double qp = qc > 0.0 ? qc : 0.0, qn = qc < 0.0 ? -qc : 0.0;
        u += MUT(36) ? qp * (-kmax[c]) + qn * kmin[c] : qp * (-kmin[c]) + qn * kmax[c];
      }
      out[a * in->heads + j] = u;
    }
  }
  free(kmin);
  free(kmax);
  return m;
}

/* [DOSA] block bounds of one row over the n_k keys of its sequence in blocks
 * of 2^shift (the last may be partial; every key of a block counts, legal or
 * not): out[a] = UB_a, out_lb[a] = LB_a = sum_j (w_j > 0 ? w_j ReLU(lo_j) :
 * w_j ReLU(hi_j)) (the box's smallest score; may be NULL), out_slack[a] = the
 * rounding allowance (may be NULL); blocks holding none of the row's legal
 * keys: -inf, -inf and 0.  Returns the number of blocks, ceil(n_k / 2^shift). */
int64_t orc_dosa_bounds(const orc_inputs* in, int64_t row, int32_t shift, double* out,
                        double* out_lb, double* out_slack) {
  int32_t b = (int32_t)(row / in->n_q);
  int64_t bs = (int64_t)1 << shift;
  int64_t nblk = (in->n_k + bs - 1) / bs;
  int64_t nleg = row_legal(in, row);
  int64_t nb_leg = (nleg + bs - 1) / bs;
  double* kmin = (double*)malloc(sizeof(double) * in->dim);
  double* kmax = (double*)malloc(sizeof(double) * in->dim);
  for (int64_t a = 0; a < nblk; ++a) {
    if (a >= nb_leg) {
      out[a] = -INFINITY;
      if (out_lb) out_lb[a] = -INFINITY;
      if (out_slack) out_slack[a] = 0.0;
      continue;
    }
    int64_t lo = a * bs, hi = lo + bs < in->n_k ? lo + bs : in->n_k;
    double kabs = 0.0;
    for (int32_t c = 0; c < in->dim; ++c) {
      kmin[c] = INFINITY;
      kmax[c] = -INFINITY;
      for (int64_t s = lo; s < hi; ++s) {
        double v = k_val(in, b, s, c);
        if (v < kmin[c]) kmin[c] = v;
        if (v > kmax[c]) kmax[c] = v;
      }
      if (fabs(kmin[c]) > kabs) kabs = fabs(kmin[c]);
      if (fabs(kmax[c]) > kabs) kabs = fabs(kmax[c]);
    }
    double ub = 0.0, lb = 0.0, sl = 0.0;
    for (int32_t j = 0; j < in->heads; ++j) {
      double zhi = 0.0, zlo = 0.0, l1 = 0.0;
      for (int32_t c = 0; c < in->dim; ++c) {
        double qc = q_val(in, row, j, c);
        double a0 = qc * kmin[c], a1 = qc * kmax[c];
        zhi += MUT(47) ? a0 : (a0 > a1 ? a0 : a1);
        zlo += a0 < a1 ? a0 : a1;
        l1 += fabs(qc);
      }
      double wj = (double)in->w[row * in->heads + j];
      ub += wj > 0.0 ? wj * (zhi > 0.0 ? zhi : 0.0) : wj * (zlo > 0.0 ? zlo : 0.0);
      if (MUT(48) ? wj > 0.0 : wj <= 0.0)
        lb += wj * (zhi > 0.0 ? zhi : 0.0);
      else
        lb += wj * (zlo > 0.0 ? zlo : 0.0);
      sl += fabs(wj) * l1;
    }
    out[a] = ub;
    if (out_lb) out_lb[a] = lb;
    if (out_slack) out_slack[a] = ldexp(sl * kabs, -12);
  }
  free(kmin);
  free(kmax);
  return nblk;
}

/* [DOSA] seed-set lower bound of one row's keep-th best score: the blocks of
 * largest LB (ties to the lower block), taken in that order until they hold
 * keep of the row's legal keys; the seed is the last block's LB (-INFINITY when
 * the row has fewer than keep legal keys).  Every key of a chosen block scores
 * at least its LB, so keep legal keys score at least the seed. */
double orc_dosa_seed(const orc_inputs* in, int64_t row, int32_t shift, int32_t keep) {
  int64_t bs = (int64_t)1 << shift;
  int64_t nblk = (in->n_k + bs - 1) / bs;
  int64_t nleg = row_legal(in, row);
  if (nleg < keep) return -INFINITY;
  double* ub = (double*)malloc(sizeof(double) * nblk);
  double* lb = (double*)malloc(sizeof(double) * nblk);
  orc_dosa_bounds(in, row, shift, ub, lb, NULL);
  int64_t nb = (nleg + bs - 1) / bs;
  char* used = (char*)calloc((size_t)nb, 1);
  int64_t got = 0;
  double seed = -INFINITY;
  while (got < keep) {
    int64_t best = -1;
    for (int64_t a = 0; a < nb; ++a)
      if (!used[a] && (best < 0 || lb[a] > lb[best])) best = a;
    if (best < 0) break;
    used[best] = 1;
    int64_t cnt = nleg - best * bs;
    if (cnt > bs) cnt = bs;
    got += MUT(49) ? bs : cnt;
    seed = lb[best];
  }
  free(ub);
  free(lb);
  free(used);
  return got >= keep ? seed : -INFINITY;
}

/* Exported for tests: U^- [M_t, H] of one row; returns M_t. */
int64_t orc_residual_bounds(const orc_inputs* in, int64_t row, int32_t blk, double* out) {
  return residual_bounds(in, row, blk, out);
}

/* [RES] ResMiSA for the listed rows: residual routing S_{t,j} =
 * |w_{t,j}| max_a ReLU(U^-_{t,a,j}), A_t = top-r by (S desc, j asc) (or
 * forced_heads [n_rows, r]), then I^ = l + sum_{j in A_t} w_{t,j} ReLU(-q_{t,j}.k_s)
 * over the legal prefix; top-k, scores I^.
 * out_heads [n_rows, r] ascending; out_S [n_rows, H]; out_dots = (1 + r) |legal|
 * key dots (the router's H M_t block bounds are extra). */
int orc_resmisa_rows(const orc_inputs* in, int32_t topk, int32_t blk, int32_t r_res,
                     const int64_t* rows, int64_t n_rows, const int32_t* forced_heads,
                     int32_t* out_idx, float* out_score, double* out_score64, int32_t* out_heads,
                     double* out_S, int64_t* out_dots) {
  if (r_res < 0 || r_res > in->heads || blk < 1) return ORC_ERR;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t row = rows[r];
    int64_t n = row_legal(in, row);
    int64_t mmax = (in->n_k + blk - 1) / blk + 1;
    double* U = (double*)malloc(sizeof(double) * (size_t)mmax * in->heads);
    int64_t m = residual_bounds(in, row, blk, U);
    double* S = (double*)malloc(sizeof(double) * in->heads);
    ranked* order = (ranked*)malloc(sizeof(ranked) * in->heads);
    for (int32_t j = 0; j < in->heads; ++j) {
      double best = 0.0;
      for (int64_t a = 0; a < m; ++a) {
        double u = U[a * in->heads + j];
        if (u > best) best = u;
      }
      double wj = (double)in->w[row * in->heads + j];
      S[j] = (MUT(37) ? wj : fabs(wj)) * best;
      order[j].v = S[j];
      order[j].i = j;
    }
    qsort(order, (size_t)in->heads, sizeof(ranked), by_value_then_index);
    int32_t* heads = (int32_t*)malloc(sizeof(int32_t) * (r_res > 0 ? r_res : 1));
    if (forced_heads) {
      memcpy(heads, forced_heads + r * r_res, sizeof(int32_t) * r_res);
    } else {
      for (int32_t a = 0; a < r_res; ++a) heads[a] = (int32_t)order[a].i;
    }
    qsort(heads, (size_t)r_res, sizeof(int32_t), cmp_i32);
    if (out_heads) memcpy(out_heads + r * r_res, heads, sizeof(int32_t) * r_res);
    if (out_S) memcpy(out_S + r * in->heads, S, sizeof(double) * in->heads);
    double* g = (double*)malloc(sizeof(double) * in->dim);
    fused_query(in, row, g);
    ranked* cand = (ranked*)malloc(sizeof(ranked) * (n > 0 ? n : 1));
    row_cache rc = row_cache_new(in, row);
    int32_t b = (int32_t)(row / in->n_q);
    for (int64_t s = 0; s < n; ++s) {
      double v = linear_score(in, row, s, g);
      for (int32_t c = 0; c < in->dim; ++c) rc.kd[c] = k_val(in, b, s, c);
      for (int32_t a = 0; a < r_res; ++a) {
        int32_t j = heads[a];
        const double* qj = rc.q + (size_t)j * in->dim;
        double z = 0.0;
        for (int32_t c = 0; c < in->dim; ++c) z += qj[c] * rc.kd[c];
        double neg = MUT(35) ? z : -z;
        v += (double)in->w[row * in->heads + j] * (neg > 0.0 ? neg : 0.0);
      }
      cand[s].v = v;
      cand[s].i = s;
    }
    qsort(cand, (size_t)n, sizeof(ranked), by_value_then_index);
    emit_topk(cand, n, topk, out_idx + r * topk, out_score + r * topk,
              out_score64 ? out_score64 + r * topk : NULL);
    if (out_dots) out_dots[r] = (int64_t)(1 + r_res) * n;
    row_cache_free(&rc);
    free(cand);
    free(g);
    free(heads);
    free(order);
    free(S);
    free(U);
  }
  return ORC_OK;
}

/* fp64 linear terms l_{t,s} = g_t . k_s at explicit (row, s) pairs. [LISA] */
int orc_linear_pairs(const orc_inputs* in, const int64_t* rows, const int64_t* s, int64_t n,
                     double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    double* g = (double*)malloc(sizeof(double) * in->dim);
    fused_query(in, rows[a], g);
    out[a] = linear_score(in, rows[a], s[a], g);
    free(g);
  }
  return ORC_OK;
}

/* fp64 ResMiSA scores I^ = l + sum_{j in heads} w_j ReLU(-q_j . k_s) at explicit
 * (row, s) pairs; heads [n, r] (one residual head list per pair). [RES] */
int orc_resmisa_pairs(const orc_inputs* in, const int64_t* rows, const int64_t* s, int64_t n,
                      const int32_t* heads, int32_t r, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t a = 0; a < n; ++a) {
    int64_t row = rows[a];
    int32_t b = (int32_t)(row / in->n_q);
    double* g = (double*)malloc(sizeof(double) * in->dim);
    fused_query(in, row, g);
    double v = linear_score(in, row, s[a], g);
    for (int32_t x = 0; x < r; ++x) {
      int32_t j = heads[a * r + x];
      double z = 0.0;
      for (int32_t c = 0; c < in->dim; ++c) z += q_val(in, row, j, c) * k_val(in, b, s[a], c);
      v += (double)in->w[row * in->heads + j] * (-z > 0.0 ? -z : 0.0);
    }
    out[a] = v;
    free(g);
  }
  return ORC_OK;
}

/* ---------------------------------------------------- indexer backward -- */

/* [BWD] Gradients of L = sum_t sum_{s in S_t} g_{t,s} I_{t,s} with respect to q,
 * k and w, recomputing z over each row's selected positions sel [rows, topk]
 * (entries < 0 ignored) with upstream gradients grad [rows, topk].
 * dq [rows, heads, dim] and dw [rows, heads] are written; dk [batch, n_k, dim]
 * is written too (zero where no row selected the key).  Rows are processed in
 * order, so dk sums in a fixed order (single-threaded for that reason). */
int orc_indexer_backward(const orc_inputs* in, const int32_t* sel, const float* grad,
                         int32_t topk, double* dq, double* dk, double* dw) {
  int64_t rows = (int64_t)in->batch * in->n_q;
  memset(dq, 0, sizeof(double) * (size_t)rows * in->heads * in->dim);
  memset(dw, 0, sizeof(double) * (size_t)rows * in->heads);
  memset(dk, 0, sizeof(double) * (size_t)in->batch * in->n_k * in->dim);
  double* kd = (double*)malloc(sizeof(double) * in->dim);
  for (int64_t row = 0; row < rows; ++row) {
    int32_t b = (int32_t)(row / in->n_q);
    for (int32_t i = 0; i < topk; ++i) {
      int32_t s = sel[row * topk + i];
      if (s < 0) continue;
      double g = (double)grad[row * topk + i];
      for (int32_t c = 0; c < in->dim; ++c) kd[c] = k_val(in, b, s, c);
      for (int32_t j = 0; j < in->heads; ++j) {
        double z = 0.0;
        for (int32_t c = 0; c < in->dim; ++c) z += q_val(in, row, j, c) * kd[c];
        double wj = (double)in->w[row * in->heads + j];
        dw[row * in->heads + j] += g * (MUT(46) ? z : (z > 0.0 ? z : 0.0));
        if (!(MUT(44) ? z >= 0.0 : z > 0.0)) continue;
        double coef = g * (MUT(45) ? 1.0 : wj);
        for (int32_t c = 0; c < in->dim; ++c) {
          dq[(row * in->heads + j) * in->dim + c] += coef * kd[c];
          dk[((int64_t)b * in->n_k + s) * in->dim + c] += coef * q_val(in, row, j, c);
        }
      }
    }
  }
  free(kd);
  return ORC_OK;
}

/* --------------------------------------------------------- Sparse MLA -- */

/* [SMLA] Naive gather attention over a fixed candidate set.  Token t (of
 * sequence b = t / tps) with query heads q[t, h, 0:dqk] attends to the cached
 * latent rows kv[b, s, 0:dqk] of its selected positions s = idx[t, i] >= 0
 * (entries < 0 are empty):
 *   x_s = scale * q_h . kv_s                     (logits)
 *   m   = max_s x_s,  den = sum_s exp(x_s - m)   (row maximum, denominator)
 *   o_h = sum_s exp(x_s - m) kv_s[0:dv] / den    (the value is the latent's
 *                                                 first dv dimensions)
 *   lse = m + log(den)
 * q and kv are bf16 words; everything else fp64.  A token with no selected
 * position gets o = 0, m = lse = -inf, den = 0.
 * Reading: the value of MLA's absorbed form is the latent part of the cached
 * row (the first dv of its dqk dimensions), the rope part joins the logits only. */
int orc_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int64_t T,
                   int32_t tps, int32_t n_k, int32_t heads, int32_t dqk, int32_t dv, int32_t topk,
                   double scale, double* out_o, double* out_lse, double* out_max,
                   double* out_den) {
  if (dv > dqk || tps < 1) return ORC_ERR;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    int64_t b = t / tps;
    double* x = (double*)malloc(sizeof(double) * (topk > 0 ? topk : 1));
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (topk > 0 ? topk : 1));
    for (int32_t i = 0; i < topk; ++i) {
      int32_t s = idx[t * topk + i];
      pos[i] = (s < 0 && MUT(43)) ? 0 : s;   /* planted mistake 43: empty read as position 0 */
    }
    for (int32_t h = 0; h < heads; ++h) {
      const uint16_t* qh = q + (t * heads + h) * (int64_t)dqk;
      double m = -INFINITY;
      for (int32_t i = 0; i < topk; ++i) {
        int32_t s = pos[i];
        if (s < 0) { x[i] = -INFINITY; continue; }
        const uint16_t* ks = kv + (b * n_k + s) * (int64_t)dqk;
        double acc = 0.0;
        for (int32_t c = 0; c < dqk; ++c) acc += bf16_value(qh[c]) * bf16_value(ks[c]);
        x[i] = (MUT(40) ? 1.0 : scale) * acc;
        if (x[i] > m) m = x[i];
      }
      double den = 0.0;
      double* o = out_o + (t * heads + h) * (int64_t)dv;
      for (int32_t c = 0; c < dv; ++c) o[c] = 0.0;
      if (m > -INFINITY) {
        for (int32_t i = 0; i < topk; ++i) {
          if (x[i] == -INFINITY) continue;
          double p = exp(x[i] - m);
          den += p;
          const uint16_t* ks = kv + (b * n_k + pos[i]) * (int64_t)dqk;
          int32_t off = MUT(41) ? dqk - dv : 0;
          for (int32_t c = 0; c < dv; ++c) o[c] += p * bf16_value(ks[off + c]);
        }
        for (int32_t c = 0; c < dv; ++c) o[c] /= den;
      }
      if (out_lse) out_lse[t * heads + h] = m > -INFINITY ? m + log(den) : -INFINITY;
      if (out_max) out_max[t * heads + h] = m;
      if (out_den) out_den[t * heads + h] = den;
    }
    free(pos);
    free(x);
  }
  return ORC_OK;
}

/* Full fp64 score row (all legal s) of one query row for the listed heads
 * (NULL = all); returns |legal|.  Used by tests for margins and tie checks. */
int64_t orc_score_row(const orc_inputs* in, int64_t row, const int32_t* heads, int32_t nh,
                      double* out) {
  int64_t n = row_legal(in, row);
  int32_t* all = NULL;
  if (!heads) {
    all = (int32_t*)malloc(sizeof(int32_t) * in->heads);
    for (int32_t j = 0; j < in->heads; ++j) all[j] = j;
    heads = all;
    nh = in->heads;
  }
#pragma omp parallel for schedule(static)
  for (int64_t s = 0; s < n; ++s) out[s] = score_heads(in, row, s, heads, nh);
  free(all);
  return n;
}
