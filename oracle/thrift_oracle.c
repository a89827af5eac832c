/*
 * CPU oracle for the selective mixed-precision (NVFP4 + FP16) attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file: only the tests, the package smoke check and the bench's CPU
 * baseline leg use it.  It shares no code, header or table with the CUDA
 * library; the two meet only in the seeded inputs of the `workloads` module.
 *
 * Plain, slow and written for a reader who checks it against the pages:
 *   ThriftAttention technical summary (gist.science 2605.23081, Dutch and
 *   French versions), section "Methodologie": block partition, block-mean
 *   score S^_ij = q_i . k_j, top-k pairs in FP16, the other pairs in NVFP4,
 *   online-softmax merge, two-level quantisation of the probability blocks.
 * Floating point is float64 unless a step names FP32 (the NVFP4 codec is
 * defined on FP32 values and is evaluated with IEEE FP32 operations here;
 * the build uses -ffp-contract=off so no product is fused).
 *
 * Readings of points the pages leave open:
 *   R-amax   one FP32 tensor scale per tensor: s_t = amax|X| / 2688 (2688 =
 *            6 * 448 maps the largest element onto the largest NVFP4 value);
 *            s_t = 1 when the tensor is all zero.
 *   R-group  Q and K grouped in 16s along d, V grouped in 16s along tokens
 *            (each group lies along the contraction axis of its product).
 *   R-block  s_b = E4M3(fp32(fp32(amax16 / 6) / s_t)); eff = fp32(s_b * s_t);
 *            code = E2M1(fp32(x / eff)); a group with eff == 0 gets +0 codes.
 *   R-round  E2M1 and E4M3 encodes round to nearest, ties to the even code,
 *            and saturate to the largest finite value; the sign of a value
 *            that rounds to zero is kept (E2M1 code 0x8).
 *   R-score  block means taken from the FP16 inputs, in float64; S^ carries
 *            no softmax scale; a causal pair is valid when its key block
 *            holds at least one key not above the last query of the block.
 *   R-topk   top-k over all valid pairs of one (batch, query head); ties to
 *            the smaller flat index i * nKb + j; k = ceil(bp * V / 10000).
 *   R1       first-level P scale per (row, key block): P' = 2688 exp(S - M)
 *            with M the row's maximum inside the key block; second level one
 *            E4M3 scale per 16 keys; the block's result is merged with weight
 *            exp(M - m) (m = row maximum over all valid keys); the softmax
 *            denominator sums the unquantised FP32 exp(S - M).
 *   R-fp16   the FP16 pairs use P rounded to FP16 and the FP16 V.
 *   R-decode decode (Nq query rows against a cache of Nk >= Nq keys): the
 *            query rows are the newest Nq positions Nk-Nq .. Nk-1, so causal
 *            masking is aligned bottom-right (key t visible to query row r
 *            when t <= Nk - Nq + r); the Nq rows form one query block, so the
 *            selection is one top-k per (batch, query head) over the key
 *            blocks with qbar the mean of the Nq rows; the query rows are
 *            quantised as their own tensor (their own FP32 tensor scale).
 *            Prefill is the case Nq = Nk.
 *   R-sparse the compute-matched sparse variant keeps only the selected
 *            pairs (in FP16) and drops every other pair, as if masked; a row
 *            left with no key has output 0 and lse -inf.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ FP16 */

double orc_half_to_double(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m | 0x400), e - 25);
  return s ? -v : v;
}

/* IEEE binary16 round to nearest even of a double (overflow gives inf). */
uint16_t orc_double_to_half(double x) {
  uint16_t s = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (isnan(x)) return 0x7e00;
  if (a >= 65520.0) return s | 0x7c00;
  if (a < ldexp(1.0, -14)) {
    /* subnormal grid: multiples of 2^-24 */
    double q = a * ldexp(1.0, 24);
    double f = floor(q), r = q - f;
    uint32_t m = (uint32_t)f;
    if (r > 0.5 || (r == 0.5 && (m & 1))) m++;
    return s | (uint16_t)m; /* m == 1024 is the smallest normal, encoded alike */
  }
  int e;
  double fr = frexp(a, &e); /* a = fr * 2^e, fr in [0.5, 1) */
  double q = fr * 2048.0;   /* 11 significant bits */
  double f = floor(q), r = q - f;
  uint32_t m = (uint32_t)f;
  if (r > 0.5 || (r == 0.5 && (m & 1))) m++;
  if (m == 2048) { m = 1024; e++; }
  int be = e - 1 + 15;
  if (be >= 31) return s | 0x7c00;
  return s | (uint16_t)((be << 10) | (m - 1024));
}

/* ------------------------------------------------------------------ E2M1 */

/* The 8 magnitudes of FP4 E2M1 (2 exponent bits, 1 mantissa bit); code bit 3 is the sign. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_decode(uint8_t c) {
  double v = E2M1_MAG[c & 7];
  return (c & 8) ? -v : v;
}

/* Nearest magnitude, ties to the even code, saturating at 6, sign kept. */
uint8_t orc_e2m1_encode(float x) {
  double a = fabs((double)x);
  uint8_t sign = signbit(x) ? 8 : 0;
  int best = 0;
  double bd = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double dd = fabs(a - E2M1_MAG[c]);
    if (dd < bd || (dd == bd && (c & 1) == 0)) { bd = dd; best = c; }
  }
  if (a >= 6.0) best = 7;
  return sign | (uint8_t)best;
}

/* ------------------------------------------------------------------ E4M3 */

/* FP8 E4M3 "fn" variant: bias 7, no infinities, 0x7f is NaN, largest 448. */
double orc_e4m3_decode(uint8_t c) {
  int e = (c >> 3) & 0xf, m = c & 7;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return (c & 0x80) ? -v : v;
}

/* Non-negative input only (scales): nearest finite value, ties to the even code, saturate at 448. */
uint8_t orc_e4m3_encode(float x) {
  double a = (double)x;
  if (!(a > 0.0)) return 0;
  if (a >= 448.0) return 0x7e;
  int lo = 0, hi = 0x7e; /* decode is increasing on [0, 0x7e] */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (orc_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid;
  }
  double dl = a - orc_e4m3_decode((uint8_t)lo), dh = orc_e4m3_decode((uint8_t)hi) - a;
  if (dl < dh) return (uint8_t)lo;
  if (dh < dl) return (uint8_t)hi;
  return (uint8_t)((lo & 1) ? hi : lo);
}

/* ----------------------------------------------------------------- NVFP4 */

static void quantize_group(const float* xs, float s_t, uint8_t* codes16, uint8_t* scale) {
  float amax16 = 0.0f;
  for (int t = 0; t < 16; ++t) {
    float a = fabsf(xs[t]);
    if (a > amax16) amax16 = a;
  }
  float r = amax16 / 6.0f;
  uint8_t sb = orc_e4m3_encode(r / s_t);
  float eff = (float)orc_e4m3_decode(sb) * s_t;
  *scale = sb;
  for (int t = 0; t < 16; ++t) codes16[t] = eff == 0.0f ? 0 : orc_e2m1_encode(xs[t] / eff);
}

/* NVFP4 quantisation of an FP16 tensor viewed as [outer, N, d] with a given FP32 tensor scale s_t
 * (reading R-append: a double-cached KV cache keeps the tensor scales it was built with and
 * encodes appended tokens with them; a value above the build-time amax saturates).
 *   group_axis 0: groups of 16 along d;  codes [outer, N, d/2], scales [outer, N, d/16].
 *   group_axis 1: groups of 16 along N;  codes [outer, d, N/2], scales [outer, d, N/16].
 * Element 2t of a code row is the low nibble of byte t. */
void orc_quantize_nvfp4_scaled(const uint16_t* x, int64_t outer, int32_t N, int32_t d, int32_t group_axis,
                               float s_t, uint8_t* codes, uint8_t* scales) {
  float xs[16];
  uint8_t c16[16];
  if (group_axis == 0) {
    int64_t rows = outer * (int64_t)N;
    for (int64_t r = 0; r < rows; ++r)
      for (int g = 0; g < d / 16; ++g) {
        for (int t = 0; t < 16; ++t) xs[t] = (float)orc_half_to_double(x[r * d + g * 16 + t]);
        quantize_group(xs, s_t, c16, &scales[r * (d / 16) + g]);
        for (int t = 0; t < 16; t += 2)
          codes[r * (d / 2) + (g * 16 + t) / 2] = (uint8_t)((c16[t] & 15) | ((c16[t + 1] & 15) << 4));
      }
  } else {
    for (int64_t o = 0; o < outer; ++o)
      for (int c = 0; c < d; ++c)
        for (int g = 0; g < N / 16; ++g) {
          for (int t = 0; t < 16; ++t)
            xs[t] = (float)orc_half_to_double(x[(o * N + (int64_t)g * 16 + t) * d + c]);
          quantize_group(xs, s_t, c16, &scales[(o * d + c) * (int64_t)(N / 16) + g]);
          for (int t = 0; t < 16; t += 2)
            codes[(o * d + c) * (int64_t)(N / 2) + (g * 16 + t) / 2] =
                (uint8_t)((c16[t] & 15) | ((c16[t + 1] & 15) << 4));
        }
  }
}

/* NVFP4 quantisation with the tensor's own scale s_t = amax|x| / 2688 (1 for an all-zero
 * tensor).  Returns s_t. */
float orc_quantize_nvfp4(const uint16_t* x, int64_t outer, int32_t N, int32_t d, int32_t group_axis,
                         uint8_t* codes, uint8_t* scales) {
  int64_t total = outer * (int64_t)N * d;
  float amax = 0.0f;
  for (int64_t i = 0; i < total; ++i) {
    float a = (float)fabs(orc_half_to_double(x[i]));
    if (a > amax) amax = a;
  }
  float s_t = amax > 0.0f ? amax / 2688.0f : 1.0f;
  orc_quantize_nvfp4_scaled(x, outer, N, d, group_axis, s_t, codes, scales);
  return s_t;
}

/* Dequantised value of element e of code row `row` (codes and scales as above),
 * without the tensor scale: E2M1 value times its E4M3 block scale. */
static inline double nvfp4_elem(const uint8_t* codes, const uint8_t* scales, int64_t row, int32_t len,
                                int32_t e) {
  uint8_t b = codes[row * (len / 2) + e / 2];
  uint8_t c = (e & 1) ? (b >> 4) : (b & 15);
  return orc_e2m1_decode(c) * orc_e4m3_decode(scales[row * (len / 16) + e / 16]);
}

double orc_nvfp4_elem(const uint8_t* codes, const uint8_t* scales, int64_t row, int32_t len, int32_t e) {
  return nvfp4_elem(codes, scales, row, len, e);
}

/* ---------------------------------------------------------- block select */

/* Pair (query block i, key block j) is valid when some key of block j is visible to some
 * row of block i; with the causal offset qoff, query row r sits at position qoff + r.  Keys at
 * or past nvalid (the cache's valid length, reading R-append) are never visible. */
static inline int pair_valid(int causal, int64_t qoff, int i, int j, int bq, int bk, int64_t nvalid) {
  if ((int64_t)j * bk >= nvalid) return 0;
  return !causal || (int64_t)j * bk <= qoff + (int64_t)(i + 1) * bq - 1;
}

int orc_pair_valid(int causal, int i, int j, int bq, int bk) {
  return pair_valid(causal, 0, i, j, bq, bk, (int64_t)1 << 62);
}

/* S^_ij = qbar_i . kbar_j per (batch, query head); -inf for invalid pairs.
 * q [B,Hq,Nq,d], k [B,Hkv,Nk,d] FP16, of which the first nvalid keys are the cache's valid
 * length (query row r at position nvalid - Nq + r); scores [B,Hq,Nq/bq,Nk/bk] float64.  A key
 * block's mean is over its keys below nvalid (reading R-append: a partly filled last block
 * averages the keys it holds). */
void orc_block_scores_qk(const uint16_t* q, const uint16_t* k, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         int bq, int bk, int causal, int nvalid, double* scores) {
  int nqb = Nq / bq, nkb = Nk / bk, grp = Hq / Hkv;
  int64_t qoff = (int64_t)nvalid - Nq;
  double* kbar = (double*)malloc(sizeof(double) * (size_t)nkb * d);
  double* qbar = (double*)malloc(sizeof(double) * (size_t)d);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < Hq; ++h) {
      const uint16_t* kh = k + ((int64_t)b * Hkv + h / grp) * (int64_t)Nk * d;
      const uint16_t* qh = q + ((int64_t)b * Hq + h) * (int64_t)Nq * d;
      for (int j = 0; j < nkb; ++j) {
        int64_t cnt = (int64_t)nvalid - (int64_t)j * bk;
        if (cnt > bk) cnt = bk;
        for (int c = 0; c < d; ++c) {
          double s = 0.0;
          for (int t = 0; t < cnt; ++t) s += orc_half_to_double(kh[((int64_t)j * bk + t) * d + c]);
          kbar[(int64_t)j * d + c] = cnt > 0 ? s / (double)cnt : 0.0;
        }
      }
      for (int i = 0; i < nqb; ++i) {
        for (int c = 0; c < d; ++c) {
          double s = 0.0;
          for (int t = 0; t < bq; ++t) s += orc_half_to_double(qh[((int64_t)i * bq + t) * d + c]);
          qbar[c] = s / bq;
        }
        double* row = scores + (((int64_t)b * Hq + h) * nqb + i) * nkb;
        for (int j = 0; j < nkb; ++j) {
          if (!pair_valid(causal, qoff, i, j, bq, bk, nvalid)) { row[j] = -INFINITY; continue; }
          double s = 0.0;
          for (int c = 0; c < d; ++c) s += qbar[c] * kbar[(int64_t)j * d + c];
          row[j] = s;
        }
      }
    }
  free(kbar);
  free(qbar);
}

/* Prefill form: q and k both [.., N, d]. */
void orc_block_scores(const uint16_t* q, const uint16_t* k, int B, int Hq, int Hkv, int N, int d, int bq,
                      int bk, int causal, double* scores) {
  orc_block_scores_qk(q, k, B, Hq, Hkv, N, N, d, bq, bk, causal, N, scores);
}

int64_t orc_topk_count(int64_t n_valid, int topk_abs, int topk_bp) {
  int64_t k = topk_abs >= 0 ? (int64_t)topk_abs : ((int64_t)topk_bp * n_valid + 9999) / 10000;
  if (k < 0) k = 0;
  if (k > n_valid) k = n_valid;
  return k;
}

typedef struct { double s; int64_t idx; } scored_t;

static int cmp_scored(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx);
}

/* Top-k of one head's [nQb*nKb] scores over the valid (finite) entries; sel[idx] = 1 when chosen.
 * Returns the k-th score (the smallest selected), or +inf when k == 0. */
double orc_topk(const double* scores, int64_t n, int64_t k, uint8_t* sel) {
  scored_t* v = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
  int64_t nv = 0;
  for (int64_t t = 0; t < n; ++t) {
    sel[t] = 0;
    if (isfinite(scores[t])) { v[nv].s = scores[t]; v[nv].idx = t; nv++; }
  }
  qsort(v, (size_t)nv, sizeof(scored_t), cmp_scored);
  if (k > nv) k = nv;
  for (int64_t t = 0; t < k; ++t) sel[v[t].idx] = 1;
  double kth = k > 0 ? v[k - 1].s : INFINITY;
  free(v);
  return kth;
}

/* ------------------------------------------------------------- attention */

typedef struct {
  const uint16_t *q, *k, *v;
  const uint8_t *q4c, *q4s, *k4c, *k4s, *v4c, *v4s;
  float q4t, k4t, v4t;
  const uint8_t* sel;
  int B, Hq, Hkv, Nq, Nk, d, bq, bk, causal;
  double tau;
  int sparse; /* 1: only the selected (FP16) pairs, the others dropped (R-sparse) */
  int nvalid; /* valid keys of the cache (the first nvalid positions of Nk); Nk for prefill */
} attn_problem;

/* position of query row 0 among the keys (bottom-right causal alignment) */
static inline int64_t qoff_of(const attn_problem* P) { return (int64_t)P->nvalid - P->Nq; }

static int pair_is_fp16(const attn_problem* P, int b, int h, int i, int j) {
  int nqb = P->Nq / P->bq, nkb = P->Nk / P->bk;
  return P->sel[(((int64_t)b * P->Hq + h) * nqb + i) * nkb + j] != 0;
}

/* Scores of the bq rows of query block i against key block j, [bq, bk], times tau.
 * FP4 pair: the exact sum of products of dequantised codes (each term has at most
 * 12 significant bits and d <= 256 terms, so float64 holds the sum exactly), times
 * s_tQ * s_tK * tau.  FP16 pair: sum of FP16 products in float64, times tau.
 * Keys above the query (causal) are -inf. */
static void block_scores(const attn_problem* P, int b, int h, int i, int j, int fp16, double* qd, double* kd,
                         double* S, int64_t ldS) {
  int d = P->d, hk = h / (P->Hq / P->Hkv);
  int64_t qbase = ((int64_t)b * P->Hq + h) * P->Nq + (int64_t)i * P->bq;
  int64_t kbase = ((int64_t)b * P->Hkv + hk) * P->Nk + (int64_t)j * P->bk;
  for (int t = 0; t < P->bk; ++t)
    for (int c = 0; c < d; ++c)
      kd[t * d + c] = fp16 ? orc_half_to_double(P->k[(kbase + t) * d + c])
                           : nvfp4_elem(P->k4c, P->k4s, kbase + t, d, c);
  double mult = fp16 ? P->tau : (double)P->q4t * (double)P->k4t * P->tau;
  for (int r = 0; r < P->bq; ++r) {
    for (int c = 0; c < d; ++c)
      qd[c] = fp16 ? orc_half_to_double(P->q[(qbase + r) * d + c]) : nvfp4_elem(P->q4c, P->q4s, qbase + r, d, c);
    int64_t row = qoff_of(P) + (int64_t)i * P->bq + r;
    for (int t = 0; t < P->bk; ++t) {
      int64_t key = (int64_t)j * P->bk + t;
      if ((P->causal && key > row) || key >= P->nvalid) { S[r * ldS + t] = -INFINITY; continue; }
      double s = 0.0;
      for (int c = 0; c < d; ++c) s += qd[c] * kd[t * d + c];
      S[r * ldS + t] = s * mult;
    }
  }
}

/* Two-level quantisation of one row of one key block (reading R1).
 * S: the row's scores in the block (-inf = masked).  Returns 0 when every key is
 * masked.  Otherwise writes M (row max in the block), sumP (sum of the FP32
 * exp(S - M), unquantised) and Pq (the probabilities the PV product uses, relative
 * to M: FP4 pairs dequantised NVFP4 codes / 2688, FP16 pairs FP16-rounded exp). */
static void tile_pq_at(const double* S, int bk, int fp16, double M, double* sumP_out, double* Pq);

int orc_tile_pq(const double* S, int bk, int fp16, double* M_out, double* sumP_out, double* Pq) {
  double M = -INFINITY;
  for (int t = 0; t < bk; ++t) if (S[t] > M) M = S[t];
  if (M == -INFINITY) return 0;
  tile_pq_at(S, bk, fp16, M, sumP_out, Pq);
  *M_out = M;
  return 1;
}

/* The same two-level quantisation with a given first-level reference M >= the tile's maximum:
 * P^ = exp(S - M) in FP32, P' = 2688 P^ quantised per 16 keys (NVFP4) or P^ rounded to FP16. */
static void tile_pq_at(const double* S, int bk, int fp16, double M, double* sumP_out, double* Pq) {
  float ph[512];
  double sum = 0.0;
  for (int t = 0; t < bk; ++t) {
    ph[t] = (S[t] == -INFINITY) ? 0.0f : (float)exp(S[t] - M);
    sum += (double)ph[t];
  }
  if (fp16) {
    for (int t = 0; t < bk; ++t) Pq[t] = orc_half_to_double(orc_double_to_half((double)ph[t]));
  } else {
    for (int g = 0; g < bk / 16; ++g) {
      float pp[16];
      float amax16 = 0.0f;
      for (int t = 0; t < 16; ++t) {
        pp[t] = 2688.0f * ph[g * 16 + t];
        if (pp[t] > amax16) amax16 = pp[t];
      }
      uint8_t sb = orc_e4m3_encode(amax16 / 6.0f);
      float sbv = (float)orc_e4m3_decode(sb);
      for (int t = 0; t < 16; ++t) {
        uint8_t code = sbv > 0.0f ? orc_e2m1_encode(pp[t] / sbv) : 0;
        Pq[g * 16 + t] = orc_e2m1_decode(code) * (double)sbv / 2688.0;
      }
    }
  }
  *sumP_out = sum;
}

/* V rows of key block j, [bk, d]: FP16 V, or the token-grouped NVFP4 V dequantised
 * (times its tensor scale). */
static void block_values(const attn_problem* P, int b, int h, int j, int fp16, double* vd) {
  int d = P->d, hk = h / (P->Hq / P->Hkv);
  int64_t vb = (int64_t)b * P->Hkv + hk;
  for (int t = 0; t < P->bk; ++t) {
    int key = j * P->bk + t;
    for (int c = 0; c < d; ++c)
      vd[t * d + c] = fp16 ? orc_half_to_double(P->v[(vb * P->Nk + key) * d + c])
                           : nvfp4_elem(P->v4c, P->v4s, vb * d + c, P->Nk, key) * (double)P->v4t;
  }
}

/* One (b, h, query block i) unit.  Two-pass (online = 0): m = the row maximum over all
 * valid keys, then each valid key block adds exp(M - m) * (Pq . V) to the output and
 * exp(M - m) * sumP to the denominator.  Online (online = 1): the valid blocks are visited
 * in the order `order` (a permutation of [0, nKb)) with a running maximum, rescaling the
 * running sums by exp(m_old - m_new) whenever it grows. */
static void attn_unit(const attn_problem* P, int b, int h, int i, int online, const int32_t* order,
                      uint16_t* out, float* lse, double* out64) {
  int nkb = P->Nk / P->bk, d = P->d, bq = P->bq, bk = P->bk;
  int64_t ldS = (int64_t)P->Nk, qoff = qoff_of(P);
  double* S = (double*)malloc(sizeof(double) * (size_t)bq * (size_t)P->Nk);
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  double* kd = (double*)malloc(sizeof(double) * (size_t)bk * d);
  double* vd = (double*)malloc(sizeof(double) * (size_t)bk * d);
  double* Pq = (double*)malloc(sizeof(double) * (size_t)bk);
  double* acc = (double*)calloc((size_t)bq * d, sizeof(double));
  double* m = (double*)malloc(sizeof(double) * (size_t)bq);
  double* l = (double*)calloc((size_t)bq, sizeof(double));
  for (int r = 0; r < bq; ++r) m[r] = -INFINITY;

  for (int j = 0; j < nkb; ++j) {
    if (!pair_valid(P->causal, qoff, i, j, bq, bk, P->nvalid) || (P->sparse && !pair_is_fp16(P, b, h, i, j))) {
      for (int r = 0; r < bq; ++r)
        for (int t = 0; t < bk; ++t) S[r * ldS + (int64_t)j * bk + t] = -INFINITY;
      continue;
    }
    block_scores(P, b, h, i, j, pair_is_fp16(P, b, h, i, j), qd, kd, S + (int64_t)j * bk, ldS);
  }
  if (!online)
    for (int r = 0; r < bq; ++r)
      for (int64_t t = 0; t < P->Nk; ++t) if (S[r * ldS + t] > m[r]) m[r] = S[r * ldS + t];

  for (int jj = 0; jj < nkb; ++jj) {
    int j = order ? order[jj] : jj;
    if (!pair_valid(P->causal, qoff, i, j, bq, bk, P->nvalid)) continue;
    if (P->sparse && !pair_is_fp16(P, b, h, i, j)) continue;
    int fp16 = pair_is_fp16(P, b, h, i, j);
    block_values(P, b, h, j, fp16, vd);
    for (int r = 0; r < bq; ++r) {
      double M, sumP;
      if (!orc_tile_pq(S + r * ldS + (int64_t)j * bk, bk, fp16, &M, &sumP, Pq)) continue;
      double* a = acc + (int64_t)r * d;
      if (online) {
        double mn = M > m[r] ? M : m[r];
        double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - mn);
        for (int c = 0; c < d; ++c) a[c] *= alpha;
        l[r] *= alpha;
        m[r] = mn;
      }
      double g = exp(M - m[r]);
      l[r] += g * sumP;
      for (int t = 0; t < bk; ++t) {
        if (Pq[t] == 0.0) continue;
        double w = g * Pq[t];
        for (int c = 0; c < d; ++c) a[c] += w * vd[t * d + c];
      }
    }
  }
  for (int r = 0; r < bq; ++r) {
    int64_t orow = ((int64_t)b * P->Hq + h) * P->Nq + (int64_t)i * bq + r;
    for (int c = 0; c < d; ++c) {
      /* l = 0 only when the row kept no key (R-sparse) */
      double o = l[r] > 0.0 ? acc[(int64_t)r * d + c] / l[r] : 0.0;
      out[orow * d + c] = orc_double_to_half(o);
      if (out64) out64[orow * d + c] = o;
    }
    lse[orow] = l[r] > 0.0 ? (float)(m[r] + log(l[r])) : -INFINITY;
  }
  free(S); free(qd); free(kd); free(vd); free(Pq); free(acc); free(m); free(l);
}

/* One (b, h, query block i) unit under reading R2 of the two-level P quantisation: the first level
 * is the row's running maximum m over the key blocks visited so far, in the fused kernel's order
 * (the NVFP4 blocks in ascending j, then the FP16 blocks in ascending j).  Per row and visited
 * block: m_new = max(m, M_block); the output and denominator so far are rescaled by
 * exp(m - m_new); P^ = exp(S - m_new) (so P' = 2688 P^ reaches 2688 only where the block holds
 * the running maximum); the quantised P^ times V is added to the output and the unquantised sum
 * of P^ to the denominator.  The result depends on the visiting order, unlike R1's. */
static void attn_unit_r2(const attn_problem* P, int b, int h, int i, uint16_t* out, float* lse, double* out64) {
  int nkb = P->Nk / P->bk, d = P->d, bq = P->bq, bk = P->bk;
  int64_t qoff = qoff_of(P);
  double* S = (double*)malloc(sizeof(double) * (size_t)bq * bk);
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  double* kd = (double*)malloc(sizeof(double) * (size_t)bk * d);
  double* vd = (double*)malloc(sizeof(double) * (size_t)bk * d);
  double* Pq = (double*)malloc(sizeof(double) * (size_t)bk);
  double* acc = (double*)calloc((size_t)bq * d, sizeof(double));
  double* m = (double*)malloc(sizeof(double) * (size_t)bq);
  double* l = (double*)calloc((size_t)bq, sizeof(double));
  for (int r = 0; r < bq; ++r) m[r] = -INFINITY;
  for (int phase = 0; phase < 2; ++phase) {
    for (int j = 0; j < nkb; ++j) {
      if (!pair_valid(P->causal, qoff, i, j, bq, bk, P->nvalid)) continue;
      int fp16 = pair_is_fp16(P, b, h, i, j);
      if (fp16 != phase) continue;
      block_scores(P, b, h, i, j, fp16, qd, kd, S, bk);
      block_values(P, b, h, j, fp16, vd);
      for (int r = 0; r < bq; ++r) {
        const double* Sr = S + (int64_t)r * bk;
        double M = -INFINITY;
        for (int t = 0; t < bk; ++t) if (Sr[t] > M) M = Sr[t];
        if (M == -INFINITY) continue;
        double mn = M > m[r] ? M : m[r];
        double alpha = m[r] == -INFINITY ? 0.0 : exp(m[r] - mn);
        double* a = acc + (int64_t)r * d;
        for (int c = 0; c < d; ++c) a[c] *= alpha;
        l[r] *= alpha;
        m[r] = mn;
        double sumP;
        tile_pq_at(Sr, bk, fp16, mn, &sumP, Pq);
        l[r] += sumP;
        for (int t = 0; t < bk; ++t) {
          if (Pq[t] == 0.0) continue;
          for (int c = 0; c < d; ++c) a[c] += Pq[t] * vd[t * d + c];
        }
      }
    }
  }
  for (int r = 0; r < bq; ++r) {
    int64_t orow = ((int64_t)b * P->Hq + h) * P->Nq + (int64_t)i * bq + r;
    for (int c = 0; c < d; ++c) {
      double o = l[r] > 0.0 ? acc[(int64_t)r * d + c] / l[r] : 0.0;
      out[orow * d + c] = orc_double_to_half(o);
      if (out64) out64[orow * d + c] = o;
    }
    lse[orow] = l[r] > 0.0 ? (float)(m[r] + log(l[r])) : -INFINITY;
  }
  free(S); free(qd); free(kd); free(vd); free(Pq); free(acc); free(m); free(l);
}

typedef struct {
  const attn_problem* P;
  const int32_t* units;
  int n_units;
  int online;
  const int32_t* order;
  uint16_t* out;
  float* lse;
  double* out64;
  int next;
  pthread_mutex_t mu;
} attn_job;

static void* attn_worker(void* arg) {
  attn_job* J = (attn_job*)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int u = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (u >= J->n_units) break;
    if (J->online == 2)
      attn_unit_r2(J->P, J->units[3 * u], J->units[3 * u + 1], J->units[3 * u + 2], J->out, J->lse, J->out64);
    else
      attn_unit(J->P, J->units[3 * u], J->units[3 * u + 1], J->units[3 * u + 2], J->online, J->order, J->out,
                J->lse, J->out64);
  }
  return NULL;
}

/* Attention forward over the listed (b, h, i) units (online = 0: reading R1, two-pass; 1: R1 with
 * an online merge in the order `order`; 2: reading R2, the kernel's visiting order).
 * Inputs: FP16 q [B,Hq,Nq,d], k, v
 * [B,Hkv,Nk,d] whose first nvalid keys are valid (query row r at position nvalid - Nq + r;
 * keys at or past nvalid are masked); NVFP4 codes/scales of q, k (grouped
 * along d) and v (grouped along tokens, [B,Hkv,d,Nk/2]) with their tensor scales;
 * sel [B,Hq,Nq/bq,Nk/bk] (1 = FP16 pair).  Writes O (FP16 [B,Hq,Nq,d], and float64 when
 * out64 != NULL) and lse (natural log, tau-scaled scores) for the rows of the listed units. */
void orc_attn_qk(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint8_t* q4c, const uint8_t* q4s,
                 float q4t, const uint8_t* k4c, const uint8_t* k4s, float k4t, const uint8_t* v4c,
                 const uint8_t* v4s, float v4t, const uint8_t* sel, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                 int bq, int bk, int causal, float tau, int sparse, int nvalid, const int32_t* units, int n_units,
                 int online, const int32_t* order, uint16_t* out, float* lse, double* out64, int n_threads) {
  attn_problem P = {q, k, v, q4c, q4s, k4c, k4s, v4c, v4s, q4t, k4t, v4t, sel,
                    B, Hq, Hkv, Nq, Nk, d, bq, bk, causal, (double)tau, sparse, nvalid};
  attn_job J;
  J.P = &P; J.units = units; J.n_units = n_units; J.online = online; J.order = order;
  J.out = out; J.lse = lse; J.out64 = out64; J.next = 0;
  pthread_mutex_init(&J.mu, NULL);
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  pthread_t th[256];
  for (int t = 0; t < n_threads; ++t) pthread_create(&th[t], NULL, attn_worker, &J);
  for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&J.mu);
}

/* Prefill form: q, k, v all [.., N, d]. */
void orc_attn(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint8_t* q4c, const uint8_t* q4s,
              float q4t, const uint8_t* k4c, const uint8_t* k4s, float k4t, const uint8_t* v4c,
              const uint8_t* v4s, float v4t, const uint8_t* sel, int B, int Hq, int Hkv, int N, int d, int bq,
              int bk, int causal, float tau, const int32_t* units, int n_units, int online,
              const int32_t* order, uint16_t* out, float* lse, double* out64, int n_threads) {
  orc_attn_qk(q, k, v, q4c, q4s, q4t, k4c, k4s, k4t, v4c, v4s, v4t, sel, B, Hq, Hkv, N, N, d, bq, bk, causal, tau,
              0, N, units, n_units, online, order, out, lse, out64, n_threads);
}

/* The tau-scaled scores of one (b, h, query block i, key block j) tile, [bq, bk] float64,
 * in the given precision (fp16 = 1: FP16 inputs; 0: NVFP4 inputs).  For the pins. */
void orc_tile_scores(const uint16_t* q, const uint16_t* k, const uint8_t* q4c, const uint8_t* q4s, float q4t,
                     const uint8_t* k4c, const uint8_t* k4s, float k4t, int B, int Hq, int Hkv, int N, int d,
                     int bq, int bk, int causal, float tau, int b, int h, int i, int j, int fp16, double* S) {
  attn_problem P = {q, k, NULL, q4c, q4s, k4c, k4s, NULL, NULL, q4t, k4t, 0.0f, NULL,
                    B, Hq, Hkv, N, N, d, bq, bk, causal, (double)tau, 0, N};
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  double* kd = (double*)malloc(sizeof(double) * (size_t)bk * d);
  block_scores(&P, b, h, i, j, fp16, qd, kd, S, bk);
  free(qd);
  free(kd);
}

/* ------------------------------------------------------- array helpers */

void orc_e2m1_encode_array(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(x[i]);
}

void orc_e4m3_encode_array(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

void orc_double_to_half_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_double_to_half(x[i]);
}

/* Per-head top-k over scores [heads, n]: sel [heads, n]; kth [heads]; k per head from the budget. */
void orc_select(const double* scores, int64_t heads, int64_t n, int topk_abs, int topk_bp, uint8_t* sel,
                double* kth, int64_t* kcount) {
  for (int64_t hh = 0; hh < heads; ++hh) {
    int64_t nv = 0;
    for (int64_t t = 0; t < n; ++t) nv += isfinite(scores[hh * n + t]) ? 1 : 0;
    int64_t k = orc_topk_count(nv, topk_abs, topk_bp);
    kcount[hh] = k;
    kth[hh] = orc_topk(scores + hh * n, n, k, sel + hh * n);
  }
}
