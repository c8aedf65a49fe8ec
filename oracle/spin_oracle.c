/*
 * spin_oracle.c -- plain, slow CPU oracle for the SPIN decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this code.  The product
 * library never links, loads or calls it, and it shares no code, header,
 * table or constant generator with the CUDA path.
 *
 * Sources (four web pages on SPIN; short names used below):
 *   [digest]  ai4snews digest of the SPIN paper, sections 核心概要 /
 *             arXiv深度剖析 / 启示与展望
 *   [listing] thelatestinai listing "SaveSPIN: Shadow Predictive Indexer for
 *             Sparse Attention": Abstract, Tables 1-7, Figures 1-4
 *   [v3]      paperdot record of arXiv:2610.09025 v3, 摘要 (abstract)
 *   [radio]   AI Radio episode "SPIN: Shadow Predictive Indexer for Sparse
 *             Attention", segments "Title and authors", "The paper's summary",
 *             "The paper's improvements"
 *
 * The pages do not print the indexer formula; the DSA lightning-indexer form
 * I_{t,s} = sum_h w_{t,h} * ReLU(q_{t,h} . k_s) is taken as the definition.
 * Where the pages leave a point open, the function that meets it states the
 * reading it takes.  Each function below says which passage it follows.
 *
 * Numerics: scores are computed in fp64 from the exact decoded operand
 * values.  The EMA state is fp32 by definition, and its update is written
 * with an explicit fmaf so that it can be compared bit for bit.
 * Build with -ffp-contract=off (no implicit contraction anywhere).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 counter-based generator.                                    */
/* Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", */
/* SC'11: the Philox-4x32 S-box uses two 32x32->64 multiplies per round with  */
/* multipliers 0xD2511F53 and 0xCD9E8D57; the round key is bumped by the     */
/* Weyl constants 0x9E3779B9 (golden ratio) and 0xBB67AE85 (sqrt(3)-1);      */
/* 10 rounds.                                                                */
/* ------------------------------------------------------------------------ */
ORC_API void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                               uint32_t out[4]) {
  uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x0;
    uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t y0 = hi1 ^ x1 ^ k0;
    uint32_t y1 = lo1;
    uint32_t y2 = hi0 ^ x3 ^ k1;
    uint32_t y3 = lo0;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Exploration key of logical block j: word (j mod 4) of Philox4x32-10 with
 * counter (j div 4, request, layer, step mod 2^32) and key (seed low, seed
 * high) -- one generator call gives the keys of four consecutive blocks.
 * Random exploration reserves part of the block budget for uniformly random
 * unkept blocks ([digest] arXiv深度剖析; [listing] Figure 4); drawing the
 * blocks with the smallest i.i.d. uniform keys is a uniform draw without
 * replacement. */
ORC_API uint32_t orc_explore_key(uint64_t seed, uint32_t block, uint32_t request,
                                 uint32_t layer, uint64_t step) {
  uint32_t ctr[4] = {block >> 2, request, layer, (uint32_t)step};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  return out[block & 3u];
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 (OCP 8-bit floating point spec, "E4M3" with no infinities):     */
/* 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; S.1111.111 is   */
/* NaN; the largest finite magnitude is 1.75 * 2^8 = 448; exponent field 0   */
/* encodes subnormals m * 2^-9.                                              */
/* ------------------------------------------------------------------------ */
ORC_API double orc_e4m3_decode(uint8_t code) {
  int sign = code >> 7;
  int e = (code >> 3) & 15;
  int m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m, -9);
  else mag = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* Round to nearest, ties to even mantissa, saturating to +-448 (the
 * "satfinite" behaviour: anything at or beyond the largest finite value,
 * infinities included, becomes +-448).  Written as a search over the 127
 * non-negative finite codes, which is the definition of nearest rounding. */
ORC_API uint8_t orc_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  int best = 0;
  double best_err = a;  /* distance to code 0 (value 0) */
  for (int c = 1; c <= 0x7E; ++c) {
    double err = fabs(a - orc_e4m3_decode((uint8_t)c));
    if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      best_err = err;
    }
  }
  return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------ */
/* Query quantisation for the FP8 indexer.  The pages give no precision; the */
/* reading taken here quantises each (row, head) query vector to E4M3       */
/* with a power-of-two scale 2^e and folds the scale into the head weight:   */
/* ReLU(c x) = c ReLU(x) for c > 0, so w' = w * 2^e keeps the score the same. */
/* ------------------------------------------------------------------------ */

/* Smallest integer e with amax <= 448 * 2^e; e = 0 when amax == 0. */
ORC_API int orc_q_exponent(double amax) {
  if (!(amax > 0.0)) return 0;
  int e = -300;
  while (amax > ldexp(448.0, e)) ++e;
  return e;
}

/* q: [rows][H][d] as doubles (exact widening of the bf16 / fp32 input),
 * w: [rows][H] fp32.  Outputs q8 codes [rows][H][d], w' [rows][H] fp32 and
 * the exponents e [rows][H]. */
ORC_API void orc_quantize_q(const double* q, const float* w, int rows, int H, int d,
                            uint8_t* q8, float* wq, int32_t* e_out) {
  for (int r = 0; r < rows; ++r) {
    for (int h = 0; h < H; ++h) {
      const double* v = q + ((int64_t)r * H + h) * d;
      double amax = 0.0;
      for (int i = 0; i < d; ++i) amax = fmax(amax, fabs(v[i]));
      int e = orc_q_exponent(amax);
      for (int i = 0; i < d; ++i)
        q8[((int64_t)r * H + h) * d + i] = orc_e4m3_encode(ldexp(v[i], -e));
      wq[r * H + h] = (float)ldexp((double)w[r * H + h], e);
      if (e_out) e_out[r * H + h] = e;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Positions.  ctx_len is the number of slots visible to row 0, whose own    */
/* key is already in the cache; row r (MTP verification rows) sits at        */
/* position p_r = ctx_len - 1 + r and sees slots 0..p_r.                     */
/* ------------------------------------------------------------------------ */
static int64_t pos_of_row(int64_t ctx_len, int r) { return ctx_len - 1 + r; }
static int64_t nblocks_of_row(int64_t ctx_len, int r, int b) {
  return (pos_of_row(ctx_len, r) + 1 + b - 1) / b;
}
ORC_API int64_t orc_num_blocks(int64_t ctx_len, int r, int b) {
  return nblocks_of_row(ctx_len, r, b);
}

/* Predicted slot score z_{t,i} = max(V_i, D_{t-i}) ([radio] "Title and
 * authors": "z sub t i equals max V i D ... t minus i"; [digest] arXiv深度剖析:
 * per-slot and per-relative-offset EMA states) and its block max-pool
 * S_{t,j} = max over slots i of logical block j of z_{t,i} ([radio] "Title
 * and authors": "max i: b(i)=j z sub t i"; b is the attention backend's block
 * size).  Only slots i <= p_r enter the pool (a partial last block pools its
 * valid slots).  S is [rows][n_stride]; entries j >= n_r are not written. */
ORC_API void orc_predict_pool(const float* V, const float* D, int64_t ctx_len, int rows,
                              int b, int64_t n_stride, float* S) {
  for (int r = 0; r < rows; ++r) {
    int64_t p = pos_of_row(ctx_len, r);
    int64_t n = nblocks_of_row(ctx_len, r, b);
    for (int64_t j = 0; j < n; ++j) {
      float best = -INFINITY;
      for (int64_t i = j * b; i < (j + 1) * b && i <= p; ++i) {
        float z = fmaxf(V[i], D[p - i]);
        if (z > best) best = z;
      }
      S[(int64_t)r * n_stride + j] = best;
    }
  }
}

/* Block-reduction variants of the pool ([listing] Figure 3: "Mean and Top-4
 * compared with Max pooling"; the pages do not define them, so these are the
 * plainest readings).  Over the block's visible slots of row r:
 *   Mean  = the mean of z: (sum of z) / count,
 *   Top-4 = the mean of the min(4, count) largest z,
 * each the exact value rounded once to the nearest float (ties to even), so
 * that no summation order enters the definition.  +inf (a never-observed
 * slot) makes the result +inf; -inf with no +inf makes it -inf; both, or a
 * NaN, make it NaN.  mode 0 is the max-pool above.
 *
 * The exact sum: every finite float is an integer multiple of 2^-149, and
 * |z| < 2^128, so a sum of at most 256 of them is an integer N (in units of
 * 2^-149) below 2^285.  N is held in ten base-2^32 digits, each digit kept in
 * an int64 so that signed digits and up to 2^31 additions need no carry until
 * the end. */
typedef struct {
  int64_t d[10];
} orc_exact_sum;

static void orc_exact_add(orc_exact_sum* a, float x) {
  if (x == 0.0f) return;
  int e;
  const double f = frexp((double)x, &e);      /* x = f 2^e, 0.5 <= |f| < 1 */
  int64_t m = (int64_t)ldexp(f, 24);           /* exact: a float has 24 bits */
  int shift = e - 24 + 149;                    /* x = m 2^(shift - 149) */
  if (shift < 0) {                             /* subnormal: the low bits of m are zero */
    m /= ((int64_t)1 << -shift);
    shift = 0;
  }
  const int k = shift / 32, off = shift % 32;
  const int neg = m < 0;
  const uint64_t mag = (uint64_t)(neg ? -m : m) << off;   /* < 2^56 */
  const int64_t lo = (int64_t)(mag & 0xFFFFFFFFu), hi = (int64_t)(mag >> 32);
  a->d[k] += neg ? -lo : lo;
  if (hi) a->d[k + 1] += neg ? -hi : hi;
}

/* The exact sum divided by cnt (1..256), rounded once to the nearest float. */
static float orc_exact_mean(const orc_exact_sum* a, int cnt) {
  int64_t d[11];
  for (int k = 0; k < 10; ++k) d[k] = a->d[k];
  d[10] = 0;
  for (int k = 0; k < 10; ++k) {               /* digits to [0, 2^32), the sign to the top */
    int64_t c = d[k] >> 32;                    /* floor division by 2^32 */
    d[k] -= c * ((int64_t)1 << 32);
    d[k + 1] += c;
  }
  int neg = d[10] < 0;
  if (neg) {                                   /* magnitude of a negative sum: -N */
    int64_t borrow = 0;
    for (int k = 0; k < 11; ++k) {
      int64_t v = -d[k] - borrow;
      borrow = 0;
      if (v < 0 && k < 10) { v += ((int64_t)1 << 32); borrow = 1; }
      d[k] = v;
    }
  }
  /* quotient and remainder of N / cnt, most significant digit first */
  uint64_t q[10];
  uint64_t rem = 0;
  for (int k = 9; k >= 0; --k) {
    const uint64_t cur = (rem << 32) | (uint64_t)d[k];
    q[k] = cur / (uint64_t)cnt;
    rem = cur % (uint64_t)cnt;
  }
  int top = -1;                                /* bit length of the quotient */
  for (int k = 9; k >= 0 && top < 0; --k)
    if (q[k]) {
      int b = 31;
      while (!((q[k] >> b) & 1u)) --b;
      top = 32 * k + b + 1;
    }
  if (top < 0) {                               /* below one unit: 0 or 2^-149 */
    float r = (2 * rem > (uint64_t)cnt) ? ldexpf(1.0f, -149) : 0.0f;
    return neg ? -r : r;
  }
  /* a float keeps 24 significant bits; below 2^24 units (the subnormals and
   * the lowest normal binade) its spacing is one unit */
  const int sh = top > 24 ? top - 24 : 0;
  uint64_t kept = 0;                           /* bits [sh, top) of the quotient */
  for (int bit = top - 1; bit >= sh; --bit) kept = (kept << 1) | ((q[bit / 32] >> (bit % 32)) & 1u);
  int up;
  if (sh == 0) {
    up = (2 * rem > (uint64_t)cnt) || (2 * rem == (uint64_t)cnt && (kept & 1u));
  } else {
    const int half = (int)((q[(sh - 1) / 32] >> ((sh - 1) % 32)) & 1u);
    int below = rem != 0;                      /* anything under the half bit */
    for (int bit = sh - 2; bit >= 0 && !below; --bit) below = (q[bit / 32] >> (bit % 32)) & 1u;
    up = half && (below || (kept & 1u));
  }
  const double v = ldexp((double)(kept + (uint64_t)up), sh - 149);   /* exact; a float */
  return neg ? -(float)v : (float)v;
}

static float orc_mean_of(const float* z, int cnt) {
  int pinf = 0, ninf = 0, nan = 0;
  orc_exact_sum a;
  memset(&a, 0, sizeof(a));
  for (int u = 0; u < cnt; ++u) {
    if (isnan(z[u])) nan = 1;
    else if (isinf(z[u])) { if (z[u] > 0) pinf = 1; else ninf = 1; }
    else orc_exact_add(&a, z[u]);
  }
  if (nan || (pinf && ninf)) return NAN;
  if (pinf) return INFINITY;
  if (ninf) return -INFINITY;
  return orc_exact_mean(&a, cnt);
}

ORC_API float orc_mean_exact(const float* z, int cnt) { return cnt >= 1 && cnt <= 256 ? orc_mean_of(z, cnt) : NAN; }

ORC_API void orc_predict_pool_mode(const float* V, const float* D, int64_t ctx_len, int rows, int b,
                                   int64_t n_stride, int mode, float* S) {
  if (mode == 0) {
    orc_predict_pool(V, D, ctx_len, rows, b, n_stride, S);
    return;
  }
  float z[256];  /* b <= 256 */
  for (int r = 0; r < rows; ++r) {
    int64_t p = pos_of_row(ctx_len, r);
    int64_t n = nblocks_of_row(ctx_len, r, b);
    for (int64_t j = 0; j < n; ++j) {
      int count = 0;
      for (int64_t i = j * b; i < (j + 1) * b && i <= p; ++i) z[count++] = fmaxf(V[i], D[p - i]);
      if (mode == 2) {
        /* the min(4, count) largest: a partial selection sort, descending */
        int m = count < 4 ? count : 4;
        for (int k = 0; k < m; ++k)
          for (int u = k + 1; u < count; ++u)
            if (z[u] > z[k]) { float t = z[k]; z[k] = z[u]; z[u] = t; }
        count = m;
      }
      S[(int64_t)r * n_stride + j] = orc_mean_of(z, count);
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Block selection.                                                          */
/* Budget: B = n - floor(s n) blocks for target block sparsity s ([listing]  */
/* Table 6 "Target block sparsity"); a share gamma of the same budget goes   */
/* to random exploration ([digest] arXiv深度剖析; [listing] Figure 4 "reserve */
/* 5% of the retained-block budget"; [radio] "The paper's summary"); the     */
/* rest is filled with the highest predicted blocks.  For several query rows */
/* (MTP verification) each row predicts with its own budget and the kept    */
/* mask is the union ([digest] arXiv深度剖析; [listing] Table 7 "Row-local    */
/* union").  s == 0 is the all-keep control: every visible block is kept and  */
/* labelled predicted.  Ties go to the lower block index.                    */
/* mask[j] = 1 predicted (in the union), 2 explored, 0 skipped, for          */
/* j < n_stride; blocks past the last row's visible range are 0.             */
/*                                                                          */
/* policy ORC_MTP_ROW0 is the baseline MTP policy of [listing] Table 7 and  */
/* Figure 2, "Row-0 sharing": row 0 alone predicts (its own budget, the    */
/* exploration share of that budget drawn among row 0's unkept blocks) and */
/* every row uses its mask.  Blocks past row 0's range hold only the new    */
/* keys of this step's draft tokens, which no step has scored yet; they are */
/* kept (labelled predicted) so that the draft rows see them.  With one row */
/* both policies are the same selection.                                    */
/* ------------------------------------------------------------------------ */
#define ORC_MTP_UNION_PREFIX 0
#define ORC_MTP_ROW0 1
typedef struct { float s; int64_t j; } orc_sj;
typedef struct { uint32_t key; int64_t j; } orc_kj;

static int cmp_score_desc(const void* a, const void* b) {
  const orc_sj* x = (const orc_sj*)a;
  const orc_sj* y = (const orc_sj*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);
}
static int cmp_key_asc(const void* a, const void* b) {
  const orc_kj* x = (const orc_kj*)a;
  const orc_kj* y = (const orc_kj*)b;
  if (x->key < y->key) return -1;
  if (x->key > y->key) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);
}

ORC_API int64_t orc_budget(int64_t n, double sparsity) {
  return n - (int64_t)floor(sparsity * (double)n);
}
ORC_API int64_t orc_explore_count(int64_t budget_row0, double gamma) {
  return (int64_t)floor(gamma * (double)budget_row0);
}

ORC_API void orc_select(const float* S, int64_t n_stride, int64_t ctx_len, int rows, int b,
                        float sparsity, float gamma, uint64_t seed, uint32_t request,
                        uint32_t layer, uint64_t step, int policy, uint8_t* mask) {
  int64_t n_last = nblocks_of_row(ctx_len, rows - 1, b);
  memset(mask, 0, (size_t)n_stride);
  if (sparsity == 0.0f) {
    for (int64_t j = 0; j < n_last; ++j) mask[j] = 1;
    return;
  }
  int64_t n0 = nblocks_of_row(ctx_len, 0, b);
  int64_t n_exp = orc_explore_count(orc_budget(n0, (double)sparsity), (double)gamma);
  int predicting_rows = policy == ORC_MTP_ROW0 ? 1 : rows;
  orc_sj* order = (orc_sj*)malloc(sizeof(orc_sj) * (size_t)n_last);
  for (int r = 0; r < predicting_rows; ++r) {
    int64_t n = nblocks_of_row(ctx_len, r, b);
    int64_t n_pred = orc_budget(n, (double)sparsity) - n_exp;
    for (int64_t j = 0; j < n; ++j) { order[j].s = S[(int64_t)r * n_stride + j]; order[j].j = j; }
    qsort(order, (size_t)n, sizeof(orc_sj), cmp_score_desc);
    for (int64_t t = 0; t < n_pred && t < n; ++t) mask[order[t].j] = 1;
  }
  free(order);
  if (policy == ORC_MTP_ROW0)
    for (int64_t j = n0; j < n_last; ++j) mask[j] = 1;  /* the drafts' own new keys */
  orc_kj* cand = (orc_kj*)malloc(sizeof(orc_kj) * (size_t)n_last);
  int64_t nc = 0;
  for (int64_t j = 0; j < n_last; ++j) {
    if (mask[j] == 0) {
      cand[nc].key = orc_explore_key(seed, (uint32_t)j, request, layer, step);
      cand[nc].j = j;
      ++nc;
    }
  }
  qsort(cand, (size_t)nc, sizeof(orc_kj), cmp_key_asc);
  for (int64_t t = 0; t < n_exp && t < nc; ++t) mask[cand[t].j] = 2;
  free(cand);
}

/* ------------------------------------------------------------------------ */
/* Indexer scores on the kept blocks only ([digest] arXiv深度剖析: the input */
/* of the indexer is pruned before it runs; [listing] Abstract).  Formula:   */
/* the DSA lightning indexer I_{r,s} = sum_h w_{r,h} ReLU(q_{r,h} . k_s).    */
/* Keys live in a paged cache [pages][b][d] addressed through the block      */
/* table (logical block j -> physical page); FP8 keys carry a per-token fp32 */
/* scale sigma_s, so k_s = sigma_s * decode(k8_s).  Evaluated in fp64.       */
/* scores is [rows][slot_stride]; only scored entries are written.           */
/* ------------------------------------------------------------------------ */
ORC_API void orc_score_fp8(const uint8_t* keys8, const float* kscale, const int32_t* block_table,
                           int b, int d, const uint8_t* q8, const float* wq, int H, int rows,
                           int64_t ctx_len, const uint8_t* mask, int64_t slot_stride,
                           double* scores) {
  double dec[256];
  for (int c = 0; c < 256; ++c) dec[c] = orc_e4m3_decode((uint8_t)c);
  int64_t n_last = nblocks_of_row(ctx_len, rows - 1, b);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t j = 0; j < n_last; ++j) {
    if (!mask[j]) continue;
    int64_t page = block_table[j];
    for (int t = 0; t < b; ++t) {
      int64_t s = j * b + t;
      const uint8_t* k = keys8 + (page * b + t) * (int64_t)d;
      double sigma = (double)kscale[page * b + t];
      for (int r = 0; r < rows; ++r) {
        if (s > pos_of_row(ctx_len, r)) continue;
        double acc = 0.0;
        for (int h = 0; h < H; ++h) {
          const uint8_t* qh = q8 + ((int64_t)r * H + h) * d;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += dec[qh[i]] * dec[k[i]];
          if (dot > 0.0) acc += (double)wq[r * H + h] * dot;
        }
        scores[(int64_t)r * slot_stride + s] = sigma * acc;
      }
    }
  }
}

/* Same formula with fp32 keys and queries (no scales, no quantisation). */
ORC_API void orc_score_f32(const float* keys, const int32_t* block_table, int b, int d,
                           const float* q, const float* w, int H, int rows, int64_t ctx_len,
                           const uint8_t* mask, int64_t slot_stride, double* scores) {
  int64_t n_last = nblocks_of_row(ctx_len, rows - 1, b);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t j = 0; j < n_last; ++j) {
    if (!mask[j]) continue;
    int64_t page = block_table[j];
    for (int t = 0; t < b; ++t) {
      int64_t s = j * b + t;
      const float* k = keys + (page * b + t) * (int64_t)d;
      for (int r = 0; r < rows; ++r) {
        if (s > pos_of_row(ctx_len, r)) continue;
        double acc = 0.0;
        for (int h = 0; h < H; ++h) {
          const float* qh = q + ((int64_t)r * H + h) * d;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += (double)qh[i] * (double)k[i];
          if (dot > 0.0) acc += (double)w[r * H + h] * dot;
        }
        scores[(int64_t)r * slot_stride + s] = acc;
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Token top-k.  The fixed top-k budget of core attention is unchanged by    */
/* SPIN ([digest] arXiv深度剖析); the top-k runs over the slots that were     */
/* scored (kept blocks, s <= p_r).  Order: higher score first, ties to the   */
/* lower slot; the chosen slots are emitted in ascending slot order and the  */
/* row is padded with -1 when fewer than k slots were scored.  Scores are    */
/* given as doubles (an fp32 score widens exactly, so comparisons match).     */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int64_t i; } orc_si;
static int cmp_si_desc(const void* a, const void* b) {
  const orc_si* x = (const orc_si*)a;
  const orc_si* y = (const orc_si*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->i < y->i) ? -1 : (x->i > y->i);
}
static int cmp_i64(const void* a, const void* b) {
  int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return (x < y) ? -1 : (x > y);
}

/* One row: scores_row is [slot_stride]. Returns the number of real entries. */
ORC_API int64_t orc_topk_row(const double* scores_row, const uint8_t* mask, int64_t ctx_len,
                             int row, int b, int k, int32_t* out) {
  int64_t p = pos_of_row(ctx_len, row);
  int64_t n = nblocks_of_row(ctx_len, row, b);
  orc_si* all = (orc_si*)malloc(sizeof(orc_si) * (size_t)(p + 1));
  int64_t m = 0;
  for (int64_t j = 0; j < n; ++j) {
    if (!mask[j]) continue;
    for (int64_t s = j * b; s < (j + 1) * b && s <= p; ++s) {
      all[m].s = scores_row[s];
      all[m].i = s;
      ++m;
    }
  }
  qsort(all, (size_t)m, sizeof(orc_si), cmp_si_desc);
  int64_t take = m < k ? m : k;
  int64_t* idx = (int64_t*)malloc(sizeof(int64_t) * (size_t)(take > 0 ? take : 1));
  for (int64_t t = 0; t < take; ++t) idx[t] = all[t].i;
  qsort(idx, (size_t)take, sizeof(int64_t), cmp_i64);
  for (int64_t t = 0; t < k; ++t) out[t] = t < take ? (int32_t)idx[t] : -1;
  free(idx);
  free(all);
  return take;
}

/* ------------------------------------------------------------------------ */
/* EMA update of the vertical (per slot) and diagonal (per relative offset)  */
/* states from the observed indexer scores ([digest] 核心概要, arXiv深度剖析; */
/* [radio] "The paper's summary").  Only slots that were scored are updated; */
/* skipped blocks get no update ([digest] arXiv深度剖析; [radio] "The paper's */
/* summary").  For MTP rows the update is deferred until the accepted length */
/* a is known and then replayed for the prefix-valid rows 0..a-1 in order    */
/* ([digest] arXiv深度剖析).                                                  */
/*   upd(x, y) = y                         if x is the never-observed sentinel */
/*             = fmaf(alpha, x, beta * y)  otherwise, beta = fl32(1 - alpha)   */
/* with sentinels V = +inf and D = -inf.  scores32 is [rows][slot_stride].    */
/* ------------------------------------------------------------------------ */
ORC_API float orc_ema_beta(float alpha) { return (float)(1.0 - (double)alpha); }

ORC_API void orc_ema_update(float* V, float* D, const float* scores32, const uint8_t* mask,
                            int64_t ctx_len, int accepted, int b, float alpha,
                            int64_t slot_stride) {
  float beta = orc_ema_beta(alpha);
  for (int r = 0; r < accepted; ++r) {
    int64_t p = pos_of_row(ctx_len, r);
    int64_t n = nblocks_of_row(ctx_len, r, b);
    for (int64_t j = 0; j < n; ++j) {
      if (!mask[j]) continue;
      for (int64_t s = j * b; s < (j + 1) * b && s <= p; ++s) {
        float y = scores32[(int64_t)r * slot_stride + s];
        float v = V[s];
        V[s] = (isinf(v) && v > 0) ? y : fmaf(alpha, v, beta * y);
        float dd = D[p - s];
        D[p - s] = (isinf(dd) && dd < 0) ? y : fmaf(alpha, dd, beta * y);
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Predictor quality ([listing] Table 1: Pearson correlation and top-k recall */
/* of an indexer prediction against the indexer's scores, for a random       */
/* baseline, the previous layer and the previous iteration).                 */
/*                                                                          */
/* orc_slot_prediction: the SPIN predictor before block pooling, z_{r,s} =   */
/* max(V_s, D_{p_r - s}) for s <= p_r ([radio] "Title and authors"), and     */
/* -inf where z is not finite: a slot no step has scored carries the +inf    */
/* sentinel and no prediction.  out is [rows][slot_stride]; slots past p_r   */
/* are not written.                                                          */
/* ------------------------------------------------------------------------ */
ORC_API void orc_slot_prediction(const float* V, const float* D, int64_t ctx_len, int rows,
                                 int64_t slot_stride, float* out) {
  for (int r = 0; r < rows; ++r) {
    int64_t p = pos_of_row(ctx_len, r);
    for (int64_t s = 0; s <= p; ++s) {
      float z = V[s] > D[p - s] ? V[s] : D[p - s];
      out[(int64_t)r * slot_stride + s] = isfinite(z) ? z : -INFINITY;
    }
  }
}

/* The random baseline: an independent uniform value per slot in [0, 1), the */
/* top 24 bits of the exploration key with the slot in place of the block    */
/* (word s mod 4 of Philox4x32-10 at counter (s div 4, request, layer, step  */
/* mod 2^32), key (seed low, seed high)) times 2^-24; the same for every row. */
ORC_API void orc_random_prediction(uint64_t seed, uint32_t request, uint32_t layer, uint64_t step,
                                   int64_t ctx_len, int rows, int64_t slot_stride, float* out) {
  for (int r = 0; r < rows; ++r) {
    int64_t p = pos_of_row(ctx_len, r);
    for (int64_t s = 0; s <= p; ++s) {
      uint32_t w = orc_explore_key(seed, (uint32_t)s, request, layer, step);
      out[(int64_t)r * slot_stride + s] = (float)((double)(w >> 8) / 16777216.0);
    }
  }
}

/* Pearson correlation of x and y over the entries where both are finite,   */
/* in double, two passes: the means, then the centred sums.  0 when fewer    */
/* than two pairs remain or either side is constant on them.                 */
ORC_API double orc_pearson(const float* x, const float* y, int64_t n) {
  int64_t m = 0;
  double sx = 0.0, sy = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    if (!isfinite(x[i]) || !isfinite(y[i])) continue;
    sx += (double)x[i];
    sy += (double)y[i];
    ++m;
  }
  if (m < 2) return 0.0;
  double mx = sx / (double)m, my = sy / (double)m;
  double sxy = 0.0, sxx = 0.0, syy = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    if (!isfinite(x[i]) || !isfinite(y[i])) continue;
    double dx = (double)x[i] - mx, dy = (double)y[i] - my;
    sxy += dx * dy;
    sxx += dx * dx;
    syy += dy * dy;
  }
  if (sxx == 0.0 || syy == 0.0) return 0.0;
  return sxy / sqrt(sxx * syy);
}

/* ------------------------------------------------------------------------ */
/* Fidelity metric: the fraction of the full indexer's top-k tokens that     */
/* fall in skipped blocks ([listing] Table 5 caption: mean / p99 miss over   */
/* eligible sparse decode rows).  full_topk holds k slots padded with -1.    */
/* ------------------------------------------------------------------------ */
ORC_API double orc_miss_fraction(const int32_t* full_topk, int k, const uint8_t* mask, int b) {
  int64_t total = 0, missed = 0;
  for (int t = 0; t < k; ++t) {
    if (full_topk[t] < 0) continue;
    ++total;
    if (!mask[full_topk[t] / b]) ++missed;
  }
  return total ? (double)missed / (double)total : 0.0;
}

/* ------------------------------------------------------------------------ */
/* Per-layer block budget ([v3] abstract: the block budget is spread across  */
/* layers by their measured miss rates).  The reading taken here: kept      */
/* fractions f_l = clamp(c * (m_l + 1e-3), lo_l, 1), with c chosen so that  */
/* sum_l f_l N_l = (1 - s_glob) sum_l N_l; found by bisection on c.  When   */
/* even the lower bounds exceed the global budget, f_l = lo_l.  Returns the */
/* per-layer sparsities s_l = 1 - f_l.                                       */
/* ------------------------------------------------------------------------ */
static double kept_total(double c, const double* m, const double* N, const double* lo, int L) {
  double t = 0.0;
  for (int l = 0; l < L; ++l) {
    double f = c * (m[l] + 1e-3);
    if (f < lo[l]) f = lo[l];
    if (f > 1.0) f = 1.0;
    t += f * N[l];
  }
  return t;
}

ORC_API void orc_layer_sparsity(const double* miss, const double* N, const double* lo, int L,
                                double s_glob, double* s_out) {
  double total = 0.0;
  for (int l = 0; l < L; ++l) total += N[l];
  double target = (1.0 - s_glob) * total;
  if (kept_total(0.0, miss, N, lo, L) >= target) {
    for (int l = 0; l < L; ++l) s_out[l] = 1.0 - lo[l];
    return;
  }
  double c_lo = 0.0, c_hi = 1.0;
  while (kept_total(c_hi, miss, N, lo, L) < target && c_hi < 1e30) c_hi *= 2.0;
  for (int it = 0; it < 200; ++it) {
    double c = 0.5 * (c_lo + c_hi);
    if (kept_total(c, miss, N, lo, L) < target) c_lo = c; else c_hi = c;
  }
  for (int l = 0; l < L; ++l) {
    double f = c_hi * (miss[l] + 1e-3);
    if (f < lo[l]) f = lo[l];
    if (f > 1.0) f = 1.0;
    s_out[l] = 1.0 - f;
  }
}
