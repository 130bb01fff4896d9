/*
 * MLA attention oracle: plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do. It shares no code, header or table with the CUDA library.
 *
 * What it computes (one query row = one (token t, head h) pair):
 *
 *   s_j  = scale * sum_{c<576} q[t,h,c] * k[j,c]  +  mask[t,j]
 *   M    = max_j s_j
 *   p_j  = exp(s_j - M)
 *   L    = sum_j p_j
 *   o[d] = sum_j p_j * k[j,d] / L              for d < 512
 *   lse  = M + log(L)                          (oracle_attention_lse)
 *
 * Sources (web pages on MLA flash attention):
 *  - Cache row = 512-wide latent followed by the 64-wide RoPE key, 576 in
 *    all, one row per token shared by every head: ik_llama.cpp -mla guide,
 *    section "MLA 是什麼" (kv_lora_rank + n_embd_head_qk_rope = 576).
 *  - No V cache: with flash attention only the K cache exists and V is
 *    derived from it; taken here as V = the first 512 columns of the row:
 *    ik_llama.cpp -mla guide, section "-mla四檔語義".
 *  - Tiled online softmax with a running maximum m and a running sum l,
 *    rescaling the accumulated output when m grows: Vulkan FA for DeepSeek
 *    MLA article, section 2.2; computed by oracle_attention_online below.
 *  - f16 additive mask: baguaai flash-attention tag page, item on PR #23764.
 *  - Ascending index compaction of the kept mask cells: llama.cpp b11413
 *    release note, item "single-scan sparse FA index compaction".
 *  - Attention sinks, ALiBi and logit softcap (oracle_attention_variants), named for
 *    the Metal FA kernel in the llama.cpp tag page (PR #29570); their formulas are
 *    this file's readings, written next to the function.
 *  - Value up-projection of each head (oracle_project): wkv_b split per head into
 *    wk_b and wv_b, "128 x 512 x 128": ik_llama.cpp -mla guide, section on tensor
 *    derivation; p[n] = sum_d o[d] * wv[h][d][n].
 *
 * Readings where the pages are silent:
 *  - The mask is added after scaling and is not scaled itself.
 *  - A row whose every score is -inf (nothing kept) yields o = 0.
 *  - A mask cell is "dropped" iff its f16 bit pattern is -inf (0xFC00).
 *  - q8_0 row = 18 blocks of {f16 d; int8 q[32]} (34 bytes), 612 bytes per
 *    row; value = d * q, exact in double.
 *
 * Head width: the cache row and the query are dk wide, 576 above; the
 * DK = DV = 512 shape (one of the head shapes the llama.cpp tag page lists for the
 * Metal FA kernel, PR #29570) takes dk = 512 with the same V = first 512 columns,
 * i.e. the whole row (oracle_attention_dk, f16 cache only).
 *
 * Everything is fp64: each f16 input is converted exactly to double
 * (-inf stays -inf, exp(-inf) = 0); results are returned as double and
 * rounded to fp32 once by the caller.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_DK 576
#define ORC_DV 512
#define ORC_Q8_BLOCK 32
#define ORC_Q8_BLOCK_BYTES 34
#define ORC_Q8_ROW_BYTES 612

enum { ORC_KV_F16 = 0, ORC_KV_Q8_0 = 1 };

/* Exact IEEE binary16 -> double, from the format's definition:
 * normal  (1024 + mant) * 2^(exp - 25), subnormal mant * 2^-24. */
static double half_to_double_exact(uint16_t h) {
  int sign = h >> 15;
  int ex = (h >> 10) & 0x1f;
  int mant = h & 0x3ff;
  double v;
  if (ex == 0)
    v = ldexp((double)mant, -24);
  else if (ex == 31)
    v = mant ? NAN : INFINITY;
  else
    v = ldexp((double)(mant | 0x400), ex - 25);
  return sign ? -v : v;
}

static double g_half[65536];
static int g_ready = 0;

void oracle_init(void) {
  if (g_ready) return;
  for (int i = 0; i < 65536; ++i) g_half[i] = half_to_double_exact((uint16_t)i);
  g_ready = 1;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

double oracle_half_to_double(uint16_t h) {
  oracle_init();
  return g_half[h];
}

/* Value of column c of cache row `key` (f16 rows are dk wide). */
static inline double kval_w(const void* kc, int kv_type, long key, int c, int dk) {
  if (kv_type == ORC_KV_F16) {
    const uint16_t* k = (const uint16_t*)kc;
    return g_half[k[key * dk + c]];
  } else {
    const uint8_t* row = (const uint8_t*)kc + key * ORC_Q8_ROW_BYTES;
    const uint8_t* blk = row + (c / ORC_Q8_BLOCK) * ORC_Q8_BLOCK_BYTES;
    uint16_t dbits;
    memcpy(&dbits, blk, 2);
    int8_t qv = (int8_t)blk[2 + (c % ORC_Q8_BLOCK)];
    return g_half[dbits] * (double)qv;
  }
}
static inline double kval(const void* kc, int kv_type, long key, int c) {
  return kval_w(kc, kv_type, key, c, ORC_DK);
}

void oracle_dequant_q8_0(const uint8_t* rows, long n_rows, double* out) {
  oracle_init();
  for (long r = 0; r < n_rows; ++r)
    for (int c = 0; c < ORC_DK; ++c) out[r * ORC_DK + c] = kval(rows, ORC_KV_Q8_0, r, c);
}

/* Score of key `key` for query row q (576 doubles). */
static inline double score_w(const double* q, const void* kc, int kv_type, long key,
                             const uint16_t* mrow, double scale, int dk) {
  double dot = 0.0;
  for (int c = 0; c < dk; ++c) dot += q[c] * kval_w(kc, kv_type, key, c, dk);
  double s = scale * dot;
  if (mrow) s += g_half[mrow[key]];
  return s;
}
static inline double score(const double* q, const void* kc, int kv_type, long key,
                           const uint16_t* mrow, double scale) {
  return score_w(q, kc, kv_type, key, mrow, scale, ORC_DK);
}

/* Selected keys: all of 0..n_kv-1 when idx == NULL, else idx[0..n_sel). */
static inline long key_at(const int32_t* idx, long i) { return idx ? (long)idx[i] : i; }

/* Two-pass softmax-weighted sum for one query row; with lse != NULL also the
 * row's natural log-sum-exp of the scores, M + log(L) (-inf when every cell is
 * masked). */
static void attend_two_pass(const double* q, const void* kc, int kv_type, const uint16_t* mrow,
                            const int32_t* idx, long n_sel, double scale, double* s,
                            double* out, double* lse, int dk) {
  double M = -INFINITY;
  for (long i = 0; i < n_sel; ++i) {
    s[i] = score_w(q, kc, kv_type, key_at(idx, i), mrow, scale, dk);
    if (s[i] > M) M = s[i];
  }
  for (int d = 0; d < ORC_DV; ++d) out[d] = 0.0;
  if (lse) *lse = -INFINITY;
  if (M == -INFINITY) return; /* every cell masked: o = 0 */
  double L = 0.0;
  for (long i = 0; i < n_sel; ++i) {
    double p = exp(s[i] - M);
    L += p;
    if (p == 0.0) continue;
    long key = key_at(idx, i);
    for (int d = 0; d < ORC_DV; ++d) out[d] += p * kval_w(kc, kv_type, key, d, dk);
  }
  for (int d = 0; d < ORC_DV; ++d) out[d] /= L;
  if (lse) *lse = M + log(L);
}

/* One-pass tiled online softmax for one query row: running max m and running
 * sum l over tiles of `tile` keys; the accumulator is rescaled by exp(m-m')
 * whenever the maximum grows. */
static void attend_online(const double* q, const void* kc, int kv_type, const uint16_t* mrow,
                          const int32_t* idx, long n_sel, double scale, long tile, double* s,
                          double* out) {
  double m = -INFINITY, l = 0.0;
  double acc[ORC_DV];
  for (int d = 0; d < ORC_DV; ++d) acc[d] = 0.0;
  for (long t0 = 0; t0 < n_sel; t0 += tile) {
    long t1 = t0 + tile < n_sel ? t0 + tile : n_sel;
    double mt = -INFINITY;
    for (long i = t0; i < t1; ++i) {
      s[i - t0] = score(q, kc, kv_type, key_at(idx, i), mrow, scale);
      if (s[i - t0] > mt) mt = s[i - t0];
    }
    double m_new = mt > m ? mt : m;
    if (m_new == -INFINITY) continue; /* nothing kept so far */
    double alpha = exp(m - m_new);    /* exp(-inf) = 0 on the first kept tile */
    l *= alpha;
    for (int d = 0; d < ORC_DV; ++d) acc[d] *= alpha;
    for (long i = t0; i < t1; ++i) {
      double p = exp(s[i - t0] - m_new);
      l += p;
      if (p == 0.0) continue;
      long key = key_at(idx, i);
      for (int d = 0; d < ORC_DV; ++d) acc[d] += p * kval(kc, kv_type, key, d);
    }
    m = m_new;
  }
  for (int d = 0; d < ORC_DV; ++d) out[d] = l > 0.0 ? acc[d] / l : 0.0;
}

/* Split the selected keys into contiguous parts [bounds[i], bounds[i+1]), take
 * per-part (acc_s, m_s, l_s) and merge them with
 *   O = sum_s e^{m_s - M} acc_s / sum_s e^{m_s - M} l_s,   M = max_s m_s,
 * ignoring parts with l_s = 0. */
static void attend_split(const double* q, const void* kc, int kv_type, const uint16_t* mrow,
                         const int32_t* idx, long n_sel, double scale, const int32_t* bounds,
                         int n_split, double* s, double* out) {
  double* acc = (double*)calloc((size_t)n_split * ORC_DV, sizeof(double));
  double* ms = (double*)malloc(sizeof(double) * n_split);
  double* ls = (double*)malloc(sizeof(double) * n_split);
  for (int sp = 0; sp < n_split; ++sp) {
    long a = bounds[sp], b = bounds[sp + 1];
    if (a < 0) a = 0;
    if (b > n_sel) b = n_sel;
    double m = -INFINITY;
    for (long i = a; i < b; ++i) {
      s[i - a] = score(q, kc, kv_type, key_at(idx, i), mrow, scale);
      if (s[i - a] > m) m = s[i - a];
    }
    ms[sp] = m;
    ls[sp] = 0.0;
    if (m == -INFINITY) continue;
    for (long i = a; i < b; ++i) {
      double p = exp(s[i - a] - m);
      ls[sp] += p;
      long key = key_at(idx, i);
      for (int d = 0; d < ORC_DV; ++d) acc[(size_t)sp * ORC_DV + d] += p * kval(kc, kv_type, key, d);
    }
  }
  double M = -INFINITY;
  for (int sp = 0; sp < n_split; ++sp)
    if (ls[sp] > 0.0 && ms[sp] > M) M = ms[sp];
  for (int d = 0; d < ORC_DV; ++d) out[d] = 0.0;
  if (M != -INFINITY) {
    double den = 0.0;
    for (int sp = 0; sp < n_split; ++sp) {
      if (ls[sp] == 0.0) continue;
      double w = exp(ms[sp] - M);
      den += w * ls[sp];
      for (int d = 0; d < ORC_DV; ++d) out[d] += w * acc[(size_t)sp * ORC_DV + d];
    }
    for (int d = 0; d < ORC_DV; ++d) out[d] /= den;
  }
  free(acc);
  free(ms);
  free(ls);
}

enum { MODE_TWO_PASS = 0, MODE_ONLINE = 1, MODE_SPLIT = 2 };

/* Driver shared by the three entry points.
 * q      : f16 bits [n_q][n_head][576]
 * kcache : f16 bits [n_kv][576] (kv_type 0) or q8_0 bytes [n_kv][612] (kv_type 1)
 * mask   : f16 bits [n_q][n_kv], or NULL for no mask
 * idx    : NULL for all keys, else n_idx ascending cache rows (sparse)
 * rows   : NULL for every (t, h) in order, else n_rows row ids t*n_head + h
 * out    : double [n_rows or n_q*n_head][512]
 * lse    : NULL, or double [n_rows or n_q*n_head] (two-pass mode only)
 * Returns 0, or -1 on a bad argument. */
static int run(int mode, const uint16_t* q, const void* kcache, int kv_type, const uint16_t* mask,
               const int32_t* idx, long n_idx, int n_q, int n_head, long n_kv, double scale,
               const int32_t* rows, long n_rows, long tile, const int32_t* bounds, int n_split,
               double* out, double* lse, int dk) {
  if (!q || !kcache || !out || n_q < 1 || n_head < 1 || n_kv < 1) return -1;
  if (kv_type != ORC_KV_F16 && kv_type != ORC_KV_Q8_0) return -1;
  if (dk != ORC_DK && (dk != ORC_DV || kv_type != ORC_KV_F16 || mode != MODE_TWO_PASS)) return -1;
  if (idx) {
    for (long i = 0; i < n_idx; ++i)
      if (idx[i] < 0 || idx[i] >= n_kv) return -1;
  }
  oracle_init();
  long n_sel = idx ? n_idx : n_kv;
  long total = rows ? n_rows : (long)n_q * n_head;
  int bad = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n_sel > 0 ? n_sel : 1));
    double qd[ORC_DK];
#pragma omp for schedule(dynamic, 1)
    for (long r = 0; r < total; ++r) {
      long row = rows ? rows[r] : r;
      if (row < 0 || row >= (long)n_q * n_head) {
        bad = 1;
        continue;
      }
      long t = row / n_head;
      const uint16_t* qrow = q + row * dk;
      for (int c = 0; c < dk; ++c) qd[c] = g_half[qrow[c]];
      const uint16_t* mrow = mask ? mask + t * n_kv : NULL;
      double* o = out + r * ORC_DV;
      if (mode == MODE_TWO_PASS)
        attend_two_pass(qd, kcache, kv_type, mrow, idx, n_sel, scale, s, o, lse ? lse + r : NULL, dk);
      else if (mode == MODE_ONLINE)
        attend_online(qd, kcache, kv_type, mrow, idx, n_sel, scale, tile, s, o);
      else
        attend_split(qd, kcache, kv_type, mrow, idx, n_sel, scale, bounds, n_split, s, o);
    }
    free(s);
  }
  return bad ? -1 : 0;
}

int oracle_attention(const uint16_t* q, const void* kcache, int kv_type, const uint16_t* mask,
                     const int32_t* idx, long n_idx, int n_q, int n_head, long n_kv, double scale,
                     const int32_t* rows, long n_rows, double* out) {
  return run(MODE_TWO_PASS, q, kcache, kv_type, mask, idx, n_idx, n_q, n_head, n_kv, scale, rows,
             n_rows, 0, NULL, 0, out, NULL, ORC_DK);
}

/* Two-pass attention with the head width dk (576, or 512 for the DK = DV = 512
 * shape, f16 cache only): q [n_q][n_head][dk], kcache [n_kv][dk], V = the first 512
 * columns. lse may be NULL. */
int oracle_attention_dk(const uint16_t* q, const void* kcache, const uint16_t* mask,
                        const int32_t* idx, long n_idx, int n_q, int n_head, long n_kv, int dk,
                        double scale, const int32_t* rows, long n_rows, double* out, double* lse) {
  return run(MODE_TWO_PASS, q, kcache, ORC_KV_F16, mask, idx, n_idx, n_q, n_head, n_kv, scale,
             rows, n_rows, 0, NULL, 0, out, lse, dk);
}

/* oracle_attention plus each row's natural log-sum-exp of its scores. */
int oracle_attention_lse(const uint16_t* q, const void* kcache, int kv_type, const uint16_t* mask,
                         const int32_t* idx, long n_idx, int n_q, int n_head, long n_kv,
                         double scale, const int32_t* rows, long n_rows, double* out,
                         double* lse) {
  if (!lse) return -1;
  return run(MODE_TWO_PASS, q, kcache, kv_type, mask, idx, n_idx, n_q, n_head, n_kv, scale, rows,
             n_rows, 0, NULL, 0, out, lse, ORC_DK);
}

int oracle_attention_online(const uint16_t* q, const void* kcache, int kv_type,
                            const uint16_t* mask, const int32_t* idx, long n_idx, int n_q,
                            int n_head, long n_kv, double scale, const int32_t* rows, long n_rows,
                            long tile, double* out) {
  if (tile < 1) return -1;
  return run(MODE_ONLINE, q, kcache, kv_type, mask, idx, n_idx, n_q, n_head, n_kv, scale, rows,
             n_rows, tile, NULL, 0, out, NULL, ORC_DK);
}

int oracle_attention_split(const uint16_t* q, const void* kcache, int kv_type,
                           const uint16_t* mask, const int32_t* idx, long n_idx, int n_q,
                           int n_head, long n_kv, double scale, const int32_t* rows, long n_rows,
                           const int32_t* bounds, int n_split, double* out) {
  long n_sel = idx ? n_idx : n_kv;
  if (!bounds || n_split < 1 || bounds[0] != 0 || bounds[n_split] != n_sel) return -1;
  for (int i = 0; i < n_split; ++i)
    if (bounds[i + 1] < bounds[i]) return -1;
  return run(MODE_SPLIT, q, kcache, kv_type, mask, idx, n_idx, n_q, n_head, n_kv, scale, rows,
             n_rows, 0, bounds, n_split, out, NULL, ORC_DK);
}

/* Keep rule: a cell is kept iff its f16 bits are not -inf (0xFC00).
 * Writes the kept cell indices in ascending order; returns their count. */
long oracle_compact(const uint16_t* mask_row, long n_kv, int32_t* idx_out) {
  long n = 0;
  for (long j = 0; j < n_kv; ++j)
    if (mask_row[j] != 0xFC00u) idx_out[n++] = (int32_t)j;
  return n;
}

/* Value up-projection W_UV of each head (ik_llama.cpp -mla guide, section on tensor
 * derivation: wkv_b is split per head into wk_b and wv_b, "128 x 512 x 128"), applied
 * to attention rows:
 *   p[r][n] = sum_{d<512} o[r][d] * wv[h(r)][d][n],   n < proj_dim
 * o      : double [n_rows][512] (attention rows, e.g. from oracle_attention)
 * heads  : int32 [n_rows], the head h(r) of each row, in [0, n_head)
 * wv     : f16 bits [n_head][512][proj_dim]
 * out    : double [n_rows][proj_dim]
 * Returns 0, or -1 on a bad argument. */
int oracle_project(const double* o, const int32_t* heads, long n_rows, const uint16_t* wv,
                   int n_head, int proj_dim, double* out) {
  if (!o || !heads || !wv || !out || n_rows < 0 || n_head < 1 || proj_dim < 1) return -1;
  for (long r = 0; r < n_rows; ++r)
    if (heads[r] < 0 || heads[r] >= n_head) return -1;
  oracle_init();
#pragma omp parallel for schedule(static)
  for (long r = 0; r < n_rows; ++r) {
    const uint16_t* w = wv + (long)heads[r] * ORC_DV * proj_dim;
    for (int n = 0; n < proj_dim; ++n) {
      double acc = 0.0;
      for (int d = 0; d < ORC_DV; ++d) acc += o[r * ORC_DV + d] * g_half[w[(long)d * proj_dim + n]];
      out[r * proj_dim + n] = acc;
    }
  }
  return 0;
}

/* Variants on the same attention (Metal FA kernel of the llama.cpp tag page, PR
 * #29570: attention sinks, ALiBi, logit softcap), written out as definitions.
 * For query row (t, h) and selected cache position j:
 *   s_j = scale * sum_c q[t,h,c] k[j,c]
 *   s_j = softcap * tanh(s_j / softcap)                 if softcap > 0
 *   s_j = s_j + mask[t, j] + slopes[h] * (j - (pos0 + t))  (slopes optional)
 *   M   = max(max_j s_j, sinks[h])                       (sinks optional)
 *   L   = sum_j exp(s_j - M) + exp(sinks[h] - M)
 *   o   = sum_j exp(s_j - M) k[j, :512] / L,  0 when M = -inf
 * q: f16 bits [n_q][n_head][576]; slopes, sinks: double [n_head] or NULL;
 * out: double [n_q*n_head][512]. Returns 0, or -1 on a bad argument. */
int oracle_attention_variants(const uint16_t* q, const void* kcache, int kv_type,
                              const uint16_t* mask, const int32_t* idx, long n_idx, int n_q,
                              int n_head, long n_kv, double scale, double softcap,
                              const double* slopes, long pos0, const double* sinks, double* out) {
  if (!q || !kcache || !out || n_q < 1 || n_head < 1 || n_kv < 1) return -1;
  if (kv_type != ORC_KV_F16 && kv_type != ORC_KV_Q8_0) return -1;
  if (softcap < 0.0) return -1;
  if (idx) {
    for (long i = 0; i < n_idx; ++i)
      if (idx[i] < 0 || idx[i] >= n_kv) return -1;
  }
  oracle_init();
  const long n_sel = idx ? n_idx : n_kv;
  const long total = (long)n_q * n_head;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n_sel > 0 ? n_sel : 1));
    double qd[ORC_DK];
#pragma omp for schedule(dynamic, 1)
    for (long row = 0; row < total; ++row) {
      const long t = row / n_head, h = row % n_head;
      const uint16_t* qrow = q + row * ORC_DK;
      for (int c = 0; c < ORC_DK; ++c) qd[c] = g_half[qrow[c]];
      const uint16_t* mrow = mask ? mask + t * n_kv : NULL;
      double* o = out + row * ORC_DV;
      double M = sinks ? sinks[h] : -INFINITY;
      for (long i = 0; i < n_sel; ++i) {
        const long key = key_at(idx, i);
        double dot = 0.0;
        for (int c = 0; c < ORC_DK; ++c) dot += qd[c] * kval(kcache, kv_type, key, c);
        double v = scale * dot;
        if (softcap > 0.0) v = softcap * tanh(v / softcap);
        if (mrow) v += g_half[mrow[key]];
        if (slopes) v += slopes[h] * (double)(key - (pos0 + t));
        s[i] = v;
        if (v > M) M = v;
      }
      for (int d = 0; d < ORC_DV; ++d) o[d] = 0.0;
      if (M == -INFINITY) continue;
      double L = sinks ? exp(sinks[h] - M) : 0.0;
      for (long i = 0; i < n_sel; ++i) {
        const double p = exp(s[i] - M);
        L += p;
        if (p == 0.0) continue;
        const long key = key_at(idx, i);
        for (int d = 0; d < ORC_DV; ++d) o[d] += p * kval(kcache, kv_type, key, d);
      }
      for (int d = 0; d < ORC_DV; ++d) o[d] /= L;
    }
    free(s);
  }
  return 0;
}
