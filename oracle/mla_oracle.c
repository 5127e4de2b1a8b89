/*
 * fp64 CPU oracle for paged MLA decoding.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code:
 * only the tests, the smoke check and the benchmark's CPU-baseline / reference
 * arm use it.  It shares no code, header or table with the CUDA path.
 *
 * What it computes is the plain definition of the attention that FlashMLA
 * decodes, written out with no blocking, no online softmax and no splitting:
 *
 *   FlashMLA overview (deepseek.csdn.net), section 2.2 "DeepSeek-V3 MLA":
 *     o_{t,i} = sum_{j<=t} Softmax_j( q_{t,i}^T k_{j,i} / sqrt(d_h + d_h^R) ) v^C_{j,i}
 *   and, in the same section, only c^KV_t and k^R_t are cached; with the
 *   up-projections absorbed into q ("matrix absorption"), one cached row
 *   [c^KV (512) ; k^R (64)] serves as the 576-wide key of every query head and
 *   its first 512 entries serve as the value.
 *
 *   Paged cache, same article section 4.2(1): logical 64-token blocks map to
 *   physical blocks through block_table.
 *
 * Readings where the pages leave a step open:
 *   - query token i of s_q (0-based) sees cached tokens j <= L - s_q + i when
 *     causal, all j < L otherwise (the sum over j <= t, with the new tokens
 *     being the last s_q of the sequence);
 *   - the softmax scale is an argument (1/sqrt(192) = 1/sqrt(128+64) in all
 *     configurations);
 *   - lse is the natural log of sum_j exp(scaled score_j);
 *   - a row that sees no token gets o = 0 and lse = -inf (log of an empty sum);
 *   - query head h reads KV head h / (h_q / h_kv).
 *
 * bf16 inputs are given as 16-bit patterns and widened to double exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Address of cached row (token j of sequence b, KV head g). */
static const uint16_t* kv_row(const uint16_t* kv, const int32_t* block_table, int max_pages,
                              int b, int j, int g, int h_kv, int d, int page_size) {
  int page = block_table[(size_t)b * max_pages + j / page_size];
  size_t row = ((size_t)page * page_size + (size_t)(j % page_size)) * (size_t)h_kv + (size_t)g;
  return kv + row * (size_t)d;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Decode attention for every (sequence b, query token i, query head h).
 *
 *   q            [batch][s_q][h_q][d]          bf16 bits
 *   kv           [num_pages][page][h_kv][d]    bf16 bits
 *   block_table  [batch][max_pages]            int32
 *   seqlens      [batch]                       int32
 *   key_lo/key_hi  optional per-sequence window [lo, hi) of key positions
 *                  (NULL: the whole sequence); used to form partial results.
 *   o            [batch][s_q][h_q][dv]         fp64 out
 *   lse          [batch][h_q][s_q]             fp64 out
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_mla_decode(const uint16_t* q, const uint16_t* kv, const int32_t* block_table,
                      const int32_t* seqlens, const int32_t* key_lo, const int32_t* key_hi,
                      int batch, int s_q, int h_q, int h_kv, int d, int dv, int page_size,
                      int max_pages, int causal, double softmax_scale, double* o, double* lse,
                      int nthreads) {
  if (batch < 0 || s_q < 1 || h_q < 1 || h_kv < 1 || h_q % h_kv != 0 || dv > d || page_size < 1)
    return -1;
  const int heads_per_kv = h_q / h_kv;
  const long long rows = (long long)batch * s_q * h_q;
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
#endif
  for (long long rix = 0; rix < rows; ++rix) {
    const int h = (int)(rix % h_q);
    const int i = (int)((rix / h_q) % s_q);
    const int b = (int)(rix / ((long long)h_q * s_q));
    const int g = h / heads_per_kv;
    const int L = seqlens[b];
    /* last visible key index (inclusive) */
    int last = causal ? L - s_q + i : L - 1;
    int first = 0;
    if (key_lo) first = key_lo[b] > first ? key_lo[b] : first;
    if (key_hi && key_hi[b] - 1 < last) last = key_hi[b] - 1;
    double* orow = o + (size_t)rix * dv;
    double* lse_out = lse + ((size_t)b * h_q + h) * s_q + i;
    for (int c = 0; c < dv; ++c) orow[c] = 0.0;
    if (last < first) {
      *lse_out = -INFINITY;
      continue;
    }
    const int n = last - first + 1;
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    if (!s) {
      failed |= 1;
      continue;
    }
    const uint16_t* qrow = q + (size_t)rix * d;
    /* scaled scores */
    double m = -INFINITY;
    for (int j = first; j <= last; ++j) {
      const uint16_t* krow = kv_row(kv, block_table, max_pages, b, j, g, h_kv, d, page_size);
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += bf16_to_double(qrow[c]) * bf16_to_double(krow[c]);
      s[j - first] = softmax_scale * acc;
      if (s[j - first] > m) m = s[j - first];
    }
    /* softmax normaliser, log-sum-exp */
    double z = 0.0;
    for (int t = 0; t < n; ++t) z += exp(s[t] - m);
    *lse_out = m + log(z);
    /* weighted sum of the value rows (first dv entries of each cached row) */
    for (int j = first; j <= last; ++j) {
      const double w = exp(s[j - first] - m) / z;
      const uint16_t* vrow = kv_row(kv, block_table, max_pages, b, j, g, h_kv, d, page_size);
      for (int c = 0; c < dv; ++c) orow[c] += w * bf16_to_double(vrow[c]);
    }
    free(s);
  }
  return failed ? -1 : 0;
}

/*
 * Merge n partial results of one query row that cover disjoint key ranges
 * (the "combine of split results" the FlashMLA article names, section 4.2(1)):
 *   lse = log sum_k exp(lse_k),  o = sum_k exp(lse_k - lse) o_k.
 * Partials with lse_k = -inf (empty ranges) contribute nothing; if all are
 * empty the result is o = 0, lse = -inf.
 *   part_o [n][dv], part_lse [n]  ->  o [dv], *lse
 */
void oracle_mla_combine(const double* part_o, const double* part_lse, int n, int dv, double* o,
                        double* lse) {
  double m = -INFINITY;
  for (int k = 0; k < n; ++k)
    if (part_lse[k] > m) m = part_lse[k];
  for (int c = 0; c < dv; ++c) o[c] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  double z = 0.0;
  for (int k = 0; k < n; ++k) z += exp(part_lse[k] - m);
  const double total = m + log(z);
  for (int k = 0; k < n; ++k) {
    const double w = exp(part_lse[k] - total);
    for (int c = 0; c < dv; ++c) o[c] += w * part_o[(size_t)k * dv + c];
  }
  *lse = total;
}

/*
 * Appending new tokens to the paged cache (the write side of the same paged
 * layout, FlashMLA overview section 4.2(1): logical 64-token blocks mapped to
 * physical blocks by block_table).  Token t (0-based) of the s_new new tokens
 * of sequence b sits at position L_b + t of that sequence, i.e. in physical
 * page block_table[b][(L_b + t) / page_size], slot (L_b + t) % page_size, and
 * its row [c^KV ; k^R] for KV head g is copied there unchanged.
 *
 * A row whose position lies beyond the block table (>= max_pages*page_size)
 * or whose page id is outside [0, num_pages) is not written; the function then
 * returns -1 (0 when every row was written).
 */
int oracle_append_kvcache(const uint16_t* new_kv, const int32_t* block_table,
                          const int32_t* seqlens, int batch, int s_new, int h_kv, int d,
                          int page_size, int max_pages, int num_pages, uint16_t* kvcache) {
  int bad = 0;
  for (int b = 0; b < batch; ++b) {
    const int L = seqlens[b] > 0 ? seqlens[b] : 0;
    for (int t = 0; t < s_new; ++t) {
      const long long pos = (long long)L + t;
      if (pos >= (long long)max_pages * page_size) {
        bad = 1;
        continue;
      }
      const int page = block_table[(size_t)b * max_pages + (size_t)(pos / page_size)];
      if (page < 0 || page >= num_pages) {
        bad = 1;
        continue;
      }
      for (int g = 0; g < h_kv; ++g) {
        const uint16_t* src = new_kv + (((size_t)b * s_new + t) * h_kv + g) * (size_t)d;
        uint16_t* dst =
            kvcache + (((size_t)page * page_size + (size_t)(pos % page_size)) * h_kv + g) * (size_t)d;
        memcpy(dst, src, (size_t)d * sizeof(uint16_t));
      }
    }
  }
  return bad ? -1 : 0;
}

/*
 * Unabsorbed MLA decode for one KV head (FlashMLA overview, section 2.2): per
 * query head h the key and value of cached token j are up-projected from the
 * latent c_j = row[0:512] with per-head matrices
 *     k^C_{j,h} = W^UK_h c_j   (128),    v_{j,h} = W^UV_h c_j   (128),
 * with W^UK_h, W^UV_h stored [h][128][512]; the RoPE part k^R_j = row[512:576]
 * is shared by all heads.  Score_h(j) = scale * (q^C_h . k^C_{j,h} + q^R_h . k^R_j),
 * o_h = sum_j softmax_j(Score_h) v_{j,h}, lse_h = log sum_j exp(Score_h(j)).
 * Same masking readings as oracle_mla_decode; h_kv = 1.  q_nope [b][s_q][h_q][128]
 * and q_rope [b][s_q][h_q][64] are fp64; o [b][s_q][h_q][128], lse [b][h_q][s_q].
 */
int oracle_mla_decode_unabsorbed(const double* q_nope, const double* q_rope, const double* w_uk,
                                 const double* w_uv, const uint16_t* kv, const int32_t* block_table,
                                 const int32_t* seqlens, int batch, int s_q, int h_q, int page_size,
                                 int max_pages, int causal, double softmax_scale, double* o,
                                 double* lse, int nthreads) {
  const int dn = 128, dr = 64, dc = 512, d = 576, dvo = 128;
  if (batch < 0 || s_q < 1 || h_q < 1 || page_size < 1) return -1;
  (void)nthreads;
  double* s = NULL;
  double* c = (double*)malloc(sizeof(double) * d);
  for (int b = 0; b < batch; ++b) {
    const int L = seqlens[b] > 0 ? seqlens[b] : 0;
    free(s);
    s = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
    for (int i = 0; i < s_q; ++i) {
      const int last = causal ? (L - s_q) + i : L - 1;
      for (int h = 0; h < h_q; ++h) {
        const double* qn = q_nope + (((size_t)b * s_q + i) * h_q + h) * dn;
        const double* qr = q_rope + (((size_t)b * s_q + i) * h_q + h) * dr;
        const double* wk = w_uk + (size_t)h * dn * dc;
        const double* wv = w_uv + (size_t)h * dvo * dc;
        double* orow = o + (((size_t)b * s_q + i) * h_q + h) * dvo;
        for (int c2 = 0; c2 < dvo; ++c2) orow[c2] = 0.0;
        double* lse_out = lse + ((size_t)b * h_q + h) * s_q + i;
        if (last < 0) {
          *lse_out = -INFINITY;
          continue;
        }
        double m = -INFINITY;
        for (int j = 0; j <= last; ++j) {
          const uint16_t* row = kv_row(kv, block_table, max_pages, b, j, 0, 1, d, page_size);
          for (int k = 0; k < d; ++k) c[k] = bf16_to_double(row[k]);
          double acc = 0.0;
          for (int r = 0; r < dn; ++r) {  /* k^C_{j,h}[r] = sum_k W^UK_h[r][k] c_j[k] */
            double t = 0.0;
            for (int k = 0; k < dc; ++k) t += wk[(size_t)r * dc + k] * c[k];
            acc += qn[r] * t;
          }
          for (int r = 0; r < dr; ++r) acc += qr[r] * c[dc + r];
          s[j] = softmax_scale * acc;
          if (s[j] > m) m = s[j];
        }
        double z = 0.0;
        for (int j = 0; j <= last; ++j) z += exp(s[j] - m);
        for (int j = 0; j <= last; ++j) {
          const double w = exp(s[j] - m) / z;
          const uint16_t* row = kv_row(kv, block_table, max_pages, b, j, 0, 1, d, page_size);
          for (int k = 0; k < dc; ++k) c[k] = bf16_to_double(row[k]);
          for (int r = 0; r < dvo; ++r) {  /* v_{j,h}[r] = sum_k W^UV_h[r][k] c_j[k] */
            double t = 0.0;
            for (int k = 0; k < dc; ++k) t += wv[(size_t)r * dc + k] * c[k];
            orow[r] += w * t;
          }
        }
        *lse_out = log(z) + m;
      }
    }
  }
  free(s);
  free(c);
  return 0;
}
