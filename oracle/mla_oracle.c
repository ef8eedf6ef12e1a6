/*
 * Plain fp64 CPU oracle for Multi-head Latent Attention (MLA, DeepSeek-V2),
 * absorbed-form decode.
 *
 * TEST INFRASTRUCTURE ONLY. This file is compiled into liboracle.so and is
 * loaded by tests/, by __graft_entry__.smoke() and by the cpu_baseline /
 * reference arm of bench.py. The product path (the CUDA library) never links,
 * loads or calls it, and it shares no code, header, table or helper with the
 * CUDA path.
 *
 * Every routine is the plain definition of the step it computes, written with
 * naive loops in double precision: no blocking, no fusion, no reordering
 * beyond what the definition states. Sources (page title, section/equation):
 *
 *  - "MLA (Multi-head latent attention)" walk-through (h.sjds.net), section 1,
 *    step 1 (write memory: joint KV down-projection to a 512-d latent and a
 *    64-d decoupled RoPE key shared by every head), step 2 (per-head K/V
 *    up-projection), step 3 (query down-projection to 1536-d, per-head
 *    up-projection and per-head RoPE query taken from the query latent),
 *    step 4 (per-head 192-d scoring and softmax), section 3 (order A =
 *    decompress then dot; order B = absorb W_UK into the query and read out
 *    in latent space, decompress once with W_UV at the end).
 *  - "DeepSeek-V2 MLA" explainer (modelers.csdn.net), equations (9)-(13) and
 *    the absorption remark in section 3.
 *  - "Attention / RoPE tutorial" (xianlaiwan.cn): RoPE rotates q and k by
 *    position so that scores depend on the relative offset (RoFormer).
 *
 * Readings taken where the pages are silent:
 *  - softmax scale 1/sqrt(d_h + d_R) (the score lives in the 192-d
 *    concatenated space of step 4);
 *  - RoPE pairs are interleaved (2i, 2i+1), theta_i = base^(-2i/d_R);
 *  - a new query token j of sequence b (n_q tokens appended this step, L_b
 *    cached entries after the append) sits at position L_b - n_q + j and sees
 *    cached positions 0 .. L_b - n_q + j (causal within the step);
 *  - no normalisation layers and no biases.
 *
 * Parity pins (tests/test_oracle_pins.py): every function below is pinned by
 * at least one check that does not re-run this code's own formula:
 *  - orc_rope: the d_R = 2 closed form at position 1, the theta table, norm
 *    preservation, RoPE(x, 0) = x and the relative-position property;
 *  - orc_slot: hand-computed slots, paged = contiguous on the same rows;
 *  - orc_append, orc_absorb_q: the same chains through torch.matmul in fp64,
 *    RoPE shift invariance end to end, and (absorb) the merged matrix;
 *  - orc_decode (orc_attend_latent, orc_visible): worked examples computed by
 *    hand (tests/golden/hand_examples.json), one cached row, identical rows,
 *    q = 0, causal masking within a step, the reduction to torch's
 *    scaled-dot-product attention, order A = order B;
 *  - orc_attend_range, orc_combine: any split merged equals the unsplit result;
 *  - orc_out_proj, orc_o_proj, orc_absorb_wo, orc_absorb_merge: library
 *    products, and each absorbed form against its two-stage form;
 *  - orc_decode_order_a: order A = order B, and torch's scaled-dot-product
 *    attention over heads decompressed by numpy;
 *  - bf16 reads: exact values.
 * tests/test_oracle_mutants.py plants plausible mistakes in a copy of this
 * file, one at a time, and requires a pin to fail against each.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t d;      /* model width                      */
  int32_t n_h;    /* heads                            */
  int32_t d_h;    /* per-head dim                     */
  int32_t d_c;    /* KV latent dim                    */
  int32_t d_cq;   /* query latent dim                 */
  int32_t d_r;    /* decoupled RoPE dim               */
  double rope_base;
  double scale;   /* softmax scale; <= 0 selects 1/sqrt(d_h + d_r) */
} orc_dims;

/* Cache description. Rows are d_c + d_r numbers: [c_KV | k_R].
 * dtype 0: bf16 bit patterns (uint16), 1: float32, 2: float64.            */
typedef struct {
  const void *data;
  int32_t dtype;
  int32_t paged;
  int32_t block_size;
  int32_t max_blocks_per_seq;
  const int32_t *block_table; /* [num_seqs][max_blocks_per_seq] (paged)    */
  int64_t max_len;            /* contiguous: rows per sequence             */
} orc_cache;

static double orc_scale(const orc_dims *p) {
  return p->scale > 0.0 ? p->scale : 1.0 / sqrt((double)(p->d_h + p->d_r));
}

/* bf16 -> real: the 16 stored bits are the top half of an IEEE binary32. */
static double orc_bf16(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double orc_read(const void *base, int32_t dtype, int64_t i) {
  if (dtype == 0) return orc_bf16(((const uint16_t *)base)[i]);
  if (dtype == 1) return (double)((const float *)base)[i];
  return ((const double *)base)[i];
}

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* y[r] = sum_k W[r][k] x[k], W row-major rows x cols (out x in, as eq. (9)). */
static void orc_matvec(const double *W, int rows, int cols, const double *x, double *y) {
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int k = 0; k < cols; ++k) acc += W[(int64_t)r * cols + k] * x[k];
    y[r] = acc;
  }
}

/* RoPE, RoFormer interleaved pairs: rotate (x[2i], x[2i+1]) by pos*theta_i. */
void orc_rope(double *x, int d_r, double pos, double base) {
  for (int i = 0; i < d_r / 2; ++i) {
    double theta = pow(base, -2.0 * (double)i / (double)d_r);
    double a = pos * theta;
    double c = cos(a), s = sin(a);
    double x0 = x[2 * i], x1 = x[2 * i + 1];
    x[2 * i] = x0 * c - x1 * s;
    x[2 * i + 1] = x0 * s + x1 * c;
  }
}

/* Physical row of logical (sequence b, position pos) in the cache. */
int64_t orc_slot(const orc_cache *c, int32_t b, int64_t pos) {
  if (!c->paged) return (int64_t)b * c->max_len + pos;
  int64_t blk = c->block_table[(int64_t)b * c->max_blocks_per_seq + pos / c->block_size];
  return blk * c->block_size + pos % c->block_size;
}

/* Step 1 (eq. 9 + decoupled key): rows[t] = [W_DKV h_t ; RoPE(W_KR h_t, pos_t)]. */
void orc_append(const orc_dims *p, const double *h, const double *W_DKV, const double *W_KR,
                const int32_t *positions, int T, double *rows) {
  const int D = p->d_c + p->d_r;
  /* token rows are independent: one row per OpenMP iteration */
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    const double *ht = h + (int64_t)t * p->d;
    double *out = rows + (int64_t)t * D;
    orc_matvec(W_DKV, p->d_c, p->d, ht, out);
    orc_matvec(W_KR, p->d_r, p->d, ht, out + p->d_c);
    orc_rope(out + p->d_c, p->d_r, (double)positions[t], p->rope_base);
  }
}

/* Step 3 + absorption (eqs. 12-13, order B):
 *   c_Q = W_DQ h;  q_C,h = W_UQ_h c_Q;  q_R,h = RoPE(W_QR_h c_Q, pos);
 *   q_lat,h = W_UK_h^T q_C,h.
 * q_out[t][h] = [q_lat,h | q_R,h] (d_c + d_r). q_C_out (optional) = q_C,h. */
void orc_absorb_q(const orc_dims *p, const double *h, const double *W_DQ, const double *W_UQ,
                  const double *W_QR, const double *W_UK, const int32_t *positions, int T,
                  double *q_out, double *q_C_out) {
  const int D = p->d_c + p->d_r;
  /* token rows are independent: one row per OpenMP iteration, each thread
   * with its own c_Q and q_C scratch */
#pragma omp parallel
  {
  double *cq = (double *)malloc(sizeof(double) * p->d_cq);
  double *qc = (double *)malloc(sizeof(double) * p->d_h);
#pragma omp for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) {
    orc_matvec(W_DQ, p->d_cq, p->d, h + (int64_t)t * p->d, cq);
    for (int hh = 0; hh < p->n_h; ++hh) {
      double *q = q_out + ((int64_t)t * p->n_h + hh) * D;
      orc_matvec(W_UQ + (int64_t)hh * p->d_h * p->d_cq, p->d_h, p->d_cq, cq, qc);
      orc_matvec(W_QR + (int64_t)hh * p->d_r * p->d_cq, p->d_r, p->d_cq, cq, q + p->d_c);
      orc_rope(q + p->d_c, p->d_r, (double)positions[t], p->rope_base);
      for (int j = 0; j < p->d_c; ++j) {
        double acc = 0.0;
        for (int i = 0; i < p->d_h; ++i)
          acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * qc[i];
        q[j] = acc;
      }
      if (q_C_out)
        memcpy(q_C_out + ((int64_t)t * p->n_h + hh) * p->d_h, qc, sizeof(double) * p->d_h);
    }
  }
  free(cq);
  free(qc);
  }
}

/* Order B for one (query row, head) over cached positions [start, end) of
 * sequence b: s_i = scale * (q_lat . c_KV_i + q_R . k_R_i); exact two-pass
 * softmax; o_lat = sum_i p_i c_KV_i; lse = m + log sum exp(s - m). */
static void orc_attend_latent(const orc_dims *p, const double *q, const orc_cache *c, int32_t b,
                              int64_t start, int64_t end, double *o_lat, double *lse,
                              double *scores) {
  const int D = p->d_c + p->d_r;
  const double scale = orc_scale(p);
  double m = -INFINITY;
  for (int64_t i = start; i < end; ++i) {
    int64_t row = orc_slot(c, b, i);
    double acc = 0.0;
    for (int j = 0; j < D; ++j) acc += q[j] * orc_read(c->data, c->dtype, row * D + j);
    double s = scale * acc;
    scores[i - start] = s;
    if (s > m) m = s;
  }
  double z = 0.0;
  for (int64_t i = start; i < end; ++i) z += exp(scores[i - start] - m);
  for (int j = 0; j < p->d_c; ++j) o_lat[j] = 0.0;
  for (int64_t i = start; i < end; ++i) {
    double w = exp(scores[i - start] - m) / z;
    int64_t row = orc_slot(c, b, i);
    for (int j = 0; j < p->d_c; ++j) o_lat[j] += w * orc_read(c->data, c->dtype, row * D + j);
  }
  *lse = m + log(z);
}

/* Positions visible to query token j of sequence b (causal within the step). */
static int64_t orc_visible(const int32_t *seq_lens, int32_t b, int n_q, int j) {
  return (int64_t)seq_lens[b] - n_q + 1 + j;
}

/* Order B decode over the whole visible range. q: [T][n_h][d_c+d_r],
 * T = B*n_q, token row t = b*n_q + j. If pairs != NULL only the listed
 * (t, h) pairs are computed (pairs[2k], pairs[2k+1]); outputs are then packed
 * [n_pairs][d_c] / [n_pairs]. Returns 0, or -1 on an invalid length. */
int orc_decode(const orc_dims *p, const double *q, const orc_cache *c, const int32_t *seq_lens,
               int B, int n_q, double *o_lat, double *lse, const int32_t *pairs, int n_pairs) {
  const int D = p->d_c + p->d_r;
  const int64_t total = pairs ? (int64_t)n_pairs : (int64_t)B * n_q * p->n_h;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] < n_q) return -1;
  int64_t maxlen = 0;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] > maxlen) maxlen = seq_lens[b];
#pragma omp parallel
  {
    double *scores = (double *)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < total; ++k) {
      int64_t t, hh;
      if (pairs) {
        t = pairs[2 * k];
        hh = pairs[2 * k + 1];
      } else {
        t = k / p->n_h;
        hh = k % p->n_h;
      }
      int32_t b = (int32_t)(t / n_q);
      int j = (int)(t % n_q);
      orc_attend_latent(p, q + (t * p->n_h + hh) * D, c, b, 0, orc_visible(seq_lens, b, n_q, j),
                        o_lat + k * p->d_c, lse + k, scores);
    }
    free(scores);
  }
  return 0;
}

/* Order B over an arbitrary cached range [start, end): partial o (normalised
 * over the range) and its lse. Used to pin the split-KV combine algebra. */
void orc_attend_range(const orc_dims *p, const double *q_row, const orc_cache *c, int32_t b,
                      int64_t start, int64_t end, double *o_lat, double *lse) {
  double *scores = (double *)malloc(sizeof(double) * (size_t)(end - start > 0 ? end - start : 1));
  orc_attend_latent(p, q_row, c, b, start, end, o_lat, lse, scores);
  free(scores);
}

/* Log-sum-exp merge of S partial results of one (query row, head):
 * lse = log sum_s exp(lse_s); o = sum_s exp(lse_s - lse) o_s. */
void orc_combine(int S, int d_c, const double *o_parts, const double *lse_parts, double *o,
                 double *lse) {
  double m = -INFINITY;
  for (int s = 0; s < S; ++s)
    if (lse_parts[s] > m) m = lse_parts[s];
  double z = 0.0;
  for (int s = 0; s < S; ++s) z += exp(lse_parts[s] - m);
  double L = m + log(z);
  for (int j = 0; j < d_c; ++j) o[j] = 0.0;
  for (int s = 0; s < S; ++s) {
    double w = exp(lse_parts[s] - L);
    for (int j = 0; j < d_c; ++j) o[j] += w * o_parts[(int64_t)s * d_c + j];
  }
  *lse = L;
}

/* Step 2 + step 5 readout (eq. 11): o[t][h*d_h + i] = sum_j W_UV[h*d_h+i][j] o_lat[t][h][j]. */
void orc_out_proj(const orc_dims *p, const double *o_lat, const double *W_UV, int T, double *o) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t)
    for (int hh = 0; hh < p->n_h; ++hh)
      orc_matvec(W_UV + (int64_t)hh * p->d_h * p->d_c, p->d_h, p->d_c,
                 o_lat + ((int64_t)t * p->n_h + hh) * p->d_c,
                 o + (int64_t)t * p->n_h * p->d_h + (int64_t)hh * p->d_h);
}

/* Step 5 of the walk-through (section 1, "整合"): the n_h head outputs of a
 * token, concatenated (n_h * d_h numbers), are projected back to the model
 * width by W_O (d x n_h*d_h): y_t = W x_t for every token row t. The same
 * routine applies the absorbed matrix of orc_absorb_wo to o_lat. */
void orc_o_proj(const double *W, int rows, int cols, const double *x, int T, double *y) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int t = 0; t < T; ++t) orc_matvec(W, rows, cols, x + (int64_t)t * cols, y + (int64_t)t * rows);
}

/* W_UV absorbed into the output projection (DeepSeek-V2 explainer, section 3
 * remark; MLA walk-through, section 3 order B): since o_h = W_UV_h o_lat,h,
 * W_O [o_1; ...; o_n_h] = W_OV [o_lat,1; ...; o_lat,n_h] with
 *   W_OV[r][h*d_c + j] = sum_i W_O[r][h*d_h + i] W_UV[h*d_h + i][j],
 * a d x n_h*d_c matrix. W_O is d x n_h*d_h, W_UV is n_h*d_h x d_c. */
void orc_absorb_wo(const orc_dims *p, const double *W_O, const double *W_UV, double *W_OV) {
  const int64_t ko = (int64_t)p->n_h * p->d_h, kv = (int64_t)p->n_h * p->d_c;
  /* rows r are independent: one row per OpenMP iteration */
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < p->d; ++r)
    for (int hh = 0; hh < p->n_h; ++hh)
      for (int j = 0; j < p->d_c; ++j) {
        double acc = 0.0;
        for (int i = 0; i < p->d_h; ++i)
          acc += W_O[r * ko + (int64_t)hh * p->d_h + i] * W_UV[((int64_t)hh * p->d_h + i) * p->d_c + j];
        W_OV[r * kv + (int64_t)hh * p->d_c + j] = acc;
      }
}

/* Merged absorption matrix (walk-through, section 3 order B: the product of
 * the two matrices absorbed on the query side can be formed offline):
 * W_UQK_h = W_UK_h^T W_UQ_h, so that q_lat,h = W_UQK_h c_Q in one product,
 *   W_UQK[h*d_c + j][c] = sum_i W_UK[h*d_h + i][j] W_UQ[h*d_h + i][c].
 * W_UQ is n_h*d_h x d_cq, W_UK is n_h*d_h x d_c, W_UQK is n_h*d_c x d_cq. */
void orc_absorb_merge(const orc_dims *p, const double *W_UQ, const double *W_UK, double *W_UQK) {
  /* heads are independent: one head per OpenMP iteration */
#pragma omp parallel for schedule(dynamic, 1)
  for (int hh = 0; hh < p->n_h; ++hh)
    for (int j = 0; j < p->d_c; ++j)
      for (int c = 0; c < p->d_cq; ++c) {
        double acc = 0.0;
        for (int i = 0; i < p->d_h; ++i)
          acc += W_UK[((int64_t)hh * p->d_h + i) * p->d_c + j] * W_UQ[((int64_t)hh * p->d_h + i) * p->d_cq + c];
        W_UQK[((int64_t)hh * p->d_c + j) * p->d_cq + c] = acc;
      }
}

/* Order A (training form, section 3): decompress per head
 *   k_C,i = W_UK_h c_KV_i, v_i = W_UV_h c_KV_i,
 * score = scale * ([q_C ; q_R] . [k_C,i ; k_R,i]) in d_h + d_r dims,
 * o_h = sum_i p_i v_i. q_C: [T][n_h][d_h], q_R: [T][n_h][d_r].
 * pairs as in orc_decode; output o: [rows][d_h]. */
int orc_decode_order_a(const orc_dims *p, const double *q_C, const double *q_R, const double *W_UK,
                       const double *W_UV, const orc_cache *c, const int32_t *seq_lens, int B,
                       int n_q, double *o, const int32_t *pairs, int n_pairs) {
  const int D = p->d_c + p->d_r;
  const double scale = orc_scale(p);
  const int64_t total = pairs ? (int64_t)n_pairs : (int64_t)B * n_q * p->n_h;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] < n_q) return -1;
  int64_t maxlen = 0;
  for (int b = 0; b < B; ++b)
    if (seq_lens[b] > maxlen) maxlen = seq_lens[b];
#pragma omp parallel
  {
    double *scores = (double *)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
    double *ckv = (double *)malloc(sizeof(double) * p->d_c);
    double *kc = (double *)malloc(sizeof(double) * p->d_h);
    double *v = (double *)malloc(sizeof(double) * p->d_h);
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < total; ++k) {
      int64_t t, hh;
      if (pairs) {
        t = pairs[2 * k];
        hh = pairs[2 * k + 1];
      } else {
        t = k / p->n_h;
        hh = k % p->n_h;
      }
      int32_t b = (int32_t)(t / n_q);
      int j = (int)(t % n_q);
      int64_t L = orc_visible(seq_lens, b, n_q, j);
      const double *qc = q_C + (t * p->n_h + hh) * p->d_h;
      const double *qr = q_R + (t * p->n_h + hh) * p->d_r;
      const double *Wk = W_UK + hh * (int64_t)p->d_h * p->d_c;
      const double *Wv = W_UV + hh * (int64_t)p->d_h * p->d_c;
      double m = -INFINITY;
      for (int64_t i = 0; i < L; ++i) {
        int64_t row = orc_slot(c, b, i);
        for (int jj = 0; jj < p->d_c; ++jj) ckv[jj] = orc_read(c->data, c->dtype, row * D + jj);
        orc_matvec(Wk, p->d_h, p->d_c, ckv, kc);
        double acc = 0.0;
        for (int jj = 0; jj < p->d_h; ++jj) acc += qc[jj] * kc[jj];
        for (int jj = 0; jj < p->d_r; ++jj)
          acc += qr[jj] * orc_read(c->data, c->dtype, row * D + p->d_c + jj);
        scores[i] = scale * acc;
        if (scores[i] > m) m = scores[i];
      }
      double z = 0.0;
      for (int64_t i = 0; i < L; ++i) z += exp(scores[i] - m);
      double *out = o + k * p->d_h;
      for (int jj = 0; jj < p->d_h; ++jj) out[jj] = 0.0;
      for (int64_t i = 0; i < L; ++i) {
        int64_t row = orc_slot(c, b, i);
        for (int jj = 0; jj < p->d_c; ++jj) ckv[jj] = orc_read(c->data, c->dtype, row * D + jj);
        orc_matvec(Wv, p->d_h, p->d_c, ckv, v);
        double w = exp(scores[i] - m) / z;
        for (int jj = 0; jj < p->d_h; ++jj) out[jj] += w * v[jj];
      }
    }
    free(scores);
    free(ckv);
    free(kc);
    free(v);
  }
  return 0;
}
