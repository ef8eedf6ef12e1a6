// CUDA-core kernels for storage types or dims the tensor-core kernels are not
// built for (fp32 storage, small test dims). Same contracts as the
// tensor-core path; fp32 accumulation; intermediates stay fp32.
#pragma once
#include "common.cuh"

namespace mla {

// Y(bt, t, n) (fp32) = sum_k W(bt, n, k) * X(bt, t, k)
//   W(bt, n, k) = W[bt*w_sb + n*w_sn + k*w_sk]  (any strides: covers W and W^T)
//   X(bt, t, k) = X[bt*x_sb + t*x_st + k]
//   Y(bt, t, n) = Y[bt*y_sb + t*y_st + n]
// One warp per output element; grid (ceil(N/8), T, batches), block 256.
template <typename TW, typename TX>
__global__ void __launch_bounds__(256) k_simt_linear(const TW *__restrict__ W, int64_t w_sb,
                                                     int64_t w_sn, int64_t w_sk,
                                                     const TX *__restrict__ X, int64_t x_sb,
                                                     int64_t x_st, float *__restrict__ Y,
                                                     int64_t y_sb, int64_t y_st, int N, int K) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + warp;
  const int t = blockIdx.y;
  const int bt = blockIdx.z;
  if (n >= N) return;
  const TW *w = W + bt * w_sb + n * w_sn;
  const TX *x = X + bt * x_sb + t * x_st;
  float acc = 0.f;
  for (int k = lane; k < K; k += 32) acc += ld_f(w + k * w_sk) * ld_f(x + k);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) Y[bt * y_sb + t * y_st + n] = acc;
}

// Per-head product of two matrices that share their row index i (d_h rows per
// head): out(h, a, b) = sum_i L(h, i, a) R(h, i, b), rounded once to the
// storage type. X(h, i, c) = X[h*s_h + i*s_i + c*s_c] for L, R and out (whose
// i stride is unused). One thread per output element; grid (ceil(B/256), A, H).
template <typename T>
__global__ void __launch_bounds__(256) k_simt_head_product(const T *__restrict__ L, int64_t l_h, int64_t l_i,
                                                           int64_t l_a, const T *__restrict__ R, int64_t r_h,
                                                           int64_t r_i, int64_t r_b, T *__restrict__ out,
                                                           int64_t o_h, int64_t o_a, int64_t o_b, int A, int Bn,
                                                           int I) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  const int a = blockIdx.y, h = blockIdx.z;
  if (b >= Bn || a >= A) return;
  const T *l = L + h * l_h + a * l_a;
  const T *r = R + h * r_h + b * r_b;
  float acc = 0.f;
  for (int i = 0; i < I; ++i) acc += ld_f(l + i * l_i) * ld_f(r + i * r_i);
  out[h * o_h + a * o_a + b * o_b] = from_f<T>(acc);
}

// Append epilogue: rows [T][D] fp32 -> RoPE on [d_c, D) at positions[t] ->
// storage dtype -> cache row of (seq_idx[t], positions[t]). One block per t.
template <typename T>
__global__ void k_simt_append_store(const float *__restrict__ rows, int D, int d_c, int d_r,
                                    double rope_base, const int32_t *__restrict__ seq_idx,
                                    const int32_t *__restrict__ positions, CacheView cache) {
  const int t = blockIdx.x;
  const int pos = positions[t];
  const int64_t row = cache_row(cache, seq_idx[t], pos);
  if (row < 0) {
    if (threadIdx.x == 0) dev_error(MLA_DEVERR_DATA);
    return;
  }
  T *dst = static_cast<T *>(cache.data) + row * D;
  const float *src = rows + static_cast<int64_t>(t) * D;
  for (int e = threadIdx.x; e < d_c; e += blockDim.x) dst[e] = from_f<T>(src[e]);
  for (int i = threadIdx.x; i < d_r / 2; i += blockDim.x) {
    float x0 = src[d_c + 2 * i], x1 = src[d_c + 2 * i + 1];
    rope_pair(x0, x1, i, d_r, pos, rope_base);
    dst[d_c + 2 * i] = from_f<T>(x0);
    dst[d_c + 2 * i + 1] = from_f<T>(x1);
  }
}

// q[t][h] = [q_lat (d_c) | RoPE(q_R_pre) (d_r)] in storage dtype.
// q_lat: [T][n_h][d_c] fp32, q_r: [T][n_h][d_r] fp32. One block per (t, h).
template <typename T>
__global__ void k_simt_q_store(const float *__restrict__ q_lat, const float *__restrict__ q_r,
                               int n_h, int d_c, int d_r, double rope_base,
                               const int32_t *__restrict__ positions, T *__restrict__ q) {
  const int t = blockIdx.x / n_h, h = blockIdx.x % n_h;
  const int D = d_c + d_r;
  const int pos = positions[t];
  T *dst = q + (static_cast<int64_t>(t) * n_h + h) * D;
  const float *ql = q_lat + (static_cast<int64_t>(t) * n_h + h) * d_c;
  const float *qr = q_r + (static_cast<int64_t>(t) * n_h + h) * d_r;
  for (int e = threadIdx.x; e < d_c; e += blockDim.x) dst[e] = from_f<T>(ql[e]);
  for (int i = threadIdx.x; i < d_r / 2; i += blockDim.x) {
    float x0 = qr[2 * i], x1 = qr[2 * i + 1];
    rope_pair(x0, x1, i, d_r, pos, rope_base);
    dst[d_c + 2 * i] = from_f<T>(x0);
    dst[d_c + 2 * i + 1] = from_f<T>(x1);
  }
}

// Order A for one (token row t, head h) per block (d_h <= blockDim.x): for
// every visible cached row i, thread k forms k_C,i[k] = W_UK_h[k] . c_KV_i and
// v_i[k] = W_UV_h[k] . c_KV_i; the score is scale ([q_C ; q_R] . [k_C,i ; k_R,i])
// and an online softmax accumulates o[k] = sum_i p_i v_i[k] / sum_i p_i.
// qa [T][n_h][d_h + d_r], o [T][n_h][d_h]. Shared memory: 2 * blockDim floats.
template <typename T>
__global__ void k_simt_attend_a(const T *__restrict__ qa, const T *__restrict__ W_UK, const T *__restrict__ W_UV,
                                CacheView cache, const int32_t *__restrict__ seq_lens, int n_q, int n_h, int d_h,
                                int d_c, int d_r, float scale, T *__restrict__ o) {
  extern __shared__ float red[];
  const int t = blockIdx.x / n_h, h = blockIdx.x % n_h;
  const int b = t / n_q, j = t % n_q;
  const int L = seq_lens[b];
  const int D = d_c + d_r, k = threadIdx.x;
  if (L < n_q || (!cache.paged && L > cache.max_len) ||
      (cache.paged && static_cast<int64_t>(L) > static_cast<int64_t>(cache.max_blocks_per_seq) * cache.block_size)) {
    if (threadIdx.x == 0 && j == 0 && h == 0) dev_error(MLA_DEVERR_DATA);
    return;
  }
  const int vis = L - n_q + 1 + j;
  const T *q = qa + (static_cast<int64_t>(t) * n_h + h) * (d_h + d_r);
  const T *wk = W_UK + static_cast<int64_t>(h) * d_h * d_c + static_cast<int64_t>(k) * d_c;
  const T *wv = W_UV + static_cast<int64_t>(h) * d_h * d_c + static_cast<int64_t>(k) * d_c;
  const T *data = static_cast<const T *>(cache.data);
  float m = -INFINITY, l = 0.f, acc = 0.f;
  for (int i = 0; i < vis; ++i) {
    const int64_t row = cache_row(cache, b, i);
    if (row < 0) {
      if (threadIdx.x == 0) dev_error(MLA_DEVERR_DATA);
      return;
    }
    const T *c = data + row * D;
    float kc = 0.f, vv = 0.f;
    if (k < d_h)
      for (int e = 0; e < d_c; ++e) {
        const float x = ld_f(c + e);
        kc += ld_f(wk + e) * x;
        vv += ld_f(wv + e) * x;
      }
    float part = k < d_h ? ld_f(q + k) * kc : 0.f;
    if (k < d_r) part += ld_f(q + d_h + k) * ld_f(c + d_c + k);
    red[k] = part;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (k < w) red[k] += red[k + w];
      __syncthreads();
    }
    const float s = scale * red[0];
    __syncthreads();
    const float mn = fmaxf(m, s);
    const float a = __expf(m - mn), pw = __expf(s - mn);  // m = -inf on the first row: a = 0
    l = l * a + pw;
    acc = acc * a + pw * vv;
    m = mn;
  }
  if (k < d_h) o[(static_cast<int64_t>(t) * n_h + h) * d_h + k] = from_f<T>(acc / l);
}

template <typename T>
__global__ void k_simt_store(const float *__restrict__ src, T *__restrict__ dst, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = from_f<T>(src[i]);
}

// Decode, one block per (token row t, head h), 8 warps. Each warp runs an
// online softmax over tokens warp, warp+8, ...; lane l owns latent elements
// l, l+32, ... The 8 partial states are merged in shared memory at the end.
// Requires D <= 32 * 32.
template <typename T>
__global__ void __launch_bounds__(256) k_simt_decode(const T *__restrict__ q, CacheView cache,
                                                     const int32_t *__restrict__ seq_lens, int n_q,
                                                     int n_h, int d_c, int d_r, float scale,
                                                     T *__restrict__ o_lat, float *__restrict__ lse) {
  constexpr int MAXE = 32;
  const int D = d_c + d_r;
  const int t = blockIdx.x / n_h, h = blockIdx.x % n_h;
  const int b = t / n_q, j = t % n_q;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float s_m[8], s_l[8];
  extern __shared__ float s_acc[];  // [8][d_c]

  const int L = seq_lens[b];
  const int64_t cap = cache.paged ? static_cast<int64_t>(cache.max_blocks_per_seq) * cache.block_size
                                  : cache.max_len;
  if (L < n_q || L > cap) {
    if (threadIdx.x == 0) dev_error(MLA_DEVERR_DATA);
    return;
  }
  const int vis = L - n_q + 1 + j;

  float qv[MAXE];
  const T *qrow = q + (static_cast<int64_t>(t) * n_h + h) * D;
#pragma unroll
  for (int k = 0; k < MAXE; ++k) qv[k] = (lane + 32 * k < D) ? ld_f(qrow + lane + 32 * k) : 0.f;

  float m = -INFINITY, l = 0.f, acc[MAXE];
#pragma unroll
  for (int k = 0; k < MAXE; ++k) acc[k] = 0.f;
  bool bad = false;
  for (int i = warp; i < vis; i += 8) {
    const int64_t row = cache_row(cache, b, i);
    if (row < 0) {
      bad = true;
      break;
    }
    const T *kv = static_cast<const T *>(cache.data) + row * D;
    float rv[MAXE];
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < MAXE; ++k) {
      rv[k] = (lane + 32 * k < D) ? ld_f(kv + lane + 32 * k) : 0.f;
      s += qv[k] * rv[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    s *= scale;
    const float m_new = fmaxf(m, s);
    const float alpha = __expf(m - m_new);
    const float p = __expf(s - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int k = 0; k < MAXE; ++k)
      if (lane + 32 * k < d_c) acc[k] = acc[k] * alpha + p * rv[k];
    m = m_new;
  }
  if (bad && lane == 0) dev_error(MLA_DEVERR_DATA);
  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int k = 0; k < MAXE; ++k)
    if (lane + 32 * k < d_c) s_acc[warp * d_c + lane + 32 * k] = acc[k];
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < 8; ++w) M = fmaxf(M, s_m[w]);
  float Lsum = 0.f;
  for (int w = 0; w < 8; ++w) Lsum += (s_m[w] == -INFINITY) ? 0.f : s_l[w] * __expf(s_m[w] - M);
  T *out = o_lat + (static_cast<int64_t>(t) * n_h + h) * d_c;
  for (int e = threadIdx.x; e < d_c; e += blockDim.x) {
    float v = 0.f;
    for (int w = 0; w < 8; ++w)
      if (s_m[w] != -INFINITY) v += s_acc[w * d_c + e] * __expf(s_m[w] - M);
    out[e] = from_f<T>(v / Lsum);
  }
  if (lse != nullptr && threadIdx.x == 0) lse[static_cast<int64_t>(t) * n_h + h] = M + logf(Lsum);
}

}  // namespace mla
