// Weight-streaming projections of the MLA step on sm_100a tensor cores:
//   append   [W_DKV; W_KR] h           (MLA walk-through, section 1 step 1; eq. 9)
//   absorb   c_Q = W_DQ h, [W_UQ; W_QR] c_Q, q_lat,h = W_UK_h^T q_C,h
//                                       (section 1 step 3, section 3 order B; eqs. 12-13)
//   out_proj o_h = W_UV_h o_lat,h       (section 3 order B; eq. 11)
//
// At decode batch sizes these are skinny products: thousands of weight rows
// against at most a few hundred token rows, so they are bound by streaming
// the weights from HBM. The kernel computes D[m][n] = sum_k A[m][k] B[n][k]
// with the weight rows as the 128-row MMA operand A and the tokens as N
// (<= 256), K split across CTAs so that every SM streams weights, fp32
// partial sums to the workspace, and a small per-op finalize kernel that sums
// the splits and applies RoPE, rounding and the scatter into the cache or q.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace gemm {

constexpr int BM = 128, BK = 64, NUM_THREADS = 192;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB

struct Params {
  int m_total;       // rows of D per batch
  int m_split;       // rows [m_split, m_total) come from the second A map
  int n_total;       // tokens
  int n_tile;        // MMA N (multiple of 16, <= 256)
  int k_total;       // contraction length per batch
  int k_blocks_per_split;
  int splits;
  int a_mn_major;    // A stored with m contiguous (W_UK^T)
  int a_batch_rows;  // A row offset per batch (K-major: m rows; MN-major: k rows)
  int b_batch_cols;  // B column (k) offset per batch
  int stages;
  float *out;        // [batch][split][n_total][m_total]
};

__host__ __device__ constexpr int b_stage_bytes(int n_tile) { return n_tile * BK * 2; }

// One CTA: M tile blockIdx.x, N tile blockIdx.y, (batch, split) blockIdx.z.
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a2,
           const __grid_constant__ CUtensorMap tm_b, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b_bytes = b_stage_bytes(p.n_tile);
  const int stage_bytes = A_STAGE + b_bytes;
  const uint32_t bars = sbase + p.stages * stage_bytes;  // full[s], empty[s], done
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (p.stages + s); };
  const uint32_t done = bars + 8u * (2 * p.stages);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.stages * stage_bytes + 8 * (2 * p.stages + 1));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int m_tile = blockIdx.x, n_tile = blockIdx.y;
  const int batch = blockIdx.z / p.splits, split = blockIdx.z % p.splits;
  const int kb0 = split * p.k_blocks_per_split;
  const int kb1 = min(p.k_total / BK, kb0 + p.k_blocks_per_split);
  const int nkb = kb1 - kb0;
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(p.n_tile)) tmem_cols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<1>(smem_u32(tmem_slot), tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int m0 = m_tile * BM;
  const bool second = m0 >= p.m_split;
  const CUtensorMap *am = second ? &tm_a2 : &tm_a;
  const int am0 = second ? m0 - p.m_split : m0;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    for (int i = 0; i < nkb; ++i) {
      const int s = i % p.stages;
      if (i >= p.stages && !mbar_wait(empty(s), ((i / p.stages) - 1) & 1, abort_flag)) break;
      mbar_arrive_expect_tx(full(s), stage_bytes);
      const uint32_t a_dst = sbase + s * stage_bytes;
      const int k0 = (kb0 + i) * BK;
      if (!p.a_mn_major) {
        tma_load_2d(a_dst, am, k0, am0 + batch * p.a_batch_rows, full(s));
      } else {
        // A(m, k) at W[k][m]: two 64-wide m boxes of 64 k-rows each
        tma_load_2d(a_dst, am, am0, k0 + batch * p.a_batch_rows, full(s));
        tma_load_2d(a_dst + A_STAGE / 2, am, am0 + 64, k0 + batch * p.a_batch_rows, full(s));
      }
      tma_load_2d(a_dst + A_STAGE, &tm_b, k0 + batch * p.b_batch_cols, n_tile * p.n_tile, full(s));
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16(BM, p.n_tile, p.a_mn_major != 0, false);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % p.stages;
      if (!mbar_wait(full(s), (i / p.stages) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t a_src = sbase + s * stage_bytes;
      const uint32_t b_src = a_src + A_STAGE;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t ad = p.a_mn_major ? sdesc_sw128(a_src + kk * 2048, A_STAGE / 2, 1024)
                                         : sdesc_sw128(a_src + kk * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(b_src + kk * 32, 16, 1024);
        tc_mma<1>(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(empty(s));
    }
    tc_commit(done);
  } else if (warp >= 2) {
    // ------------------------------------------------------------- epilogue
    const int sp = warp & 3;
    const int row = 32 * sp + lane;  // m within tile
    mbar_wait_warp(done, 0, abort_flag);
    tc_fence_after();
    const int m = m0 + row;
    float *out = p.out + (static_cast<int64_t>(batch) * p.splits + split) * p.n_total * p.m_total;
    const int n_base = n_tile * p.n_tile;
    for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + c0, v);
      tmem_wait_ld();
      if (m < p.m_total) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int n = n_base + c0 + c;
          if (c0 + c < p.n_tile && n < p.n_total)
            out[static_cast<int64_t>(n) * p.m_total + m] = nkb > 0 ? __uint_as_float(v[c]) : 0.f;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc<1>(tmem, tmem_cols);
}

// ---------------------------------------------------------- finalizers ----

__device__ __forceinline__ float sum_splits(const float *part, int splits, int64_t stride, int64_t idx) {
  float acc = 0.f;
  for (int s = 0; s < splits; ++s) acc += part[s * stride + idx];
  return acc;
}

// rows [T][576] = sum of splits; RoPE on [512, 576); bf16; store at the
// cache row of (seq_idx[t], positions[t]). One block of 288 threads per
// token, one thread per element pair.
__global__ void k_fin_append(const float *part, int splits, int T, int d_c, int d_r, double rope_base,
                             const int32_t *seq_idx, const int32_t *positions, CacheView cache) {
  const int t = blockIdx.x;
  const int D = d_c + d_r;
  const int64_t stride = static_cast<int64_t>(T) * D;
  const int pos = positions[t];
  const int64_t row = cache_row(cache, seq_idx[t], pos);
  if (row < 0) {
    if (threadIdx.x == 0) dev_error(MLA_DEVERR_DATA);
    return;
  }
  __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(cache.data) + row * D;
  for (int e = 2 * threadIdx.x; e < D; e += 2 * blockDim.x) {
    float x0 = sum_splits(part, splits, stride, static_cast<int64_t>(t) * D + e);
    float x1 = sum_splits(part, splits, stride, static_cast<int64_t>(t) * D + e + 1);
    if (e >= d_c) rope_pair(x0, x1, (e - d_c) / 2, d_r, pos, rope_base);
    *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(x0, x1);
  }
}

// dst[t][n] (bf16, row pitch ld) = sum of splits of part[.][t][n], n < N.
__global__ void k_fin_store(const float *part, int splits, int T, int N, __nv_bfloat16 *dst, int64_t ld) {
  const int64_t stride = static_cast<int64_t>(T) * N;
  for (int64_t i = 2 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); i < stride;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / N, n = i % N;
    const float x0 = sum_splits(part, splits, stride, i), x1 = sum_splits(part, splits, stride, i + 1);
    *reinterpret_cast<uint32_t *>(dst + t * ld + n) = pack_bf16x2(x0, x1);
  }
}

// [W_UQ; W_QR] c_Q partials: rows < n_h*d_h are q_C (bf16 [T][n_h*d_h]);
// rows above are q_R before RoPE: rotate and store into q[t][h][d_c + r].
__global__ void k_fin_uq(const float *part, int splits, int T, int n_h, int d_h, int d_c, int d_r,
                         double rope_base, const int32_t *positions, __nv_bfloat16 *qc, __nv_bfloat16 *q) {
  const int M = n_h * (d_h + d_r);
  const int64_t stride = static_cast<int64_t>(T) * M;
  const int t = blockIdx.y;
  const int pos = positions[t];
  for (int e = 2 * (blockIdx.x * blockDim.x + threadIdx.x); e < M; e += 2 * gridDim.x * blockDim.x) {
    float x0 = sum_splits(part, splits, stride, static_cast<int64_t>(t) * M + e);
    float x1 = sum_splits(part, splits, stride, static_cast<int64_t>(t) * M + e + 1);
    if (e < n_h * d_h) {
      *reinterpret_cast<uint32_t *>(qc + static_cast<int64_t>(t) * n_h * d_h + e) = pack_bf16x2(x0, x1);
    } else {
      const int r = e - n_h * d_h, h = r / d_r, i = r % d_r;
      rope_pair(x0, x1, i / 2, d_r, pos, rope_base);
      *reinterpret_cast<uint32_t *>(q + (static_cast<int64_t>(t) * n_h + h) * (d_c + d_r) + d_c + i) =
          pack_bf16x2(x0, x1);
    }
  }
}

// Per-head partials part[h][split][t][m] (m < M) -> bf16 dst[t][h][m] with
// head pitch hp and token pitch tp.
__global__ void k_fin_heads(const float *part, int splits, int T, int M, int n_h, __nv_bfloat16 *dst,
                            int64_t tp, int64_t hp) {
  const int h = blockIdx.y;
  const int64_t stride = static_cast<int64_t>(T) * M;
  const float *ph = part + static_cast<int64_t>(h) * splits * stride;
  for (int64_t i = 2 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); i < stride;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / M, m = i % M;
    const float x0 = sum_splits(ph, splits, stride, i), x1 = sum_splits(ph, splits, stride, i + 1);
    *reinterpret_cast<uint32_t *>(dst + t * tp + h * hp + m) = pack_bf16x2(x0, x1);
  }
  (void)n_h;
}

// Split-K choice: enough CTAs to cover the GPU about twice, at least 2 K
// blocks per split where K allows.
inline int choose_splits(int tiles, int k_blocks, int sms) {
  int s = (2 * sms + tiles - 1) / tiles;
  s = s < 1 ? 1 : s;
  const int max_s = k_blocks >= 4 ? k_blocks / 2 : k_blocks;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  // equalise: every split gets ceil(k_blocks / s) blocks
  const int per = (k_blocks + s - 1) / s;
  return (k_blocks + per - 1) / per;
}

inline int n_tile_for(int T) {
  int n = ((T < 256 ? T : 256) + 15) / 16 * 16;
  return n < 16 ? 16 : n;
}

inline int stages_for(int n_tile) {
  const int budget = 200 * 1024;
  int s = budget / (A_STAGE + b_stage_bytes(n_tile));
  return s > 8 ? 8 : (s < 2 ? 2 : s);
}

inline size_t smem_for(int n_tile, int stages) {
  return static_cast<size_t>(stages) * (A_STAGE + b_stage_bytes(n_tile)) + 8 * (2 * stages + 1) + 16 + 1024;
}

}  // namespace gemm
}  // namespace mla
