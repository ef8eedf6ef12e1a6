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

// k_gemm: TMA producer warps 0, 6 and 7 (stage s is issued by producer s % 3),
// the MMA warp 1, the epilogue warps 2-5. The TMA operations one warp issues
// complete one after another (~50 GB/s per warp), so a CTA that must stream
// its operands faster needs several issuing warps.
constexpr int BM = 128, BK = 64, NUM_THREADS = 256, PRODUCERS = 3;
constexpr int A_STAGE = BM * BK * 2;  // 16 KB

// Epilogue of one GEMM launch.
enum Epi : int {
  EPI_PARTIAL = 0,  // fp32 partial sums: out[batch][split][n][m]
  EPI_BF16 = 1,     // bf16 dst[batch * e_bs + n * e_ns + m]
  EPI_UQ = 2,       // rows < e_split: bf16 q_C at dst[n * e_split + m]; rows above: q_R rotated
                    // by RoPE at positions[n], stored at q[n][h][d_c + i] (m - e_split = h * d_r + i)
  EPI_QA = 3,       // as EPI_UQ, but q_C row m = h * d_c + i goes to q[n][h][i] (d_c = the q_C width)
};

struct Params {
  int m_total;       // rows of D per batch
  int m_split;       // rows [m_split, m_split2) come from the second A map
  int m_split2;      // rows [m_split2, m_total) come from the third A map
  int n_total;       // tokens
  int n_tile;        // MMA N (multiple of 16, <= 256)
  int k_total;       // contraction length per batch
  int k_blocks_per_split;
  int splits;
  int a_mn_major;    // A stored with m contiguous (W_UK^T)
  int b_mn_major;    // B stored with n contiguous (rows are k): n_tile a multiple of 64
  int a_batch_rows;  // A row offset per batch (K-major: m rows; MN-major: k rows)
  int b_batch_cols;  // B k offset per batch (a column for K-major B, a row for MN-major B)
  int stages;
  float *out;        // EPI_PARTIAL: [batch][split][n_total][m_total]
  int epi;
  __nv_bfloat16 *dst;  // EPI_BF16 / EPI_UQ (q_C)
  int64_t e_bs, e_ns;  // EPI_BF16 strides
  int e_split;         // EPI_UQ: first q_R row
  __nv_bfloat16 *q;    // EPI_UQ: q[T][n_h][d_c + d_r]
  int n_h, d_c, d_r;
  double rope_base;
  const int32_t *positions;
  int prefetch;  // launched with launch overlap: weight boxes of the first stages go out before griddep_wait
  // failure-path self-test only: every bounded wait gives up after wait_ns
  // (0: the library's default limit) and, with idle_producer set, the TMA
  // producer issues nothing, so that the MMA thread's first wait runs out
  uint64_t wait_ns;
  int idle_producer;
};

__host__ __device__ constexpr int b_stage_bytes(int n_tile) { return n_tile * BK * 2; }

// One CTA: M tile blockIdx.x, N tile blockIdx.y, (batch, split) blockIdx.z.
__global__ void __launch_bounds__(NUM_THREADS, 2)
    k_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a2,
           const __grid_constant__ CUtensorMap tm_a3, const __grid_constant__ CUtensorMap tm_b, const Params p) {
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
  const uint64_t wait_ns = p.wait_ns != 0 ? p.wait_ns : MLA_WAIT_NS;

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
  if (threadIdx.x == 0) griddep_launch_dependents();

  const int m0 = m_tile * BM;
  const bool third = m0 >= p.m_split2, second = !third && m0 >= p.m_split;
  const CUtensorMap *am = third ? &tm_a3 : (second ? &tm_a2 : &tm_a);
  const int am0 = third ? m0 - p.m_split2 : (second ? m0 - p.m_split : m0);

  if (warp == 0 || warp >= 6) {
    // --------------------------------------------------------- TMA producers
    // Every use of stage s is issued by producer s % 3, in order (so each
    // stage's empty-barrier waits are made by one warp). Under launch overlap
    // the first stages are armed together and their weight boxes issued before
    // the wait for the previous kernel on the stream (weights do not depend on
    // it), their token boxes after it. Otherwise the stages go out in order,
    // each stage's boxes together, so that the first stage is not queued
    // behind the weights of all the others.
    const int pid = warp == 0 ? 0 : warp - 5;
    const uint32_t stage0 = sbase;
    auto issue_a = [&](int i, int box) {  // box 1: second 64-wide m box of an MN-major A
      const uint32_t a_dst = stage0 + (i % p.stages) * stage_bytes;
      const int k0 = (kb0 + i) * BK;
      if (!p.a_mn_major)
        tma_load_2d(a_dst, am, k0, am0 + batch * p.a_batch_rows, full(i % p.stages));
      else  // A(m, k) at W[k][m]: two 64-wide m boxes of 64 k-rows each
        tma_load_2d(a_dst + box * (A_STAGE / 2), am, am0 + 64 * box, k0 + batch * p.a_batch_rows, full(i % p.stages));
    };
    auto issue_b = [&](int i) {
      const uint32_t a_dst = stage0 + (i % p.stages) * stage_bytes;
      if (!p.b_mn_major) {
        tma_load_2d(a_dst + A_STAGE, &tm_b, (kb0 + i) * BK + batch * p.b_batch_cols, n_tile * p.n_tile, full(i % p.stages));
      } else {  // B(n, k) at X[k][n]: n_tile / 64 boxes of 64 n x 64 k rows
        for (int j = 0; j < p.n_tile / 64; ++j)
          tma_load_2d(a_dst + A_STAGE + j * (64 * BK * 2), &tm_b, n_tile * p.n_tile + 64 * j,
                      (kb0 + i) * BK + batch * p.b_batch_cols, full(i % p.stages));
      }
    };
    const int nkp = p.idle_producer ? 0 : nkb;  // self-test: nothing is issued, no copy is in flight
    // stages <= 12: lanes l and 16 + l serve this producer's l-th early stage
    const int pre = p.prefetch ? min(nkp, p.stages) : 0;
    const int ip = pid + PRODUCERS * (lane & 15);
    if (lane == 0)
      for (int i = pid; i < pre; i += PRODUCERS) mbar_arrive_expect_tx(full(i), stage_bytes);
    __syncwarp();
    if (ip < pre) {
      if (lane < 16) issue_a(ip, 0);
      else if (p.a_mn_major) issue_a(ip, 1);
    }
    griddep_wait();
    if (lane < 16 && ip < pre) issue_b(ip);
    __syncwarp();
    for (int i = pre; i < nkp; ++i) {
      const int s = i % p.stages;
      if (s % PRODUCERS != pid) continue;
      bool good = true;
      if (lane == 0) {
        if (i >= p.stages) good = mbar_wait(empty(s), ((i / p.stages) - 1) & 1, abort_flag, wait_ns);
        if (good) mbar_arrive_expect_tx(full(s), stage_bytes);
      }
      if (!__shfl_sync(0xffffffffu, good, 0)) break;
      if (lane == 0) issue_b(i);
      else if (lane == 1) issue_a(i, 0);
      else if (lane == 2 && p.a_mn_major) issue_a(i, 1);
      __syncwarp();
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16(BM, p.n_tile, p.a_mn_major != 0, p.b_mn_major != 0);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % p.stages;
      if (!mbar_wait(full(s), (i / p.stages) & 1, abort_flag, wait_ns)) break;
      tc_fence_after();
      const uint32_t a_src = sbase + s * stage_bytes;
      const uint32_t b_src = a_src + A_STAGE;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t ad = p.a_mn_major ? sdesc_sw128(a_src + kk * 2048, A_STAGE / 2, 1024)
                                         : sdesc_sw128(a_src + kk * 32, 16, 1024);
        const uint64_t bd = p.b_mn_major ? sdesc_sw128(b_src + kk * 2048, 64 * BK * 2, 1024)
                                         : sdesc_sw128(b_src + kk * 32, 16, 1024);
        tc_mma<1>(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(empty(s));
    }
    tc_commit(done);
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------- epilogue
    const int sp = warp & 3;
    const int row = 32 * sp + lane;  // m within tile
    griddep_wait();  // outputs are written only once the previous kernel has finished
    mbar_wait_warp(done, 0, abort_flag, wait_ns);
    tc_fence_after();
    const int m = m0 + row;
    const int n_base = n_tile * p.n_tile;
    float *out = p.out + (static_cast<int64_t>(batch) * p.splits + split) * p.n_total * p.m_total;
    const bool rope_tile = (p.epi == EPI_UQ || p.epi == EPI_QA) && m0 >= p.e_split;  // whole M tiles are q_C or q_R
    for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + c0, v);
      tmem_wait_ld();
      if (nkb == 0) {
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = 0u;
      }
      if (p.epi == EPI_PARTIAL) {
        if (m < p.m_total) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = n_base + c0 + c;
            if (c0 + c < p.n_tile && n < p.n_total) out[static_cast<int64_t>(n) * p.m_total + m] = __uint_as_float(v[c]);
          }
        }
      } else if (p.epi == EPI_BF16) {
        if (m < p.m_total) {
          __nv_bfloat16 *d = p.dst + batch * p.e_bs + m;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int n = n_base + c0 + c;
            if (c0 + c < p.n_tile && n < p.n_total) d[n * p.e_ns] = __float2bfloat16_rn(__uint_as_float(v[c]));
          }
        }
      } else if (!rope_tile) {
        const int64_t qrow = static_cast<int64_t>(p.n_h) * (p.d_c + p.d_r);
        const int64_t qa_off = static_cast<int64_t>(m / max(p.d_c, 1)) * (p.d_c + p.d_r) + m % max(p.d_c, 1);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int n = n_base + c0 + c;
          if (c0 + c < p.n_tile && n < p.n_total) {
            const __nv_bfloat16 x = __float2bfloat16_rn(__uint_as_float(v[c]));
            if (p.epi == EPI_QA) p.q[n * qrow + qa_off] = x;
            else p.dst[static_cast<int64_t>(n) * p.e_split + m] = x;
          }
        }
      } else {
        // q_R rows: lanes (2k, 2k+1) hold the RoPE pair (x[2i], x[2i+1]); the
        // angle depends on the token only through its position
        const int r = m - p.e_split, h = r / p.d_r, i = r % p.d_r;
        const bool odd = (i & 1) != 0;
        const double theta = rope_theta(i >> 1, p.d_r, p.rope_base);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int n = n_base + c0 + c;
          const float mine = __uint_as_float(v[c]);
          const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
          if (c0 + c < p.n_tile && n < p.n_total) {
            float x0 = odd ? other : mine, x1 = odd ? mine : other;
            rope_rotate(x0, x1, p.positions[n], theta);
            p.q[(static_cast<int64_t>(n) * p.n_h + h) * (p.d_c + p.d_r) + p.d_c + i] = __float2bfloat16_rn(odd ? x1 : x0);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc<1>(tmem, tmem_cols);
}

// ------------------------------------------------ fused per-head absorb ----
//
// For one head h (one CTA), T <= 128 token rows:
//   q_C,h = W_UQ_h c_Q   (128 x T)  -> bf16, kept in shared memory
//   q_R,h = W_QR_h c_Q   ( 64 x T)  -> RoPE at positions[t] -> q[t][h][d_c + i]
//   q_lat,h = W_UK_h^T q_C,h (512 x T) -> q[t][h][j]
// (MLA walk-through, section 1 step 3 and section 3 order B; DeepSeek-V2
// explainer, eqs. 12-13.) Every CTA streams its head's 192 + 128 weight rows
// once; q_C never leaves the SM. A stage holds the W_UQ box (128 rows), the
// W_QR box (64 rows) and the c_Q box back to back; the q_R product runs as an
// M = 128 MMA whose upper 64 rows read the c_Q box (or, for a small c_Q box,
// whatever follows it in shared memory) into accumulator rows that are
// discarded. Packing the 64-row box keeps 24 KB of weights in every 32 KB
// stage (at T = 64), so six stages fit. While product 1 streams, the epilogue
// warps fill a table of the RoPE cosines and sines of every (token, pair), so
// that rotating q_R after it costs a few multiplies per element.
namespace ab {
constexpr int A_BYTES = BM * BK * 2;  // 16 KB: a 128-row A tile (or two 64 x 64 W_UK^T boxes)
constexpr int QR_BYTES = 64 * BK * 2;  // 8 KB
// 8 warps: TMA producers 0, 6 and 7 (stage s is issued by producer s % 3), the
// MMA warp 1, and the epilogue warps 2-5 (warp w reaches tensor-memory lanes
// 32 (w % 4) .. + 31). A TMA instruction holds its issuing thread for a few
// hundred ns, so one producer alone would cap the stage rate.
constexpr int NUM_THREADS = 256;
struct Params {
  int T, n_tile, n_h, d_c, d_r, k_blocks;  // k_blocks = d_cq / 64
  int stages, stage_bytes, col_stride;      // col_stride: TMEM columns per accumulator
  __nv_bfloat16 *q;                         // [T][n_h][d_c + d_r]
  const int32_t *positions;
  double rope_base;
  int prefetch;  // launched with launch overlap: weight boxes of the first stages go out before griddep_wait
};
constexpr int RPAIRS = 32;  // RoPE pairs (d_R = 64)
__host__ __device__ inline int b2_bytes(int n_tile) { return ((n_tile + 63) / 64) * 128 * 128; }
__host__ __device__ inline int tab_bytes(int n_tile) { return n_tile * RPAIRS * 8; }  // float2 (cos, sin) [t][pair]
inline int stage_bytes(int n_tile) { return A_BYTES + QR_BYTES + n_tile * BK * 2; }
inline int stages(int n_tile) {
  const int budget = 224 * 1024 - b2_bytes(n_tile) - tab_bytes(n_tile);
  const int s = budget / stage_bytes(n_tile);
  return s > 8 ? 8 : s;
}
inline size_t smem(int n_tile, int st) {
  return static_cast<size_t>(st) * stage_bytes(n_tile) + b2_bytes(n_tile) + tab_bytes(n_tile) + 8 * (2 * st + 3) + 16 +
         1024;
}
}  // namespace ab

__global__ void __launch_bounds__(ab::NUM_THREADS, 1)
    k_absorb_head(const __grid_constant__ CUtensorMap tm_uq, const __grid_constant__ CUtensorMap tm_qr,
                  const __grid_constant__ CUtensorMap tm_cq, const __grid_constant__ CUtensorMap tm_uk,
                  const ab::Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x;
  const uint32_t b2 = sbase + p.stages * p.stage_bytes;  // q_C,h as the MN-major B of the second product
  float2 *rope_tab = reinterpret_cast<float2 *>(smem + p.stages * p.stage_bytes + ab::b2_bytes(p.n_tile));
  const uint32_t bars = b2 + ab::b2_bytes(p.n_tile) + ab::tab_bytes(p.n_tile);
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (p.stages + s); };
  const uint32_t p1_done = bars + 8u * (2 * p.stages), b2_full = p1_done + 8, p2_done = p1_done + 16;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + p.stages * p.stage_bytes + ab::b2_bytes(p.n_tile) +
                                                     ab::tab_bytes(p.n_tile) + 8 * (2 * p.stages + 3));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int n_p2 = 4 * 2;  // second product: 4 M tiles (512 latent rows) x 2 K blocks (d_h = 128)

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(p1_done, 1);
    mbar_init(b2_full, 4);
    mbar_init(p2_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<1>(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0 || warp >= 6) {
    // ------------------------------------------------------- TMA producers
    // Under launch overlap the first stages are armed together by producer 0
    // and their weight boxes issued by lanes l (W_UQ or W_UK box 0) and 8 + l
    // (W_QR or W_UK box 1) before the wait for the previous kernel on the
    // stream; their c_Q boxes (lane l) only after it. Every later use of stage
    // s goes out from producer s % 3, in order (so each stage's empty-barrier
    // waits are made by one warp): lane 0 waits and arms, lanes 0-2 issue.
    const int pid = warp == 0 ? 0 : warp - 5;
    const int total = p.k_blocks + n_p2;
    const int pre = p.prefetch ? min(total, p.stages) : 0;  // stages <= 8
    auto stage_tx = [&](int g) { return g < p.k_blocks ? ab::A_BYTES + ab::QR_BYTES + p.n_tile * BK * 2 : ab::A_BYTES; };
    auto issue_w = [&](int g, int box) {  // weight box `box` (0, 1) of item g
      const int s = g % p.stages;
      const uint32_t st = sbase + s * p.stage_bytes;
      if (g < p.k_blocks) {
        if (box == 0) tma_load_2d(st, &tm_uq, g * BK, head * BM, full(s));
        else tma_load_2d(st + ab::A_BYTES, &tm_qr, g * BK, head * p.d_r, full(s));
      } else {
        // W_UK_h^T tile: latent columns [128 mt + 64 box, +64) of k rows [64 kb, +64)
        const int u = g - p.k_blocks, mt = u >> 1, kb = u & 1;
        tma_load_2d(st + box * (ab::A_BYTES / 2), &tm_uk, BM * mt + 64 * box, head * BM + 64 * kb, full(s));
      }
    };
    auto issue_cq = [&](int g) {
      const int s = g % p.stages;
      tma_load_2d(sbase + s * p.stage_bytes + ab::A_BYTES + ab::QR_BYTES, &tm_cq, g * BK, 0, full(s));
    };
    if (pid == 0) {
      if (lane == 0)
        for (int g = 0; g < pre; ++g) mbar_arrive_expect_tx(full(g), stage_tx(g));
      __syncwarp();
      if (lane < pre) issue_w(lane, 0);
      else if (lane >= 8 && lane - 8 < pre) issue_w(lane - 8, 1);
    }
    griddep_wait();
    if (pid == 0 && lane < pre && lane < p.k_blocks) issue_cq(lane);
    __syncwarp();
    int g = pre;
    for (; g < total; ++g) {
      const int s = g % p.stages;
      if (s % PRODUCERS != pid) continue;
      const bool first = g < p.k_blocks;
      bool good = true;
      if (lane == 0) {
        if (g >= p.stages) good = mbar_wait(empty(s), ((g / p.stages) - 1) & 1, abort_flag);
        if (good) mbar_arrive_expect_tx(full(s), stage_tx(g));
      }
      if (!__shfl_sync(0xffffffffu, good, 0)) break;
      if (lane < 2) issue_w(g, lane);
      else if (lane == 2 && first) issue_cq(g);
      __syncwarp();
    }
    if (lane == 0)  // drain: the MMA commits to this producer's empty barriers have landed
      for (int q = g - p.stages; q < g; ++q)
        if (q >= 0 && (q % p.stages) % PRODUCERS == pid) mbar_wait(empty(q % p.stages), (q / p.stages) & 1, abort_flag);
  } else if (warp == 1 && lane == 0) {
    // --------------------------------------------------------- MMA issuer
    const uint32_t id1 = idesc_bf16(BM, p.n_tile, false, false);
    const uint32_t id2 = idesc_bf16(BM, p.n_tile, true, true);
    const uint32_t d1 = tmem, d2 = tmem + p.col_stride;
    int g = 0;
    bool ok = true;
    for (; g < p.k_blocks && ok; ++g) {
      const int s = g % p.stages;
      if (!mbar_wait(full(s), (g / p.stages) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t st = sbase + s * p.stage_bytes;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t bd = sdesc_sw128(st + ab::A_BYTES + ab::QR_BYTES + kk * 32, 16, 1024);
        tc_mma<1>(d1, sdesc_sw128(st + kk * 32, 16, 1024), bd, id1, (g > 0 || kk > 0) ? 1u : 0u);
        tc_mma<1>(d2, sdesc_sw128(st + ab::A_BYTES + kk * 32, 16, 1024), bd, id1, (g > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(empty(s));
    }
    tc_commit(p1_done);
    // second product once q_C,h sits in shared memory (and d1, d2 are drained)
    if (ok && mbar_wait(b2_full, 0, abort_flag)) {
      tc_fence_after();
      for (int u = 0; u < n_p2; ++u, ++g) {
        const int s = g % p.stages, mt = u >> 1, kb = u & 1;
        if (!mbar_wait(full(s), (g / p.stages) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t st = sbase + s * p.stage_bytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma<1>(tmem + mt * p.col_stride, sdesc_sw128(st + kk * 2048, ab::A_BYTES / 2, 1024),
                    sdesc_sw128(b2 + kb * 8192 + kk * 2048, 128 * 128, 1024), id2, (kb > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty(s));
      }
    }
    tc_commit(p2_done);
  } else if (warp >= 2 && warp < 6) {
    // ----------------------------------------------------------- epilogue
    const int sp = warp & 3;
    const int row = 32 * sp + lane;  // accumulator row of this thread
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * sp) << 16);
    const int64_t q_row = static_cast<int64_t>(p.n_h) * (p.d_c + p.d_r);  // q elements per token
    griddep_wait();  // positions are read and q written only once the previous kernel has finished
    // RoPE table while product 1 streams: (cos, sin) of token t, pair i
    for (int e = threadIdx.x - 64; e < p.n_tile * ab::RPAIRS; e += 128) {
      const int t = e / ab::RPAIRS, i = e % ab::RPAIRS;
      float c = 1.f, s = 0.f;
      if (t < p.T) rope_cos_sin(p.positions[t], rope_theta(i, p.d_r, p.rope_base), c, s);
      rope_tab[e] = make_float2(c, s);
    }
    named_bar_sync(1, 128);  // the four epilogue warps
    mbar_wait_warp(p1_done, 0, abort_flag);
    tc_fence_after();
    // q_C,h row `row` -> B2 (MN-major, 128-byte swizzle): k = row, n = token
    for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(lane_addr + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {  // 8 tokens per 16-byte chunk
        const int t0 = c0 + 8 * ch;
        if (t0 >= p.n_tile) break;
        const uint32_t w0 = pack_bf16x2(__uint_as_float(v[8 * ch]), __uint_as_float(v[8 * ch + 1]));
        const uint32_t w1 = pack_bf16x2(__uint_as_float(v[8 * ch + 2]), __uint_as_float(v[8 * ch + 3]));
        const uint32_t w2 = pack_bf16x2(__uint_as_float(v[8 * ch + 4]), __uint_as_float(v[8 * ch + 5]));
        const uint32_t w3 = pack_bf16x2(__uint_as_float(v[8 * ch + 6]), __uint_as_float(v[8 * ch + 7]));
        const int a = t0 >> 6, c16 = (t0 & 63) >> 3;
        uint8_t *dst = smem + (b2 - sbase) + a * (128 * 128) + (row >> 3) * 1024 + (row & 7) * 128 + ((c16 ^ (row & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst) = make_uint4(w0, w1, w2, w3);
      }
    }
    // q_R,h rows 0..63 (warps of sub-partitions 0, 1): lanes (2k, 2k+1) hold a
    // RoPE pair. The second product overwrites q_R's accumulator, so up to 64
    // tokens are read into registers first and the shared q_C is released
    // before they are rotated and stored; larger tiles rotate before release.
    const bool odd = (row & 1) != 0;
    auto rotate_store = [&](const uint32_t (&v)[32], int c0) {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int t = c0 + c;
        const float mine = __uint_as_float(v[c]);
        const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
        if (t < p.T) {
          float x0 = odd ? other : mine, x1 = odd ? mine : other;
          const float2 cs = rope_tab[t * ab::RPAIRS + (row >> 1)];
          rope_apply(x0, x1, cs.x, cs.y);
          p.q[t * q_row + static_cast<int64_t>(head) * (p.d_c + p.d_r) + p.d_c + row] = __float2bfloat16_rn(odd ? x1 : x0);
        }
      }
    };
    const bool early = p.n_tile <= 64;
    uint32_t qr[2][32];
    if (sp < 2) {
      if (early) {
        tmem_ld32(lane_addr + p.col_stride, qr[0]);
        if (p.n_tile > 32) tmem_ld32(lane_addr + p.col_stride + 32, qr[1]);
        tmem_wait_ld();
      } else {
        for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
          tmem_ld32(lane_addr + p.col_stride + c0, qr[0]);
          tmem_wait_ld();
          rotate_store(qr[0], c0);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(b2_full);
    if (sp < 2 && early) {
      rotate_store(qr[0], 0);
      if (p.n_tile > 32) rotate_store(qr[1], 32);
    }
    // q_lat,h: rows 128 mt + row of the second product
    mbar_wait_warp(p2_done, 0, abort_flag);
    tc_fence_after();
    for (int mt = 0; mt < 4; ++mt) {
      const int j = BM * mt + row;
      for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_addr + mt * p.col_stride + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int t = c0 + c;
          if (t < p.T) p.q[t * q_row + static_cast<int64_t>(head) * (p.d_c + p.d_r) + j] = __float2bfloat16_rn(__uint_as_float(v[c]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc<1>(tmem, 512);
}

// ------------------------------------------- batched GEMM, resident A ----
//
// For batch b (weight matrix W = A map 0 for b < split, A map 1 otherwise;
// head h = b mod split): out_b[n][m] = sum_k W[h * 128 + m][k] X[n][k], m <
// 128, n < N, k < K (a multiple of 64, 192 <= K <= 512), bf16 out, fp32
// accumulation. This is the decompression of order A (MLA walk-through,
// section 3 order A: K_C,h = W_UK,h c_KV and V_h = W_UV,h c_KV for every
// cached row; X = the c_KV columns of the cache rows), a long run of tiles
// that share A within a batch and X across batches.
//
// A pair of SMs (a 2-CTA cluster) takes batches 2c and 2c + 1 together: CTA r
// keeps batch 2c + r's A (128 x K, up to 128 KB) in shared memory and loads
// rows [128 r, 128 r + 128) of each 256-row X tile, and one
// tcgen05.mma.cta_group::2 with M = 256, N = 256 multiplies both heads by the
// whole tile, so every X byte read serves two heads. Each cluster takes a
// contiguous range of (batch pair, 256-row tile) units; X half-tiles stream
// through a six-slot ring, and two tensor-memory accumulators alternate so
// that the epilogue of one tile overlaps the MMAs of the next. Eight epilogue
// warps, two per tensor-memory sub-partition (one per half of the columns),
// drain a tile in about half the time the MMAs of the next one take.
namespace rs {
// warps: producers 0, 6, 7; MMA 1; epilogue 2-5 and 8-11 (warp w reaches lanes 32 (w % 4) .. + 31)
constexpr int KBLK_MAX = 8, NT = 256, NHALF = 128, STAGES = 6, NUM_THREADS = 384, EPI_WARPS = 8;
constexpr int A_BLK = BM * BK * 2;       // 16 KB: 128 rows x 64 k
constexpr int B_STAGE = NHALF * BK * 2;  // 16 KB: this CTA's 128 rows x 64 k
constexpr int OFF_B = KBLK_MAX * A_BLK, OFF_BAR = OFF_B + STAGES * B_STAGE;
constexpr int BAR_A_FULL = 0, BAR_A_EMPTY = 1, BAR_B_FULL = 2, BAR_B_EMPTY = BAR_B_FULL + STAGES,
              BAR_ACC_FULL = BAR_B_EMPTY + STAGES, BAR_ACC_EMPTY = BAR_ACC_FULL + 2, BAR_EXIT = BAR_ACC_EMPTY + 2,
              NUM_BARS = BAR_EXIT + 1;
constexpr int SMEM_BYTES = OFF_BAR + 8 * NUM_BARS + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "resident-A GEMM shared memory budget");
static_assert(STAGES % PRODUCERS == 0, "each producer owns whole ring slots");
struct Params {
  int batches, split;  // batches (even) < split read A map 0, the rest A map 1
  int n_tiles, N;      // 256-row tiles per batch, rows of X
  int kblk;            // K / 64
  __nv_bfloat16 *out0, *out1;  // [split][N][128] each
};
}  // namespace rs

__global__ void __launch_bounds__(rs::NUM_THREADS, 1) __cluster_dims__(2, 1, 1)
    k_gemm_resident(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                    const __grid_constant__ CUtensorMap tm_x, const rs::Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bars = sbase + rs::OFF_BAR;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  auto lead = [&](int i) { return rank == 0 ? bar(i) : mapa_shared(bar(i), 0); };  // the leader CTA's barrier
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + rs::OFF_BAR + 8 * rs::NUM_BARS);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int units = (p.batches / 2) * p.n_tiles, cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int u0 = static_cast<int>(static_cast<int64_t>(cluster) * units / nclusters);
  const int u1 = static_cast<int>(static_cast<int64_t>(cluster + 1) * units / nclusters);
  auto pair_start = [&](int u) { return u == u0 || u % p.n_tiles == 0; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < rs::NUM_BARS; ++i)
      mbar_init(bar(i), i == rs::BAR_ACC_EMPTY || i == rs::BAR_ACC_EMPTY + 1 ? 2 * rs::EPI_WARPS : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<2>(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers initialised and tensor memory allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 0 || warp == 6 || warp == 7) {
    // ---------------------------------------------------------- producers
    // Producer q owns ring slots q and q + 3 of this CTA. The A boxes of a
    // batch are shared out (kb = q, q + 3, ..), each producer waiting for the
    // previous A to be released, so every A phase needs every producer and
    // each wait is exact. Loads complete on the leader CTA's full barriers,
    // which the leader's producer 0 (A) or slot owner (X) arms for both CTAs.
    const int pid = warp == 0 ? 0 : warp - 5;
    griddep_wait();  // the cache rows may come from the kernel ahead on the stream
    if (lane == 0) {
      int na = 0, g = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u) {
        const int bp = u / p.n_tiles, nt = u % p.n_tiles, b = 2 * bp + static_cast<int>(rank);
        if (pair_start(u)) {
          if (na > 0) ok = mbar_wait(bar(rs::BAR_A_EMPTY), (na - 1) & 1, abort_flag);
          if (!ok) break;
          if (pid == 0 && rank == 0) mbar_arrive_expect_tx(bar(rs::BAR_A_FULL), 2 * p.kblk * rs::A_BLK);
          const CUtensorMap *am = b < p.split ? &tm_a0 : &tm_a1;
          const int h = b < p.split ? b : b - p.split;
          for (int kb = pid; kb < p.kblk; kb += PRODUCERS)
            tma_load_2d_pair(sbase + kb * rs::A_BLK, am, kb * BK, h * BM, lead(rs::BAR_A_FULL));
          ++na;
        }
        for (int kb = 0; kb < p.kblk; ++kb, ++g) {
          const int s = g % rs::STAGES, use = g / rs::STAGES;
          if (s % PRODUCERS != pid) continue;
          if (use > 0 && !(ok = mbar_wait(bar(rs::BAR_B_EMPTY + s), (use - 1) & 1, abort_flag))) break;
          if (rank == 0) mbar_arrive_expect_tx(bar(rs::BAR_B_FULL + s), 2 * rs::B_STAGE);
          tma_load_2d_pair(sbase + rs::OFF_B + s * rs::B_STAGE, &tm_x, kb * BK, nt * rs::NT + rs::NHALF * rank,
                           lead(rs::BAR_B_FULL + s));
        }
      }
      // drain: the releases of this producer's last slot uses and of the last A have arrived
      for (int sl = pid; ok && sl < rs::STAGES; sl += PRODUCERS) {
        const int uses = g > sl ? (g - sl + rs::STAGES - 1) / rs::STAGES : 0;
        if (uses > 0) ok = mbar_wait(bar(rs::BAR_B_EMPTY + sl), (uses - 1) & 1, abort_flag);
      }
      if (ok && na > 0) mbar_wait(bar(rs::BAR_A_EMPTY), (na - 1) & 1, abort_flag);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * BM, rs::NT, false, false);
      const uint64_t a0 = sdesc_sw128(sbase, 16, 1024);
      int na = 0, g = 0, lt = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok; ++u, ++lt) {
        if (pair_start(u)) {
          if (!(ok = mbar_wait(bar(rs::BAR_A_FULL), na & 1, abort_flag))) break;
          ++na;
        }
        const int buf = lt & 1;
        if (lt >= 2 && !(ok = mbar_wait(bar(rs::BAR_ACC_EMPTY + buf), ((lt >> 1) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        for (int kb = 0; kb < p.kblk; ++kb, ++g) {
          const int s = g % rs::STAGES;
          if (!(ok = mbar_wait(bar(rs::BAR_B_FULL + s), (g / rs::STAGES) & 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t bd = sdesc_sw128(sbase + rs::OFF_B + s * rs::B_STAGE, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma<2>(tmem + 256 * buf, sdesc_advance(a0, kb * rs::A_BLK + kk * 32), sdesc_advance(bd, kk * 32), idesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit_pair(bar(rs::BAR_B_EMPTY + s), 0x3);
        }
        if (!ok) break;
        tc_commit_pair(bar(rs::BAR_ACC_FULL + buf), 0x3);
        if (u + 1 == u1 || (u + 1) % p.n_tiles == 0) tc_commit_pair(bar(rs::BAR_A_EMPTY), 0x3);
      }
    }
  } else if ((warp >= 2 && warp < 6) || warp >= 8) {
    // ----------------------------------------------------------- epilogue
    const int sp = warp & 3, m = 32 * sp + lane;  // accumulator row (lane) = output column m of this CTA's head
    const int cbeg = warp >= 8 ? rs::NT / 2 : 0;  // this warp's half of the tile's columns (tokens)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * sp) << 16);
    griddep_wait();  // outputs are written only once the previous kernel has finished
    int lt = 0;
    for (int u = u0; u < u1; ++u, ++lt) {
      const int bp = u / p.n_tiles, nt = u % p.n_tiles, b = 2 * bp + static_cast<int>(rank), buf = lt & 1;
      mbar_wait_warp(bar(rs::BAR_ACC_FULL + buf), (lt >> 1) & 1, abort_flag);
      tc_fence_after();
      __nv_bfloat16 *out = (b < p.split ? p.out0 : p.out1) +
                           static_cast<int64_t>(b < p.split ? b : b - p.split) * p.N * BM;
      for (int c0 = cbeg; c0 < cbeg + rs::NT / 2; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(lane_addr + 256 * buf + c0, v);
        tmem_wait_ld();
        const int n0 = nt * rs::NT + c0;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (n0 + c < p.N) out[static_cast<int64_t>(n0 + c) * BM + m] = __float2bfloat16_rn(__uint_as_float(v[c]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(bar(rs::BAR_ACC_EMPTY + buf));
        else mbar_arrive_cluster(mapa_shared(bar(rs::BAR_ACC_EMPTY + buf), 0));
      }
    }
  }
  // ---- teardown: both CTAs done with each other's barriers, then free TMEM
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(mapa_shared(bar(rs::BAR_EXIT), rank ^ 1));
    mbar_wait(bar(rs::BAR_EXIT), 0, nullptr);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<2>(tmem, 512);
}

// ---------------------------------------------------------- finalizers ----

__device__ __forceinline__ float2 sum_splits2(const float *part, int splits, int64_t stride, int64_t idx) {
  // all loads of a batch of 8 splits are issued before any of them is used
  float2 acc = make_float2(0.f, 0.f);
  for (int s0 = 0; s0 < splits; s0 += 8) {
    float2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = s0 + u < splits ? __ldcg(reinterpret_cast<const float2 *>(part + (s0 + u) * stride + idx)) : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      acc.x += v[u].x;
      acc.y += v[u].y;
    }
  }
  return acc;
}

// rows [T][576] = sum of splits; RoPE on [512, 576); bf16; store at the
// cache row of (seq_idx[t], positions[t]). grid (ceil(D / 256), T), one
// thread per element pair.
__global__ void k_fin_append(const float *part, int splits, int T, int d_c, int d_r, double rope_base,
                             const int32_t *seq_idx, const int32_t *positions, CacheView cache) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.y;
  const int D = d_c + d_r;
  const int e = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (e >= D) return;
  const int64_t stride = static_cast<int64_t>(T) * D;
  const int pos = positions[t];
  const int64_t row = cache_row(cache, seq_idx[t], pos);
  if (row < 0) {
    if (e == 0) dev_error(MLA_DEVERR_DATA);
    return;
  }
  __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(cache.data) + row * D;
  const float2 x = sum_splits2(part, splits, stride, static_cast<int64_t>(t) * D + e);
  float x0 = x.x, x1 = x.y;
  if (e >= d_c) rope_pair(x0, x1, (e - d_c) / 2, d_r, pos, rope_base);
  *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(x0, x1);
}

// Finalize of the fused front end: the split sums of the stacked product
// [W_DKV; W_KR; W_DQ] h (partials [split][T][m_total]). Rows [0, d_c + d_r)
// are the append (RoPE on [d_c, d_c + d_r), bf16, stored at the cache row of
// (seq_idx[t], positions[t])); rows [cq_row, cq_row + d_cq) are c_Q (bf16 into
// cq[t][.]). grid (ceil((d_c + d_r + d_cq) / 256), T), one thread per pair.
__global__ void k_fin_front(const float *part, int splits, int T, int m_total, int d_c, int d_r, int cq_row,
                            int d_cq, double rope_base, const int32_t *seq_idx, const int32_t *positions,
                            CacheView cache, __nv_bfloat16 *cq) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.y;
  const int D = d_c + d_r;
  const int e = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (e >= D + d_cq) return;
  const int64_t stride = static_cast<int64_t>(T) * m_total;
  if (e >= D) {
    const int c = e - D;
    const float2 x = sum_splits2(part, splits, stride, static_cast<int64_t>(t) * m_total + cq_row + c);
    *reinterpret_cast<uint32_t *>(cq + static_cast<int64_t>(t) * d_cq + c) = pack_bf16x2(x.x, x.y);
    return;
  }
  const int pos = positions[t];
  const int64_t row = cache_row(cache, seq_idx[t], pos);
  if (row < 0) {
    if (e == 0) dev_error(MLA_DEVERR_DATA);
    return;
  }
  __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(cache.data) + row * D;
  const float2 x = sum_splits2(part, splits, stride, static_cast<int64_t>(t) * m_total + e);
  float x0 = x.x, x1 = x.y;
  if (e >= d_c) rope_pair(x0, x1, (e - d_c) / 2, d_r, pos, rope_base);
  *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(x0, x1);
}

// dst[t][n] (bf16, row pitch ld) = sum of splits of part[.][t][n], n < N.
__global__ void k_fin_store(const float *part, int splits, int T, int N, __nv_bfloat16 *dst, int64_t ld) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();
  const int64_t stride = static_cast<int64_t>(T) * N;
  for (int64_t i = 2 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); i < stride;
       i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / N, n = i % N;
    const float2 x = sum_splits2(part, splits, stride, i);
    *reinterpret_cast<uint32_t *>(dst + t * ld + n) = pack_bf16x2(x.x, x.y);
  }
}

// Split-K choice: about one CTA per SM, at least 4 K blocks per split.
inline int choose_splits(int tiles, int k_blocks, int sms) {
  int s = (sms + tiles - 1) / tiles;
  s = s < 1 ? 1 : s;
  const int max_s = k_blocks >= 8 ? k_blocks / 4 : 1;
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

// Pipeline depth: a launch that fits in one wave runs one CTA per SM and may
// keep ~200 KB of stages in flight; larger launches fit two CTAs per SM
// (~100 KB each) when three stages fit in that, else one CTA per SM again.
inline int stages_for(int n_tile, int ctas, int sms) {
  const int stage = A_STAGE + b_stage_bytes(n_tile);
  // two CTAs per SM only while each still gets three stages; otherwise one
  // CTA per SM keeps as many stages in flight as ~200 KB allow
  const bool two = ctas > sms && 3 * stage <= 100 * 1024;
  int s = (two ? 100 : 200) * 1024 / stage;
  const int max_s = two ? 8 : 12;
  return s > max_s ? max_s : (s < 3 ? 3 : s);
}

inline size_t smem_for(int n_tile, int stages) {
  return static_cast<size_t>(stages) * (A_STAGE + b_stage_bytes(n_tile)) + 8 * (2 * stages + 1) + 16 + 1024;
}

}  // namespace gemm
}  // namespace mla
