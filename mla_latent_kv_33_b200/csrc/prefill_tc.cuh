// Order A of MLA attention on sm_100a tensor cores (MLA walk-through,
// h.sjds.net, section 3 order A, the training form: decompress, then the
// ordinary dot product; MLA wiki, the per-head K/V of MHA rebuilt from the
// latent). For head h and cached position i of sequence b:
//   K_h,i = [W_UK_h c_KV_i ; k_R,i]  (d_h + d_R = 192),  V_h,i = W_UV_h c_KV_i  (d_h = 128),
// and for token row t = b n_q + j at position L_b - n_q + j (causal within the
// chunk of n_q new tokens):
//   o[t][h] = sum_i softmax_i(scale [q_C,h ; q_R,h] . K_h,i) V_h,i,  i <= L_b - n_q + j.
//
// The decompressed K_C = W_UK c_KV and V = W_UV c_KV come from the projection
// GEMM (one launch each, over every physical cache row) into the workspace,
// [n_h][rows][128] bf16. This kernel is the attention: one CTA per (head,
// sequence, block of 128 query rows), 1-SM tcgen05 MMAs with M = 128 query
// rows:
//   S = Q K^T  (N = 128 keys, K = 192: 12 MMAs per key tile) into tensor memory,
//   online softmax by four warps (thread = query row = tensor-memory lane),
//   P written in bf16 over its scores and read as the A operand of
//   O += P V   (N = 128 = d_h, K = 128 keys: 8 MMAs; V as an MN-major B).
// Two S buffers let QK^T of tile i + 1 run while tile i's softmax runs. A key
// tile is two 64-row blocks (contiguous or paged); blocks wholly past the
// sequence end load at an out-of-range row (TMA zero fill); the rows past the
// end inside the last partial block are zeroed in the V tile before its PV
// (their scores are masked, but 0 * NaN would still poison O).
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace pre {

constexpr int DQK = 192, DV = 128, KTILE = 128, BLK = 64, QROWS = 128;
constexpr int NUM_THREADS = 256, WARP_PROD = 0, WARP_MMA = 1, WARP_SMX = 4;
constexpr int CHUNK = QROWS * 128;       // 128 rows x 64 columns bf16 (one swizzle-128 column)
constexpr int Q_BYTES = 3 * CHUNK;       // 48 KB
constexpr int K_BYTES = 3 * CHUNK;       // 48 KB: K_C chunks 0, 1 and the k_R chunk
constexpr int V_BYTES = 2 * CHUNK;       // 32 KB
constexpr int OFF_Q = 0, OFF_K = Q_BYTES, OFF_V = OFF_K + 2 * K_BYTES, OFF_BAR = OFF_V + 2 * V_BYTES;
constexpr int BAR_Q = 0, BAR_KF = 1, BAR_KE = 3, BAR_VF = 5, BAR_VE = 7, BAR_S = 9, BAR_P = 11, BAR_O = 12,
              BAR_Z = 13, NUM_BARS = 14;
constexpr int SMEM_BYTES = OFF_BAR + 8 * NUM_BARS + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "order-A attention shared memory budget");
constexpr uint32_t IDESC_S = idesc_bf16(QROWS, KTILE, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(QROWS, DV, false, true);
constexpr int S_COL = 0, O_COL = 256;  // tensor memory: S/P buffers at 0 and 128, O at 256
constexpr float RESCALE_LOG2 = 8.f;

struct Params {
  const int32_t *seq_lens;
  const int32_t *block_table;
  int64_t max_len, rows;  // rows: physical cache rows (TMA out-of-range coordinate)
  int32_t paged, block_size, max_blocks_per_seq, num_blocks_i32;
  int32_t B, n_q, n_h, qblocks;
  int64_t capacity;
  float scale_log2;
  __nv_bfloat16 *o;  // [B n_q][n_h][128]
};

// Physical row of the 64-row block holding position pos of sequence b, or
// p.rows (out of range: zero fill) past the end or on a bad table entry.
__device__ __forceinline__ int32_t block_row(const Params &p, int b, int64_t pos, int L) {
  if (pos >= L) return static_cast<int32_t>(p.rows);
  if (!p.paged) return static_cast<int32_t>(static_cast<int64_t>(b) * p.max_len + pos);
  const int32_t blk = p.block_table[static_cast<int64_t>(b) * p.max_blocks_per_seq + pos / p.block_size];
  if (blk < 0 || blk >= p.num_blocks_i32) {
    dev_error(MLA_DEVERR_DATA);
    return static_cast<int32_t>(p.rows);
  }
  return static_cast<int32_t>(static_cast<int64_t>(blk) * p.block_size + pos % p.block_size);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_attend_a(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
               const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bars = sbase + OFF_BAR;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8 * NUM_BARS);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  // work item: block of query rows, head, sequence (the query blocks of one
  // head and sequence are neighbours in the grid, so they run together and
  // read that head's K_C and V tiles from L2 rather than once each from HBM)
  const int qb = blockIdx.x % p.qblocks;
  const int h = (blockIdx.x / p.qblocks) % p.n_h;
  const int b = blockIdx.x / (p.qblocks * p.n_h);
  const int j0 = qb * QROWS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(bar(i), (i == BAR_P || i == BAR_Z) ? 4 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) tmem_alloc<1>(smem_u32(tmem_slot), 512);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kc);
    tma_prefetch_desc(&tm_kr);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();  // q, the cache, the decompressed K/V and seq_lens come from earlier kernels

  const int L = p.seq_lens[b];
  const bool bad = L < p.n_q || static_cast<int64_t>(L) > p.capacity;
  if (bad && threadIdx.x == 0 && h == 0 && qb == 0) dev_error(MLA_DEVERR_DATA);
  // keys visible to the last valid query row of this block
  const int jl = min(j0 + QROWS, p.n_q) - 1;
  const int kmax = bad || j0 >= p.n_q ? 0 : L - p.n_q + jl + 1;
  const int n = (kmax + KTILE - 1) / KTILE;  // key tiles (0: nothing to do)

  if (warp == WARP_PROD || warp == 2 || warp == 3) {
    // ----------------------------------------------------------- producers
    // TMA operations issued by one warp complete one after another, so the
    // loads of a key tile come from three warps: warp 0 loads Q and the K_C
    // chunks, warp 3 the k_R chunk (both fill the K slot: each waits for it
    // to be free, warp 0 arms it), warp 2 the V tile.
    const int role = warp == WARP_PROD ? 0 : (warp == 2 ? 1 : 2);  // 0: Q + K_C, 1: V, 2: k_R
    if (lane == 0 && n > 0) {
      bool ok = true;
      if (role == 0) {
        mbar_arrive_expect_tx(bar(BAR_Q), Q_BYTES);
        for (int c = 0; c < 3; ++c)  // q rows b n_q + j0 .. (+128), head h; rows past T read zeros
          tma_load_3d(sbase + OFF_Q + c * CHUNK, &tm_q, 64 * c, h, b * p.n_q + j0, bar(BAR_Q));
      }
      for (int i = 0; i < n && ok; ++i) {
        const int s = i & 1, use = i >> 1;
        int32_t r[2];
        for (int kb = 0; kb < 2; ++kb) r[kb] = block_row(p, b, static_cast<int64_t>(i) * KTILE + BLK * kb, L);
        if (role != 1) {
          if (use > 0 && !mbar_wait(bar(BAR_KE + s), (use - 1) & 1, abort_flag)) { ok = false; break; }
          const uint32_t kd = sbase + OFF_K + s * K_BYTES;
          if (role == 0) {
            mbar_arrive_expect_tx(bar(BAR_KF + s), K_BYTES);
            for (int kb = 0; kb < 2; ++kb)
              for (int c = 0; c < 2; ++c)
                tma_load_3d(kd + c * CHUNK + kb * (CHUNK / 2), &tm_kc, 64 * c, r[kb], h, bar(BAR_KF + s));
          } else {
            for (int kb = 0; kb < 2; ++kb)
              tma_load_2d(kd + 2 * CHUNK + kb * (CHUNK / 2), &tm_kr, 512, r[kb], bar(BAR_KF + s));
          }
        } else {
          if (use > 0 && !mbar_wait(bar(BAR_VE + s), (use - 1) & 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(BAR_VF + s), V_BYTES);
          const uint32_t vd = sbase + OFF_V + s * V_BYTES;
          for (int kb = 0; kb < 2; ++kb)
            for (int c = 0; c < 2; ++c)
              tma_load_3d(vd + c * CHUNK + kb * (CHUNK / 2), &tm_v, 64 * c, r[kb], h, bar(BAR_VF + s));
        }
      }
      // drain: the MMA's releases of the last use of each slot this warp fills have arrived
      for (int i = max(0, n - 2); ok && i < n; ++i)
        mbar_wait(bar((role != 1 ? BAR_KE : BAR_VE) + (i & 1)), (i >> 1) & 1, abort_flag);
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      bool ok = mbar_wait(bar(BAR_Q), 0, abort_flag);
      const uint64_t dq = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      auto qk = [&](int i) -> bool {
        const int s = i & 1;
        if (!mbar_wait(bar(BAR_KF + s), (i >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dk = sdesc_sw128(sbase + OFF_K + s * K_BYTES, 16, 1024);
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma<1>(tmem + S_COL + 128 * s, dq + static_cast<uint64_t>((c * CHUNK + kk * 32) >> 4),
                      dk + static_cast<uint64_t>((c * CHUNK + kk * 32) >> 4), IDESC_S, (c > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(BAR_KE + s));
        tc_commit(bar(BAR_S + s));
        return true;
      };
      auto pv = [&](int i) -> bool {
        const int s = i & 1;
        if (!mbar_wait(bar(BAR_VF + s), (i >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(bar(BAR_P), i & 1, abort_flag)) return false;
        if (i == n - 1 && !mbar_wait(bar(BAR_Z), 0, abort_flag)) return false;  // partial rows zeroed
        tc_fence_after();
        const uint64_t dv = sdesc_sw128(sbase + OFF_V + s * V_BYTES, CHUNK, 1024);
#pragma unroll
        for (int m = 0; m < KTILE / 16; ++m)
          tc_mma_ts<1>(tmem + O_COL, tmem + S_COL + 128 * s + 8 * m, dv + static_cast<uint64_t>((m * 2048) >> 4),
                       IDESC_PV, (i > 0 || m > 0) ? 1u : 0u);
        tc_commit(bar(BAR_VE + s));
        tc_commit(bar(BAR_O));
        return true;
      };
      for (int i = 0; i < n && ok; ++i) {
        if (!qk(i)) { ok = false; break; }
        if (i > 0 && !pv(i - 1)) { ok = false; break; }
      }
      if (ok) pv(n - 1);
    }
  } else if (warp >= WARP_SMX) {
    // ------------------------------------------------- softmax + epilogue
    // thread = query row r = tensor-memory lane; a failed wait does not break
    // the loop: every warp keeps the same sequence and the error word reports it
    const int r = 32 * (warp - WARP_SMX) + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * (warp - WARP_SMX)) << 16);
    const int j = j0 + r;
    const bool row_valid = j < p.n_q && !bad;
    const int pos = L - p.n_q + j;  // this row's position: keys 0 .. pos are visible
    const float c2 = p.scale_log2;
    float m_ref = -INFINITY, lsum = 0.f;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      mbar_wait_warp(bar(BAR_S + s), (i >> 1) & 1, abort_flag);
      tc_fence_after();
      const uint32_t s_addr = lane_addr + S_COL + 128 * s;
      uint32_t sr[128];
      tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
      const int k0 = i * KTILE;
      if (row_valid && pos - k0 < KTILE - 1) {  // causal edge (and the sequence end) in this tile
#pragma unroll
        for (int c = 0; c < KTILE; ++c)
          if (k0 + c > pos) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < KTILE; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
      bool rescale = false;
      float alpha = 1.f;
      if (i == 0) {
        m_ref = mx;  // key 0 is visible to every row: finite
      } else {
        const bool need = (mx - m_ref) * c2 > RESCALE_LOG2;
        rescale = __any_sync(0xffffffffu, need);
        if (need) {
          alpha = ex2_approx((m_ref - mx) * c2);
          m_ref = mx;
        }
      }
      const float mo = m_ref * c2;
      float ps = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 2; ++q4) {
        uint32_t pw[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[64 * q4 + 2 * c]), c2, -mo));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[64 * q4 + 2 * c + 1]), c2, -mo));
          ps += p0 + p1;
          pw[c] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_addr + 32 * q4, pw);  // P over the first 64 columns of its scores
      }
      tmem_wait_st();
      // P is released only after the previous tile's PV has finished (O may be
      // rescaled, and the MMA thread has consumed the previous P phase)
      if (i > 0) mbar_wait_warp(bar(BAR_O), (i - 1) & 1, abort_flag);
      tc_fence_after();
      if (rescale) {
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t o[32];
          tmem_ld32(lane_addr + O_COL + 32 * q4, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(lane_addr + O_COL + 32 * q4, o);
        }
        tmem_wait_st();
      }
      lsum = lsum * alpha + ps;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_P));
      if (i == n - 1) {
        // rows of the last tile past the sequence end: zero them in the V tile
        const int valid = L - k0;  // keys of this tile inside the sequence (1 .. 128 when not bad)
        mbar_wait_warp(bar(BAR_VF + s), (i >> 1) & 1, abort_flag);
        if (!bad && valid < KTILE && (valid % BLK) != 0) {
          uint8_t *vb = smem + OFF_V + s * V_BYTES;
          // V tile: [chunk c][128 keys][128 B]; zero keys valid .. end of their block
          const int end = (valid / BLK + 1) * BLK;
          const int tid = threadIdx.x - 32 * WARP_SMX;
          for (int e = tid; e < (end - valid) * 16; e += 128) {
            const int key = valid + e / 16, w16 = e & 15, c = w16 >> 3;
            *reinterpret_cast<uint4 *>(vb + c * CHUNK + key * 128 + (w16 & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_Z));
      }
    }
    // ---------------------------------------------------------- epilogue
    if (n > 0) {
      mbar_wait_warp(bar(BAR_O), (n - 1) & 1, abort_flag);
      tc_fence_after();
      const float inv = 1.f / lsum;
      __nv_bfloat16 *dst = p.o + (static_cast<int64_t>(b * p.n_q + j) * p.n_h + h) * DV;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t o[32];
        tmem_ld32(lane_addr + O_COL + 32 * q4, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4 *>(dst + 32 * q4 + 8 * u) =
                make_uint4(pack_bf16x2(__uint_as_float(o[8 * u]) * inv, __uint_as_float(o[8 * u + 1]) * inv),
                           pack_bf16x2(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv),
                           pack_bf16x2(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv),
                           pack_bf16x2(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_MMA) tmem_dealloc<1>(tmem, 512);
}

}  // namespace pre
}  // namespace mla
