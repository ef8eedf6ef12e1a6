// Absorbed-form MLA decode on sm_100a tensor cores (MLA walk-through,
// h.sjds.net, section 1 step 4 and section 3 order B).
//
// For every token row t (sequence b, new token j) and head h:
//   s_i = scale * (q_lat,h . c_KV_i + q_R,h . k_R_i) over the visible cached
//   positions i, p = softmax(s), o_lat = sum_i p_i c_KV_i, lse = log sum exp s.
//
// Design (B200, one GPU):
//  * All 128 heads of a token row share every cached row, so per 64-token
//    tile S = Q K^T is a dense 128 x 64 x 576 contraction and O += P V a dense
//    128 x 512 x 64 one. Both run as tcgen05.mma.cta_group::2 on a pair of
//    SMs (a 2-CTA cluster): CTA r holds heads 64r..64r+63 of Q, its half of
//    the tile's tokens for QK^T (B operand split by N = tokens) and all 64
//    tokens of its 256 latent columns for PV (B operand split by N = latent).
//    The 128 x 512 fp32 O accumulator is exactly one SM's tensor memory, so
//    splitting it over the pair (256 columns each) is what leaves room for
//    the double-buffered score tiles.
//  * Shared memory per CTA: Q 72 KB, two stages of (own tokens x 576 = 36 KB,
//    all tokens x own latent = 32 KB), two P tiles of 8 KB. The second copy
//    of latent columns is an L2 re-read; HBM sees each cached row once.
//  * Warp roles: warp 0 issues TMA loads (both CTAs), warp 1 of CTA 0 issues
//    the MMAs for the pair, warps 2-5 of both CTAs run the online softmax
//    (fp32, exp2, lazy rescaling of O when the running max grows by more
//    than 2^8) and the epilogue.
//  * Work: the visible tiles of all token rows are concatenated and cut into
//    equal contiguous ranges, one per cluster (persistent grid). A row whose
//    tiles fall in one range is finished in place (bf16 o_lat, lse); a row cut
//    by range boundaries leaves normalised fp32 partials that the combine
//    kernel merges with a log-sum-exp.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace dec {

constexpr int D = 576, DC = 512, DR = 64, HEADS = 128, HPC = 64;
constexpr int TILE = 64, OWN = 32;
constexpr int NS = 2;  // shared-memory stages
constexpr int NB = 2;  // score / P buffers
constexpr int NUM_THREADS = 192;
constexpr int CHUNK_Q = HPC * 128;   // 64 rows x 128 B
constexpr int CHUNK_KS = OWN * 128;  // 32 rows x 128 B
constexpr int CHUNK_V = TILE * 128;  // 64 rows x 128 B
constexpr int Q_BYTES = 9 * CHUNK_Q;
constexpr int KS_BYTES = 9 * CHUNK_KS;
constexpr int V_BYTES = 4 * CHUNK_V;
constexpr int P_BYTES = HPC * 128;
constexpr int OFF_Q = 0;
constexpr int OFF_KS = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_KS + NS * KS_BYTES;
constexpr int OFF_P = OFF_V + NS * V_BYTES;
constexpr int OFF_MISC = OFF_P + NB * P_BYTES;
// misc: barriers then exchange arrays
constexpr int BAR_Q_FULL = 0, BAR_Q_EMPTY = 1, BAR_KV_FULL = 2, BAR_KV_EMPTY = BAR_KV_FULL + NS,
              BAR_S_FULL = BAR_KV_EMPTY + NS, BAR_S_FREE = BAR_S_FULL + NB, BAR_P_FULL = BAR_S_FREE + NB,
              BAR_O_FULL = BAR_P_FULL + NB, BAR_O_FREE = BAR_O_FULL + NB, BAR_EXIT = BAR_O_FREE + 1,
              NUM_BARS = BAR_EXIT + 1;
constexpr int MISC_RED = 256;                 // float red[2][128]
constexpr int MISC_REDL = MISC_RED + 1024;    // float redl[128]
constexpr int MISC_INTS = MISC_REDL + 512;    // int scalars
constexpr int MISC_BYTES = MISC_INTS + 64;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "decode shared memory budget");
constexpr int MAX_UNITS = V_BYTES / 4 - 1;  // plan scratch aliases the second V stage
constexpr int S_COL = 256;                   // TMEM: O at [0,256), scores at [256, 256 + 32*NB)
constexpr uint32_t IDESC_S = idesc_bf16(128, TILE, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);
constexpr float RESCALE_LOG2 = 8.f;  // rescale O only when the max grows by more than 2^8

struct Params {
  const int32_t *seq_lens;
  const int32_t *block_table;
  int64_t max_len;
  int64_t cache_rows;  // rows addressable by the cache tensor map
  int32_t paged, block_size, max_blocks_per_seq, num_blocks_i32;
  int32_t B, n_q;
  int64_t capacity;  // max tokens per sequence
  float scale, scale_log2;
  __nv_bfloat16 *o_lat;
  float *lse;
  float *part_o;     // [slots][128][512]
  float *part_lse;   // [slots][128]
  int32_t *plan;     // [0] = W, [1] = Qt, [2..] = tile offsets [BJ + 1]
};

// Tiles visible to unit bj (token row): 0 if its sequence length is invalid.
__device__ __forceinline__ int unit_tiles(const Params &p, int bj, int *vis_out) {
  const int b = bj / p.n_q, j = bj % p.n_q;
  const int L = p.seq_lens[b];
  if (L < p.n_q || static_cast<int64_t>(L) > p.capacity) {
    *vis_out = 0;
    return -1;
  }
  const int vis = L - p.n_q + 1 + j;
  *vis_out = vis;
  return (vis + TILE - 1) / TILE;
}

// Physical cache row of the first token of tile `tile` of sequence b, or a
// row past the end of the tensor map (TMA zero-fills it) if the block table
// entry is out of range.
__device__ __forceinline__ int32_t tile_row(const Params &p, int b, int tile) {
  const int64_t pos = static_cast<int64_t>(tile) * TILE;
  if (!p.paged) return static_cast<int32_t>(static_cast<int64_t>(b) * p.max_len + pos);
  const int64_t bi = pos / p.block_size;
  const int32_t blk = p.block_table[static_cast<int64_t>(b) * p.max_blocks_per_seq + bi];
  if (blk < 0 || blk >= p.num_blocks_i32) {
    dev_error(MLA_DEVERR_DATA);
    return 0x7fffff00;
  }
  return static_cast<int32_t>(static_cast<int64_t>(blk) * p.block_size + pos % p.block_size);
}

struct Piece {
  int bj, t_begin, t_end, vis, nt;
  bool single;
  int slot;
};

// Iterates the pieces of this cluster's tile range in order.
struct PieceIter {
  int g, gend, bj, off, Qt, k;
  __device__ bool next(const Params &p, Piece &pc) {
    while (g < gend) {
      int vis;
      int nt = unit_tiles(p, bj, &vis);
      if (nt < 0) nt = 0;
      if (nt == 0 || off + nt <= g) {
        off += nt;
        ++bj;
        continue;
      }
      pc.bj = bj;
      pc.vis = vis;
      pc.nt = nt;
      pc.t_begin = g - off;
      const int e = min(gend, off + nt);
      pc.t_end = e - off;
      pc.single = (off / Qt) == ((off + nt - 1) / Qt);
      pc.slot = bj + k;
      g = e;
      off += nt;
      ++bj;
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ void arrive_leader(uint32_t bar_local, uint32_t rank) {
  if (rank == 0)
    mbar_arrive(bar_local);
  else
    mbar_arrive_cluster(mapa_shared(bar_local, 0));
}

__global__ void __launch_bounds__(NUM_THREADS, 1) __cluster_dims__(2, 1, 1)
    k_decode(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ks,
             const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  uint8_t *misc = smem + OFF_MISC;
  const uint32_t bars = sbase + OFF_MISC;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  float *red = reinterpret_cast<float *>(misc + MISC_RED);
  float *redl = reinterpret_cast<float *>(misc + MISC_REDL);
  int *ints = reinterpret_cast<int *>(misc + MISC_INTS);
  volatile int *abort_flag = ints + 0;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ints + 1);
  int *plan_s = ints + 2;  // W, Qt, bj_first, off_first

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q_FULL), 1);
    mbar_init(bar(BAR_Q_EMPTY), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(bar(BAR_S_FULL + b), 1);
      mbar_init(bar(BAR_S_FREE + b), 8);
      mbar_init(bar(BAR_P_FULL + b), 8);
      mbar_init(bar(BAR_O_FULL + b), 1);
    }
    mbar_init(bar(BAR_O_FREE), 8);
    mbar_init(bar(BAR_EXIT), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_ks);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc<2>(smem_u32(tmem_slot), 512);
  }

  // ---- plan: tiles per unit, prefix sums, this cluster's first unit ----
  const int BJ = p.B * p.n_q;
  int *scratch = reinterpret_cast<int *>(smem + OFF_V + V_BYTES);
  for (int u = threadIdx.x; u < BJ; u += NUM_THREADS) {
    int vis;
    int nt = unit_tiles(p, u, &vis);
    if (nt < 0) {
      if (blockIdx.x == 0 && (u % p.n_q) == 0) dev_error(MLA_DEVERR_DATA);
      nt = 0;
    }
    scratch[u] = nt;
  }
  __syncthreads();
  {
    // each thread scans a contiguous segment; block scan of the segment sums
    const int per = (BJ + NUM_THREADS - 1) / NUM_THREADS;
    const int lo = threadIdx.x * per, hi = min(BJ, lo + per);
    int sum = 0;
    for (int u = lo; u < hi; ++u) sum += scratch[u];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    __shared__ int warp_tot[NUM_THREADS / 32];
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
    int run = base + incl - sum;  // exclusive prefix of this segment
    for (int u = lo; u < hi; ++u) {
      const int nt = scratch[u];
      scratch[u] = run;
      run += nt;
    }
    if (threadIdx.x == NUM_THREADS - 1) {
      int W = 0;
      for (int w = 0; w < NUM_THREADS / 32; ++w) W += warp_tot[w];
      plan_s[0] = W;
      plan_s[1] = max(1, (W + nclusters - 1) / nclusters);
      plan_s[2] = BJ;  // bj_first (none yet)
      plan_s[3] = W;
    }
    __syncthreads();
    const int W = plan_s[0], Qt = plan_s[1];
    const int g0 = cluster * Qt;
    for (int u = lo; u < hi; ++u) {
      const int a = scratch[u];
      const int e = (u + 1 < BJ) ? scratch[u + 1] : W;
      if (a <= g0 && g0 < e) {
        plan_s[2] = u;
        plan_s[3] = a;
      }
    }
    if (blockIdx.x == 0) {
      for (int u = threadIdx.x; u < BJ; u += NUM_THREADS) p.plan[2 + u] = scratch[u];
      if (threadIdx.x == 0) {
        p.plan[0] = W;
        p.plan[1] = Qt;
        p.plan[2 + BJ] = W;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // peer barriers initialised, TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int W = plan_s[0], Qt = plan_s[1];
  PieceIter it0;
  it0.g = min(W, cluster * Qt);
  it0.gend = min(W, (cluster + 1) * Qt);
  it0.bj = plan_s[2];
  it0.off = plan_s[3];
  it0.Qt = Qt;
  it0.k = cluster;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      const uint32_t q_full = rank == 0 ? bar(BAR_Q_FULL) : mapa_shared(bar(BAR_Q_FULL), 0);
      uint32_t kv_full[NS];
      for (int s = 0; s < NS; ++s)
        kv_full[s] = rank == 0 ? bar(BAR_KV_FULL + s) : mapa_shared(bar(BAR_KV_FULL + s), 0);
      PieceIter it = it0;
      Piece pc;
      int gi = 0, npc = 0;
      bool ok = true;
      while (ok && it.next(p, pc)) {
        if (npc > 0 && !mbar_wait(bar(BAR_Q_EMPTY), (npc - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (rank == 0) mbar_arrive_expect_tx(bar(BAR_Q_FULL), 2 * Q_BYTES);
        for (int c = 0; c < 9; ++c)
          tma_load_2d_pair(sbase + OFF_Q + c * CHUNK_Q, &tm_q, 64 * c, pc.bj * HEADS + HPC * rank, q_full);
        const int b = pc.bj / p.n_q;
        for (int ti = pc.t_begin; ti < pc.t_end; ++ti, ++gi) {
          const int s = gi % NS;
          if (gi >= NS && !mbar_wait(bar(BAR_KV_EMPTY + s), ((gi / NS) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int32_t row0 = tile_row(p, b, ti);
          if (rank == 0) mbar_arrive_expect_tx(bar(BAR_KV_FULL + s), 2 * (KS_BYTES + V_BYTES));
          const uint32_t ks = sbase + OFF_KS + s * KS_BYTES;
          const uint32_t vv = sbase + OFF_V + s * V_BYTES;
          for (int c = 0; c < 9; ++c) tma_load_2d_pair(ks + c * CHUNK_KS, &tm_ks, 64 * c, row0 + OWN * rank, kv_full[s]);
          for (int c = 0; c < 4; ++c)
            tma_load_2d_pair(vv + c * CHUNK_V, &tm_v, 256 * (c >> 1) + 128 * rank + 64 * (c & 1), row0, kv_full[s]);
        }
        ++npc;
      }
      // drain: every commit aimed at this CTA's empty barriers has landed
      if (ok && npc > 0) mbar_wait(bar(BAR_Q_EMPTY), (npc - 1) & 1, abort_flag);
      for (int g = gi - NS; ok && g < gi; ++g)
        if (g >= 0) mbar_wait(bar(BAR_KV_EMPTY + g % NS), (g / NS) & 1, abort_flag);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (rank == 0 && lane == 0) {
      PieceIter it = it0;
      Piece pc;
      int gi = 0, npc = 0;
      bool ok = true;
      auto issue_pv = [&](int g, bool first) -> bool {
        const int b = g % NB, s = g % NS;
        if (!mbar_wait(bar(BAR_P_FULL + b), (g / NB) & 1, abort_flag)) return false;
        if (first && npc > 0 && !mbar_wait(bar(BAR_O_FREE), (npc - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t pbase = sbase + OFF_P + b * P_BYTES;
        const uint32_t vbase = sbase + OFF_V + s * V_BYTES;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(pbase + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(vbase + (2 * j) * CHUNK_V + kk * 2048, CHUNK_V, 1024);
            tc_mma<2>(tmem + 128 * j, ad, bd, IDESC_PV, (first && kk == 0) ? 0u : 1u);
          }
        tc_commit_pair(bar(BAR_O_FULL + b), 0x3);
        tc_commit_pair(bar(BAR_KV_EMPTY + s), 0x3);
        return true;
      };
      while (ok && it.next(p, pc)) {
        if (!mbar_wait(bar(BAR_Q_FULL), npc & 1, abort_flag)) {
          ok = false;
          break;
        }
        const int n = pc.t_end - pc.t_begin;
        for (int i = 0; i < n; ++i, ++gi) {
          const int s = gi % NS, b = gi % NB;
          if (!mbar_wait(bar(BAR_KV_FULL + s), (gi / NS) & 1, abort_flag)) { ok = false; break; }
          if (gi >= NB && !mbar_wait(bar(BAR_S_FREE + b), ((gi / NB) - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ks = sbase + OFF_KS + s * KS_BYTES;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int c = k >> 2, kk = k & 3;
            const uint64_t ad = sdesc_sw128(sbase + OFF_Q + c * CHUNK_Q + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(ks + c * CHUNK_KS + kk * 32, 16, 1024);
            tc_mma<2>(tmem + S_COL + 32 * b, ad, bd, IDESC_S, k > 0 ? 1u : 0u);
          }
          tc_commit_pair(bar(BAR_S_FULL + b), 0x3);
          if (i == n - 1) tc_commit_pair(bar(BAR_Q_EMPTY), 0x3);
          if (i > 0 && !issue_pv(gi - 1, i == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(gi - 1, n == 1)) { ok = false; break; }
        ++npc;
      }
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int sp = warp & 3;               // TMEM sub-partition of this warp
    const int L = 32 * sp + lane;          // TMEM lane
    const int row = L & 63, half = L >> 6;  // head within CTA, token / latent half
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * sp) << 16);
    const float c2 = p.scale_log2;
    PieceIter it = it0;
    Piece pc;
    int gi = 0;
    // A failed (timed-out) wait does not break these loops: every softmax
    // warp keeps the same sequence of named-barrier syncs and runs to the
    // end on whatever data is there; the device error word reports it.
    while (it.next(p, pc)) {
      const int n = pc.t_end - pc.t_begin;
      float m_ref = -INFINITY, lsum = 0.f;
      for (int i = 0; i < n; ++i, ++gi) {
        const int b = gi % NB, ti = pc.t_begin + i;
        mbar_wait_warp(bar(BAR_S_FULL + b), (gi / NB) & 1, abort_flag);
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(lane_addr + S_COL + 32 * b, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(bar(BAR_S_FREE + b), rank);
        float sv[32];
        const int tok0 = ti * TILE + OWN * half;
#pragma unroll
        for (int c = 0; c < 32; ++c) sv[c] = (tok0 + c < pc.vis) ? __uint_as_float(sr[c]) : -INFINITY;
        float mx = sv[0];
#pragma unroll
        for (int c = 1; c < 32; ++c) mx = fmaxf(mx, sv[c]);
        red[(gi & 1) * 128 + L] = mx;
        named_bar_sync(1, 128);
        mx = fmaxf(mx, red[(gi & 1) * 128 + (L ^ 64)]);
        if (i == 0) {
          m_ref = mx;
        } else {
          const bool need = (mx - m_ref) * c2 > RESCALE_LOG2;
          if (__any_sync(0xffffffffu, need)) {
            const float m_new = need ? mx : m_ref;
            const float alpha = exp2f((m_ref - m_new) * c2);
            const int gp = gi - 1;  // wait until PV of the previous tile has landed in O
            mbar_wait_warp(bar(BAR_O_FULL + gp % NB), (gp / NB) & 1, abort_flag);
            tc_fence_after();
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const uint32_t a = lane_addr + 128 * (q4 >> 2) + 32 * (q4 & 3);
              uint32_t o[32];
              tmem_ld32(a, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
              tmem_st32(a, o);
            }
            tmem_wait_st();
            lsum *= alpha;
            m_ref = m_new;
          }
        }
        const float mo = m_ref * c2;
        uint32_t pk[16];
        float ps = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float p0 = exp2f(fmaf(sv[2 * c], c2, -mo));
          const float p1 = exp2f(fmaf(sv[2 * c + 1], c2, -mo));
          ps += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        lsum += ps;
        // the P buffer is free once the PV of two tiles ago has completed
        if (gi >= NB) mbar_wait_warp(bar(BAR_O_FULL + b), ((gi - NB) / NB) & 1, abort_flag);
        uint8_t *pb = smem + OFF_P + b * P_BYTES + row * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int chunk = 4 * half + q4;
          *reinterpret_cast<uint4 *>(pb + ((chunk ^ (row & 7)) << 4)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        // last, partial tile: zero the value rows past the end (they may hold
        // anything, and 0 * NaN would poison O)
        const int valid = pc.vis - ti * TILE;
        if (valid < TILE) {
          uint8_t *vb = smem + OFF_V + (gi % NS) * V_BYTES;
          const int nrow = TILE - valid;
          for (int e = L; e < nrow * 4 * 8; e += 128) {
            const int r = valid + e / 32, c = (e >> 3) & 3, w16 = e & 7;
            *reinterpret_cast<uint4 *>(vb + c * CHUNK_V + r * 128 + w16 * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) arrive_leader(bar(BAR_P_FULL + b), rank);
      }
      // ---------------------------------------------------------- epilogue
      const int gl = gi - 1;
      mbar_wait_warp(bar(BAR_O_FULL + gl % NB), (gl / NB) & 1, abort_flag);
      tc_fence_after();
      redl[L] = lsum;
      named_bar_sync(1, 128);
      const float ltot = lsum + redl[L ^ 64];
      const float inv = 1.f / ltot;
      const float lse_v = m_ref * p.scale + logf(ltot);
      const int head = HPC * rank + row;
#pragma unroll 1
      for (int q4 = 0; q4 < 8; ++q4) {
        const int j = q4 >> 2, part = q4 & 3;
        uint32_t o[32];
        tmem_ld32(lane_addr + 128 * j + 32 * part, o);
        tmem_wait_ld();
        const int col = 256 * j + 128 * half + 32 * part;
        if (pc.single) {
          uint4 *dst = reinterpret_cast<uint4 *>(p.o_lat + (static_cast<int64_t>(pc.bj) * HEADS + head) * DC + col);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16x2(__uint_as_float(o[8 * v + 2 * e]) * inv, __uint_as_float(o[8 * v + 2 * e + 1]) * inv);
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4 *dst = reinterpret_cast<float4 *>(p.part_o + (static_cast<int64_t>(pc.slot) * HEADS + head) * DC + col);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                 __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
        }
      }
      if (half == 0) {
        if (pc.single) {
          if (p.lse != nullptr) p.lse[static_cast<int64_t>(pc.bj) * HEADS + head] = lse_v;
        } else {
          p.part_lse[static_cast<int64_t>(pc.slot) * HEADS + head] = lse_v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(bar(BAR_O_FREE), rank);
    }
  }

  // ---- teardown: both CTAs done with each other's barriers, then free TMEM
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_cluster(mapa_shared(bar(BAR_EXIT), rank ^ 1));
    mbar_wait(bar(BAR_EXIT), 0, nullptr);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<2>(tmem, 512);
}

// Merge the split partials of every token row that was cut by cluster range
// boundaries: lse = log sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s.
// grid = BJ * 16 blocks of 8 warps; one warp per head.
__global__ void __launch_bounds__(256) k_combine(Params p) {
  const int bj = blockIdx.x >> 4, head = (blockIdx.x & 15) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int a = p.plan[2 + bj], e = p.plan[3 + bj], Qt = p.plan[1];
  if (e <= a) return;
  const int k0 = a / Qt, k1 = (e - 1) / Qt;
  if (k0 == k1) return;
  float M = -INFINITY;
  for (int k = k0; k <= k1; ++k) M = fmaxf(M, p.part_lse[static_cast<int64_t>(bj + k) * HEADS + head]);
  float Z = 0.f;
  float acc[16];
#pragma unroll
  for (int v = 0; v < 16; ++v) acc[v] = 0.f;
  for (int k = k0; k <= k1; ++k) {
    const float w = __expf(p.part_lse[static_cast<int64_t>(bj + k) * HEADS + head] - M);
    Z += w;
    const float4 *src = reinterpret_cast<const float4 *>(p.part_o + (static_cast<int64_t>(bj + k) * HEADS + head) * DC);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 x = src[lane + 32 * v];
      acc[4 * v] += w * x.x;
      acc[4 * v + 1] += w * x.y;
      acc[4 * v + 2] += w * x.z;
      acc[4 * v + 3] += w * x.w;
    }
  }
  const float inv = 1.f / Z;
  __nv_bfloat16 *dst = p.o_lat + (static_cast<int64_t>(bj) * HEADS + head) * DC;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int col = 4 * (lane + 32 * v);
    uint2 w;
    w.x = pack_bf16x2(acc[4 * v] * inv, acc[4 * v + 1] * inv);
    w.y = pack_bf16x2(acc[4 * v + 2] * inv, acc[4 * v + 3] * inv);
    *reinterpret_cast<uint2 *>(dst + col) = w;
  }
  if (lane == 0 && p.lse != nullptr) p.lse[static_cast<int64_t>(bj) * HEADS + head] = M + logf(Z);
}

}  // namespace dec

// Workspace: plan (W, Qt, BJ + 1 offsets) then split partials for at most
// BJ + clusters slots.
inline size_t decode_tc_ws(int B, int n_q, int sms) {
  const size_t BJ = static_cast<size_t>(B) * n_q;
  const size_t clusters = static_cast<size_t>(sms / 2);
  const size_t plan = ((BJ + 3) * sizeof(int32_t) + 255) & ~size_t(255);
  const size_t slots = BJ + clusters;
  return plan + slots * dec::HEADS * dec::DC * sizeof(float) + slots * dec::HEADS * sizeof(float);
}

}  // namespace mla
