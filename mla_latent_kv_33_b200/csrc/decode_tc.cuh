// Absorbed-form MLA decode on sm_100a tensor cores (MLA walk-through,
// h.sjds.net, section 1 step 4 and section 3 order B).
//
// For every token row t (sequence b, new token j) and head h:
//   s_i = scale * (q_lat,h . c_KV_i + q_R,h . k_R_i) over the visible cached
//   positions i, p = softmax(s), o_lat = sum_i p_i c_KV_i, lse = log sum exp s.
//
// Design (B200, one GPU):
//  * All 128 heads of a token row share every cached row, so per 256-token
//    tile S = Q K^T is a dense 128 x 256 x 576 contraction and O += P V a
//    dense 128 x 512 x 256 one. Both run as tcgen05.mma.cta_group::2 on a
//    pair of SMs (a 2-CTA cluster) with M = 128, N = 256: CTA r holds heads
//    64r..64r+63 of Q, supplies tokens 128r..128r+127 of the tile to QK^T
//    (B split by N = tokens) and latent columns [256j + 128r, +128) of every
//    token to PV (B split by N = latent). The tensor pipe retires one MMA
//    instruction per ~35 ns whatever its shape, and only M128 x N256 pair
//    instructions carry a full 35 ns of work, so both products use that shape
//    (68 instructions per tile).
//  * The 128 x 512 fp32 accumulator O is one whole SM of tensor memory, so it
//    is split over the pair: 256 columns per CTA, plus two 128-column score
//    buffers = all 512 columns.
//  * Shared memory per CTA: Q 72 KB resident per piece and a ring of four
//    32 KB slots and one 16 KB slot consumed strictly in MMA order:
//    the score operands of tile i + 1 (column chunks {0,1} {2,3} {4,5} {6,7}
//    in big slots, chunk 8 in the small one; each chunk holds this CTA's 128
//    tokens as 128 rows so that one N = 256 MMA spans them), then the value
//    operands of tile i (one big slot per pair of blocks {v, v + 2} and latent
//    half: 128 of this CTA's latent columns of both). Every ring item costs a
//    commit (~50-70 ns of tensor-pipe time), so items are as large as the
//    shared memory allows; the small slot is released by the commit that
//    completes S rather than a commit of its own. Latent columns
//    are read twice (once per operand), the second time mostly from L2. (An
//    explicit whole-block L2 prefetch ahead of the score loads measured
//    slower: it added DRAM reads without removing the score loads' misses.)
//  * Loads: the TMA operations one warp issues complete one after another
//    (~50 GB/s per warp), those of different warps side by side, so four
//    producer warps share the ring, one per big slot: every slot's uses are
//    issued in order by one warp, and no slot waits behind another slot's
//    loads. Q arrives as three 24 KB boxes from three of the producers.
//  * P lives in tensor memory, written by the softmax over the scores it was
//    made from, as the A operand of PV. A pair MMA with M = 128 reads a row's
//    16-wide K group from both lane m and lane m + 64 (one copy per half of
//    N), so each K group pairs 8 tokens of the first CTA's half of the tile
//    (held by lane m) with 8 of the second's (lane m + 64); the two lanes
//    trade their halves through shared memory. The value item pairs blocks v
//    and v + 2 at a fixed 16 KB distance, so that one B descriptor spans both.
//  * Warp roles: warps 0-2 and 8 load, warp 3 of CTA 0 issues the MMAs of the
//    pair, warps 4-7 of both CTAs run the online softmax (fp32, exp2, O rescaled
//    only when the running max grows by more than 2^8) and the epilogue.
//  * Work: the visible 256-token tiles of all token rows are concatenated and
//    cut into equal contiguous ranges, one per cluster (persistent grid). A
//    row whose tiles fall in one range is finished in place (bf16 o_lat,
//    lse); a row cut by range boundaries leaves normalised fp32 partials
//    that k_combine merges with a log-sum-exp. (Merging them in the epilogue
//    of the CTA that finishes a row's last piece measured slower: the merge
//    then runs on one SM's bandwidth, on that cluster's critical path.)
//    With a forced split count S (Params::splits > 0) every row is instead
//    cut into min(S, its tiles) pieces of near-equal tile counts, and each
//    cluster takes the pieces that start in its equal share of the tile line.
//    With n_q > 1 new tokens per sequence (the k_decode<true> instance) the
//    rows are ordered by query position and, in the automatic plan, each
//    position's rows are cut by their own group of clusters into ranges of
//    one length, so the n_q rows of a sequence stream the same cache tiles
//    at about the same time and all but one read them from L2.
//  * Rows past a sequence's end: 64-row blocks wholly past it are loaded at
//    an out-of-range coordinate (TMA zero fill); the one partially valid block
//    has its value rows past the end zeroed in shared memory before its PV
//    (scores there are masked to -inf, but 0 * NaN would still poison O).
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace dec {

constexpr int D = 576, DC = 512, DR = 64, HEADS = 128, HPC = 64;
constexpr int TILE = 256, OWN = 128, BLK = 64;  // tokens per pair tile / per CTA / per block
// 9 warps: producers 0-2 and 8 (producer index 3), the MMA warp 3, and the
// softmax warps 4-7 (warp w reaches tensor-memory lanes 32 (w % 4) .. + 31)
constexpr int NUM_PRODUCERS = 4, WARP_MMA = 3, WARP_SOFTMAX = 4, WARP_PROD3 = 8;
constexpr int NUM_THREADS = 32 * 9;
constexpr int NBIG = 4;              // 32 KB ring slots; big slot s belongs to producer s
// the small slot's producer; Q's three 24 KB boxes come from producers 0-2
// (each waits Q's empty barrier for every piece, so each wait is exact)
constexpr int SMALL_OWNER = 1, Q_LOADERS = 3;
constexpr int CHUNK_Q = HPC * 128;   // 64 heads x 64 columns
constexpr int ATOM = BLK * 128;      // 64 rows x 64 columns (one 128-byte-swizzle atom column)
constexpr int CHUNK_K = 2 * ATOM;    // one column chunk of the CTA's 128 tokens
constexpr int BIG = 4 * ATOM, SMALL = 2 * ATOM, HALF = BIG / 2;
constexpr int K_ITEMS = 5, V_ITEMS = 4;  // per tile: chunks {0,1} {2,3} {4,5} {6,7} {8}; (block pair, latent half)
constexpr int BIG_PER_TILE = 8;          // big-slot uses per tile (4 score + 4 value items)
constexpr int Q_BYTES = 9 * CHUNK_Q;
constexpr int XBUF_BYTES = 128 * 16 * 4;  // softmax partner exchange: 16 packed P words per thread
constexpr int OFF_Q = 0;
constexpr int OFF_BIG = OFF_Q + Q_BYTES;
constexpr int OFF_SMALL = OFF_BIG + NBIG * BIG;
constexpr int OFF_XBUF = OFF_SMALL + SMALL;
constexpr int OFF_MISC = OFF_XBUF + XBUF_BYTES;
constexpr int BAR_Q_FULL = 0, BAR_Q_EMPTY = 1, BAR_BIG_FULL = 2, BAR_BIG_EMPTY = BAR_BIG_FULL + NBIG,
              BAR_SMALL_FULL = BAR_BIG_EMPTY + NBIG,
              BAR_V_LANDED = BAR_SMALL_FULL + 1, BAR_ZERO_DONE = BAR_V_LANDED + 1, BAR_S_FULL = BAR_ZERO_DONE + 1,
              BAR_P_FULL = BAR_S_FULL + 2, BAR_O_FULL = BAR_P_FULL + 1,
              BAR_O_FREE = BAR_O_FULL + 1, BAR_EXIT = BAR_O_FREE + 1, NUM_BARS = BAR_EXIT + 1;
constexpr int MISC_RED = 256;               // float red[2][128]
constexpr int MISC_REDL = MISC_RED + 1024;  // float redl[128]
constexpr int MISC_INTS = MISC_REDL + 512;
constexpr int MISC_BYTES = MISC_INTS + 64;
constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
static_assert(NUM_BARS * 8 <= MISC_RED, "barriers overlap the exchange arrays");
static_assert(SMEM_BYTES <= 232448, "decode shared memory budget");
static_assert(OFF_BIG % 1024 == 0 && OFF_SMALL % 1024 == 0, "128-byte swizzle alignment");
constexpr int MAX_UNITS = (NBIG * BIG + SMALL) / 8 - 1;  // plan scratch (two ints per row) aliases the ring
constexpr int S_COL = 256;  // TMEM: O at [0,256); scores, then P over them, at [256 + 128 b, +128)
constexpr uint32_t IDESC_S = idesc_bf16(128, 256, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);
constexpr float RESCALE_LOG2 = 8.f;

// Ring items in MMA consumption order, per piece of n tiles: the score items
// of tile 0; for every later tile its score items followed by the value items
// of the tile before it; the value items of the last tile. The big-slot use
// of the value item (tile i, block pair vp = {vp, vp + 2}, latent half j):
__host__ __device__ constexpr int value_item(int i, int n, int vp, int j) {
  return 4 * (i + 2 < n ? i + 2 : n) + 4 * i + 2 * vp + j;
}

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
  float *part_o;    // [slots][128][512]
  float *part_lse;  // [slots][128]
  // [0] = W (visible tiles), [1] = Qt (tiles per cluster, automatic plan), [2] = splits,
  // [3] = cluster groups G, [4] = clusters per group, [5 ..] tile offsets of the units
  // [BJ + 1], then (splits > 0) piece offsets [BJ + 1]
  int32_t *plan;
  int32_t splits;   // 0: automatic plan; S > 0: every row in min(S, tiles) pieces
};

// Offsets of the plan arrays in Params::plan.
__host__ __device__ constexpr int plan_tiles(int) { return 5; }
__host__ __device__ constexpr int plan_pieces(int BJ) { return 6 + BJ; }

// The tile line's units are the token rows in query-position-major order:
// unit u = j B + b is row b n_q + j (new token j of sequence b). The kernel
// is compiled twice: kGrouped = false serves n_q = 1, where unit and row
// coincide, with none of the index arithmetic or cluster groups below.
template <bool kGrouped>
__device__ __forceinline__ int row_of_unit(const Params &p, int u) {
  return !kGrouped ? u : (u % p.B) * p.n_q + u / p.B;
}
__device__ __forceinline__ int unit_of_row(const Params &p, int bj) {
  return p.n_q == 1 ? bj : (bj % p.n_q) * p.B + bj / p.n_q;
}

// Tiles visible to unit u; -1 if its sequence length is invalid.
template <bool kGrouped>
__device__ __forceinline__ int unit_tiles(const Params &p, int u, int *vis_out) {
  const int b = !kGrouped ? u : u % p.B, j = !kGrouped ? 0 : u / p.B;
  const int L = p.seq_lens[b];
  if (L < p.n_q || static_cast<int64_t>(L) > p.capacity) {
    *vis_out = 0;
    return -1;
  }
  const int vis = L - p.n_q + 1 + j;
  *vis_out = vis;
  return (vis + TILE - 1) / TILE;
}

// Cache rows of the four 64-token blocks of a 256-token tile (positions
// t0 + 64 v), or cache_rows (an out-of-range TMA coordinate: zero fill) for
// blocks past the visible length or with an invalid block-table entry. Two
// steps: tile_blocks() issues the four block-table loads, rows_of_blocks()
// checks and converts their values. The producers issue the loads of tile
// i + 2 while they convert those of tile i + 1, loaded a whole tile earlier,
// so that the check (a branch on the loaded value) never waits for memory.
__device__ __forceinline__ void tile_blocks(const Params &p, int b, int64_t t0, int vis, int32_t blk[4]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int64_t pos = t0 + BLK * v;
    blk[v] = p.paged && pos < vis ? p.block_table[static_cast<int64_t>(b) * p.max_blocks_per_seq + pos / p.block_size] : 0;
  }
}
__device__ __forceinline__ void rows_of_blocks(const Params &p, int b, int64_t t0, int vis, const int32_t blk[4],
                                               int32_t r4[4]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int64_t pos = t0 + BLK * v;
    if (pos >= vis) {
      r4[v] = static_cast<int32_t>(p.cache_rows);
    } else if (!p.paged) {
      r4[v] = static_cast<int32_t>(static_cast<int64_t>(b) * p.max_len + pos);
    } else if (blk[v] < 0 || blk[v] >= p.num_blocks_i32) {
      dev_error(MLA_DEVERR_DATA);
      r4[v] = static_cast<int32_t>(p.cache_rows);
    } else {
      r4[v] = static_cast<int32_t>(static_cast<int64_t>(blk[v]) * p.block_size + pos % p.block_size);
    }
  }
}

struct Piece {
  int bj, t_begin, t_end, vis, nt;
  bool single;  // the row's only piece: o_lat and lse are written in place
  int slot;     // split partial slot of this piece (when not single)
};

__device__ __forceinline__ int split_pieces(int S, int nt) { return nt < S ? nt : S; }

// End (row-relative tile) of the forced-split piece holding tile r of a row
// with nt tiles cut into sp pieces (piece q covers [q nt / sp, (q + 1) nt / sp)),
// and that piece's index.
__device__ __forceinline__ int split_piece_of(int r, int nt, int sp, int *end) {
  const int q = static_cast<int>((static_cast<int64_t>(r + 1) * sp - 1) / nt);
  *end = static_cast<int>(static_cast<int64_t>(q + 1) * nt / sp);
  return q;
}

// Iterates the pieces of this cluster's tile range in order. Automatic plan:
// pieces are cut by row ends and cluster boundaries, and the split slot of a
// unit's piece in cluster k is u + k (a cluster holds at most one piece of a
// row that continues into another cluster); base is the first tile of the
// cluster's group. Forced splits: pieces are also cut at the row's piece
// boundaries, and the slot is the piece's global index.
template <bool kGrouped>
struct PieceIter {
  int g, gend, u, off, poff, Qt, k, S, base;
  __device__ bool next(const Params &p, Piece &pc) {
    while (g < gend) {
      int vis;
      int nt = unit_tiles<kGrouped>(p, u, &vis);
      if (nt < 0) nt = 0;
      if (nt == 0 || off + nt <= g) {
        off += nt;
        poff += S ? split_pieces(S, nt) : 0;
        ++u;
        continue;
      }
      pc.bj = row_of_unit<kGrouped>(p, u);
      pc.vis = vis;
      pc.nt = nt;
      pc.t_begin = g - off;
      if (S) {
        const int sp = split_pieces(S, nt);
        int pend;
        const int q = split_piece_of(g - off, nt, sp, &pend);
        const int e = min(gend, off + pend);
        pc.t_end = e - off;
        pc.single = sp == 1;
        pc.slot = poff + q;
        g = e;
        if (e == off + nt) {
          off += nt;
          poff += sp;
          ++u;
        }
        return true;
      }
      const int e = min(gend, off + nt);
      pc.t_end = e - off;
      pc.single = kGrouped ? (off - base) / Qt == (off + nt - 1 - base) / Qt : off / Qt == (off + nt - 1) / Qt;
      pc.slot = u + k;
      g = e;
      off += nt;
      ++u;
      return true;
    }
    return false;
  }
};

// In-place exclusive prefix sum of a[0 .. n) by the whole block; returns the
// total to every thread. wtot: NUM_THREADS / 32 ints of shared memory.
template <int NT>
__device__ int block_exclusive_scan(int *a, int n, int *wtot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (n + NT - 1) / NT;
  const int lo = min(n, static_cast<int>(threadIdx.x) * per), hi = min(n, lo + per);
  int sum = 0;
  for (int u = lo; u < hi; ++u) sum += a[u];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  int base = 0, total = 0;
  for (int w = 0; w < NT / 32; ++w) {
    if (w < warp) base += wtot[w];
    total += wtot[w];
  }
  int run = base + incl - sum;
  for (int u = lo; u < hi; ++u) {
    const int v = a[u];
    a[u] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

// Row holding tile G of the tile line (prefix[] = exclusive tile offsets of
// the BJ rows, G < W): the last row whose offset is <= G, which is never empty.
__device__ __forceinline__ int row_of_tile(const int *prefix, int BJ, int G) {
  int lo = 0, hi = BJ - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= G) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// First forced-split piece boundary at or after tile G of the tile line.
__device__ __forceinline__ int snap_to_piece(const int *prefix, int BJ, int W, int S, int G) {
  if (G >= W) return W;
  const int u = row_of_tile(prefix, BJ, G);
  const int nt = (u + 1 < BJ ? prefix[u + 1] : W) - prefix[u];
  const int sp = split_pieces(S, nt), r = G - prefix[u];
  int pend;
  const int q = split_piece_of(r, nt, sp, &pend);
  const int pbeg = static_cast<int>(static_cast<int64_t>(q) * nt / sp);
  return pbeg == r ? G : prefix[u] + pend;
}

// The value chunk of tile ti that needs zeroed rows (holds the last visible
// token but not 64 visible tokens), or -1.
__device__ __forceinline__ int partial_chunk(int vis, int ti) {
  const int v = vis - ti * TILE;
  if (v >= TILE || (v % BLK) == 0) return -1;
  return v / BLK;
}

__device__ __forceinline__ void arrive_leader(uint32_t bar_local, uint32_t rank) {
  if (rank == 0)
    mbar_arrive(bar_local);
  else
    mbar_arrive_cluster(mapa_shared(bar_local, 0));
}

template <bool kGrouped>
__global__ void __launch_bounds__(NUM_THREADS, 1) __cluster_dims__(2, 1, 1)
    k_decode(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v0,
             const __grid_constant__ CUtensorMap tm_v1, const Params p) {
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
  int *plan_s = ints + 2;  // g0, g1, Qt, first unit, its tile offset, its piece offset, group base

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q_FULL), 1);
    mbar_init(bar(BAR_Q_EMPTY), 1);
    for (int s = 0; s < NBIG; ++s) {
      mbar_init(bar(BAR_BIG_FULL + s), 1);
      mbar_init(bar(BAR_BIG_EMPTY + s), 1);
    }
    mbar_init(bar(BAR_SMALL_FULL), 1);
    mbar_init(bar(BAR_V_LANDED), 1);
    mbar_init(bar(BAR_ZERO_DONE), 8);
    for (int b = 0; b < 2; ++b) mbar_init(bar(BAR_S_FULL + b), 1);
    mbar_init(bar(BAR_P_FULL), 8);
    mbar_init(bar(BAR_O_FULL), 1);
    mbar_init(bar(BAR_O_FREE), 8);
    mbar_init(bar(BAR_EXIT), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  const CUtensorMap *tm_v = rank == 0 ? &tm_v0 : &tm_v1;  // value slabs: this CTA's latent columns
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(tm_v);
  }
  if (warp == WARP_MMA) tmem_alloc<2>(smem_u32(tmem_slot), 512);
  if (threadIdx.x == 0) griddep_launch_dependents();
  // everything below reads sequence lengths, the cache or q, or writes the
  // workspace: only once the previous kernel on the stream has finished
  griddep_wait();

  // ---- plan: tiles (and forced pieces) per unit, prefix sums, this cluster's range ----
  const int BJ = p.B * p.n_q;
  const int S = p.splits;
  int *tiles = reinterpret_cast<int *>(smem + OFF_BIG);  // [BJ], then (S > 0) pieces [BJ]
  int *pieces = tiles + BJ;
  for (int u = threadIdx.x; u < BJ; u += NUM_THREADS) {
    int vis;
    int nt = unit_tiles<kGrouped>(p, u, &vis);
    if (nt < 0) {
      if (blockIdx.x == 0 && u < p.B) dev_error(MLA_DEVERR_DATA);  // once per sequence
      nt = 0;
    }
    tiles[u] = nt;
    if (S) pieces[u] = split_pieces(S, nt);
  }
  __syncthreads();
  {
    __shared__ int warp_tot[NUM_THREADS / 32];
    const int W = block_exclusive_scan<NUM_THREADS>(tiles, BJ, warp_tot);
    const int P = S ? block_exclusive_scan<NUM_THREADS>(pieces, BJ, warp_tot) : 0;
    // Automatic plan with n_q > 1 (and at least n_q clusters): one group of
    // clusters per query position j cuts the line of the rows of position j
    // into equal ranges, the same length Qt in every group, so that the n_q
    // rows of a sequence stream the same cache tiles at about the same time
    // and all but one of their reads hit L2.
    const int G = kGrouped && S == 0 && nclusters >= p.n_q ? p.n_q : 1;
    const int ncg = nclusters / G;
    if (threadIdx.x == 0) {
      int g0, g1, Qt = 0, base = 0;
      if (S == 0) {
        for (int q = 0; q < G; ++q) {
          const int lo = G > 1 ? tiles[q * p.B] : 0, hi = q + 1 < G ? tiles[(q + 1) * p.B] : W;
          Qt = max(Qt, (hi - lo + ncg - 1) / ncg);
        }
        Qt = max(1, Qt);
        const int grp = cluster / ncg, kl = cluster % ncg;
        if (grp < G) {
          base = G > 1 ? tiles[grp * p.B] : 0;
          const int end = grp + 1 < G ? tiles[(grp + 1) * p.B] : W;
          g0 = min(end, base + kl * Qt);
          g1 = min(end, base + (kl + 1) * Qt);
        } else {
          g0 = g1 = W;  // a cluster left over when n_q does not divide the clusters
        }
      } else {
        const auto share = [&](int c) {
          return static_cast<int>((static_cast<int64_t>(c) * W + nclusters - 1) / nclusters);
        };
        g0 = snap_to_piece(tiles, BJ, W, S, share(cluster));
        g1 = snap_to_piece(tiles, BJ, W, S, share(cluster + 1));
      }
      const int u0 = g0 < W ? row_of_tile(tiles, BJ, g0) : BJ;
      plan_s[0] = g0;
      plan_s[1] = g1;
      plan_s[2] = Qt;
      plan_s[3] = u0;
      plan_s[4] = u0 < BJ ? tiles[u0] : W;
      plan_s[5] = S && u0 < BJ ? pieces[u0] : 0;
      plan_s[6] = base;
    }
    if (blockIdx.x == 0) {  // the layout k_combine reads
      for (int u = threadIdx.x; u < BJ; u += NUM_THREADS) {
        p.plan[plan_tiles(BJ) + u] = tiles[u];
        if (S) p.plan[plan_pieces(BJ) + u] = pieces[u];
      }
      if (threadIdx.x == 0) {
        p.plan[0] = W;
        p.plan[1] = S == 0 ? max(1, plan_s[2]) : 0;
        p.plan[2] = S;
        p.plan[3] = G;
        p.plan[4] = ncg;
        p.plan[plan_tiles(BJ) + BJ] = W;
        if (S) p.plan[plan_pieces(BJ) + BJ] = P;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // peer barriers initialised, TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  PieceIter<kGrouped> it0;
  it0.g = plan_s[0];
  it0.gend = plan_s[1];
  it0.Qt = max(1, plan_s[2]);
  it0.u = plan_s[3];
  it0.off = plan_s[4];
  it0.poff = plan_s[5];
  it0.k = cluster;
  it0.S = S;
  it0.base = plan_s[6];

  if (warp < WARP_MMA || warp == WARP_PROD3) {
    // --------------------------------------------------------- ring producers
    // Every producer warp walks the same item sequence and issues the items
    // of the slots it owns, so that each slot's uses are issued in order by
    // one warp (a parity wait on the slot's empty barrier is exact only when
    // the waiter is at most one phase ahead). Lane 0 waits for the slot and
    // arms its full barrier, then lane l issues box l of the item.
    const int w = warp < WARP_MMA ? warp : 3;  // producer index
    const uint32_t q_full = rank == 0 ? bar(BAR_Q_FULL) : mapa_shared(bar(BAR_Q_FULL), 0);
    PieceIter<kGrouped> it = it0;
    Piece pc;
    int nbig = 0, nsmall = 0, npc = 0;
    bool ok = true;
    auto full_of = [&](int bi) { return rank == 0 ? bar(bi) : mapa_shared(bar(bi), 0); };
    // Next item: 0 if another warp issues it; else waits for its slot, arms
    // the barrier (*fb) and returns the slot's shared-memory offset, or -1 on
    // a failed wait (all warp-uniform).
    auto claim = [&](bool big, uint32_t bytes, int *fb) -> int {
      int slot, use;
      if (big) {
        slot = nbig % NBIG;
        use = nbig / NBIG;
        ++nbig;
      } else {
        slot = 0;
        use = nsmall++;
      }
      if ((big ? slot % NUM_PRODUCERS : SMALL_OWNER) != w) return 0;
      // the small slot's use u is tile u's score item; it is free once S(u)
      // has completed (S_FULL of buffer u & 1, phase u >> 1)
      const int eb = big ? BAR_BIG_EMPTY + slot : BAR_S_FULL + ((use - 1) & 1);
      const uint32_t epar = big ? (use - 1) & 1 : ((use - 1) >> 1) & 1;
      *fb = big ? BAR_BIG_FULL + slot : BAR_SMALL_FULL;
      bool good = true;
      if (lane == 0) {
        if (use > 0) good = mbar_wait(bar(eb), epar, abort_flag);
        if (good && rank == 0) mbar_arrive_expect_tx(bar(*fb), 2 * bytes);
      }
      return __shfl_sync(0xffffffffu, good, 0) ? (big ? OFF_BIG + slot * BIG : OFF_SMALL) : -1;
    };
    auto load_k = [&](const int32_t *own) -> bool {  // score items of one tile (own blocks)
      for (int q = 0; q < K_ITEMS; ++q) {
        const bool big = q < K_ITEMS - 1;
        int fb = 0;
        const int off = claim(big, big ? BIG : SMALL, &fb);
        if (off < 0) return false;
        if (off == 0) continue;
        if (lane < (big ? 4 : 2)) {  // lane l: column chunk 2q + l / 2 of own block l % 2
          const int c = 2 * q + (lane >> 1), kb = lane & 1;
          tma_load_2d_pair(sbase + off + (lane >> 1) * CHUNK_K + kb * ATOM, &tm_k, 64 * c, own[kb], full_of(fb));
        }
        __syncwarp();
      }
      return true;
    };
    // value items of one tile: (block pair {vp, vp + 2}, latent half j); lane l
    // loads block vp + 2 l (16 KB: two latent chunks of 64 rows)
    auto load_v = [&](const int32_t *rows) -> bool {
      for (int vp = 0; vp < 2; ++vp)
        for (int j = 0; j < 2; ++j) {
          int fb = 0;
          const int off = claim(true, BIG, &fb);
          if (off < 0) return false;
          if (off == 0) continue;
          const int32_t row = lane ? (vp ? rows[3] : rows[2]) : (vp ? rows[1] : rows[0]);  // block vp + 2 lane
          if (lane < 2) tma_load_4d_pair(sbase + off + lane * HALF, tm_v, 0, row, 0, j, full_of(fb));
          __syncwarp();
        }
      return true;
    };
    while (ok && it.next(p, pc)) {
      const int b = pc.bj / p.n_q;
      auto blocks_of = [&](int ti, int32_t *blk) { tile_blocks(p, b, static_cast<int64_t>(ti) * TILE, pc.vis, blk); };
      auto rows_of = [&](int ti, const int32_t *blk, int32_t *r4) {
        rows_of_blocks(p, b, static_cast<int64_t>(ti) * TILE, pc.vis, blk, r4);
      };
      int32_t cur[4], prev[4], nxt[4] = {0, 0, 0, 0}, raw0[4], raw[4] = {0, 0, 0, 0};
      blocks_of(pc.t_begin, raw0);
      if (pc.t_begin + 1 < pc.t_end) blocks_of(pc.t_begin + 1, raw);
      rows_of(pc.t_begin, raw0, cur);
      if (w < Q_LOADERS) {  // producer w loads Q's column chunks 3 w .. 3 w + 2
        bool good = true;
        if (lane == 0) {
          if (npc > 0) good = mbar_wait(bar(BAR_Q_EMPTY), (npc - 1) & 1, abort_flag);
          if (good) {
            if (rank == 0 && w == 0) mbar_arrive_expect_tx(bar(BAR_Q_FULL), 2 * Q_BYTES);
            tma_load_3d_pair(sbase + OFF_Q + 3 * w * CHUNK_Q, &tm_q, 0, pc.bj * HEADS + HPC * rank, 3 * w, q_full);
          }
        }
        if (!__shfl_sync(0xffffffffu, good, 0)) {
          ok = false;
          break;
        }
      }
      for (int ti = pc.t_begin; ti < pc.t_end && ok; ++ti) {
        if (ti + 1 < pc.t_end) {
          rows_of(ti + 1, raw, nxt);
          if (ti + 2 < pc.t_end) blocks_of(ti + 2, raw);
        }
        const int32_t own[2] = {rank ? cur[2] : cur[0], rank ? cur[3] : cur[1]};
        if (!load_k(own)) { ok = false; break; }
        if (ti > pc.t_begin && !load_v(prev)) { ok = false; break; }
        for (int v = 0; v < 4; ++v) {
          prev[v] = cur[v];
          cur[v] = nxt[v];
        }
      }
      if (!ok || !load_v(prev)) { ok = false; break; }
      ++npc;
    }
    // drain: every commit aimed at the empty barriers of this warp's slots
    // (and of Q) has landed; each warp waits only on what it owns, see above
    if (lane == 0) {
      for (int sl = w; ok && sl < NBIG; sl += NUM_PRODUCERS) {
        const int uses = nbig > sl ? (nbig - sl + NBIG - 1) / NBIG : 0;
        if (uses > 0) mbar_wait(bar(BAR_BIG_EMPTY + sl), (uses - 1) & 1, abort_flag);
      }
      if (ok && w == SMALL_OWNER && nsmall > 0)
        mbar_wait(bar(BAR_S_FULL + ((nsmall - 1) & 1)), ((nsmall - 1) >> 1) & 1, abort_flag);
      if (ok && w < Q_LOADERS && npc > 0) mbar_wait(bar(BAR_Q_EMPTY), (npc - 1) & 1, abort_flag);
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    if (rank == 0 && lane == 0) {
      PieceIter<kGrouped> it = it0;
      Piece pc{};
      int gi = 0, nbig = 0, nsmall = 0, gz = 0, npc = 0, empty_bar = 0;
      bool ok = true;
      auto take = [&](bool big) -> uint32_t {  // next ring item in consumption order, once it has landed
        int slot, use;
        if (big) {
          slot = nbig % NBIG;
          use = nbig / NBIG;
          ++nbig;
        } else {
          slot = 0;
          use = nsmall++;
        }
        empty_bar = BAR_BIG_EMPTY + slot;  // (small items are released by S_FULL)
        if (!mbar_wait(bar(big ? BAR_BIG_FULL + slot : BAR_SMALL_FULL), use & 1, abort_flag)) return 0;
        tc_fence_after();
        return sbase + (big ? OFF_BIG + slot * BIG : OFF_SMALL);
      };
      auto release = [&]() { tc_commit_pair(bar(empty_bar), 0x3); };
      // PV of global tile gt (tile ti of the current piece): A = P in tensor
      // memory; K step m of value item (vp, j) takes 8 tokens of block vp and 8
      // of block vp + 2 (one B descriptor over both halves of the item)
      auto issue_pv = [&](int gt, int ti, bool first) -> bool {
        const int zc = partial_chunk(pc.vis, ti);
        const uint32_t p_col = tmem + S_COL + 128 * (gt & 1);
        for (int vp = 0; vp < 2; ++vp)
          for (int j = 0; j < 2; ++j) {
            const uint32_t vb = take(true);
            if (vb == 0) return false;
            if (vp == 0 && j == 0) {
              if (!mbar_wait(bar(BAR_P_FULL), gt & 1, abort_flag)) return false;
              if (first && npc > 0 && !mbar_wait(bar(BAR_O_FREE), (npc - 1) & 1, abort_flag)) return false;
              tc_fence_after();
            }
            if (zc >= 0 && vp == (zc & 1)) {  // both CTAs zero the rows past the end first
              mbar_arrive(bar(BAR_V_LANDED));
              mbar_arrive_cluster(mapa_shared(bar(BAR_V_LANDED), 1));
              if (!mbar_wait(bar(BAR_ZERO_DONE), gz & 1, abort_flag)) return false;
              ++gz;
              tc_fence_after();
            }
            const uint64_t vd = sdesc_sw128(vb, ATOM, HALF);  // K step m: + 1024 bytes
#pragma unroll
            for (int m = 0; m < 8; ++m)
              tc_mma_ts<2>(tmem + 128 * j, p_col + 8 * (8 * vp + m), sdesc_advance(vd, m * 1024), IDESC_PV,
                           (first && vp == 0 && m == 0) ? 0u : 1u);
            release();
          }
        tc_commit_pair(bar(BAR_O_FULL), 0x3);
        return true;
      };
      while (ok && it.next(p, pc)) {
        if (!mbar_wait(bar(BAR_Q_FULL), npc & 1, abort_flag)) break;
        const int n = pc.t_end - pc.t_begin;
        for (int i = 0; i < n && ok; ++i, ++gi) {
          const int b = gi & 1;  // S(gi) goes over P(gi - 2), read by PV(gi - 2), issued before it
          for (int q = 0; q < K_ITEMS; ++q) {
            const bool big = q < K_ITEMS - 1;
            const uint32_t kbuf = take(big);
            if (kbuf == 0) { ok = false; break; }
            // descriptors of the item's first K step; the others differ only in
            // their start address (+32 bytes per K step, + a chunk per c)
            const uint64_t qd = sdesc_sw128(sbase + OFF_Q + 2 * q * CHUNK_Q, 16, 1024);
            const uint64_t kd = sdesc_sw128(kbuf, 16, 1024);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              if (!big && c == 1) break;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma<2>(tmem + S_COL + 128 * b, sdesc_advance(qd, c * CHUNK_Q + kk * 32),
                          sdesc_advance(kd, c * CHUNK_K + kk * 32), IDESC_S, (q > 0 || c > 0 || kk > 0) ? 1u : 0u);
            }
            if (big) release();  // the small item is released by the S_FULL commit below
          }
          if (!ok) break;
          tc_commit_pair(bar(BAR_S_FULL + b), 0x3);
          if (i == n - 1) tc_commit_pair(bar(BAR_Q_EMPTY), 0x3);
          if (i > 0 && !issue_pv(gi - 1, pc.t_begin + i - 1, i == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(gi - 1, pc.t_end - 1, n == 1)) break;
        ++npc;
      }
    }
  } else if (warp >= WARP_SOFTMAX && warp < WARP_SOFTMAX + 4) {
    // ------------------------------------------------- softmax + epilogue
    // A failed (timed-out) wait does not break these loops: every softmax
    // warp keeps the same sequence of named-barrier syncs and runs to the
    // end on whatever data is there; the device error word reports it.
    const int sp = warp & 3;                // TMEM sub-partition of this warp
    const int L = 32 * sp + lane;           // TMEM lane
    const int row = L & 63, half = L >> 6;  // head within CTA; token half / latent half
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * sp) << 16);
    const float c2 = p.scale_log2;
    PieceIter<kGrouped> it = it0;
    Piece pc;
    int gi = 0, gz = 0, bbase = 0;  // bbase: big-slot uses before this piece
    while (it.next(p, pc)) {
      const int n = pc.t_end - pc.t_begin;
      float m_ref = -INFINITY, lsum = 0.f;
      for (int i = 0; i < n; ++i, ++gi) {
        const int b = gi & 1, ti = pc.t_begin + i;
        const int vis_t = pc.vis - ti * TILE;  // visible tokens of this tile
        const int tok0 = OWN * half;            // this thread's first token within the tile
        mbar_wait_warp(bar(BAR_S_FULL + b), (gi >> 1) & 1, abort_flag);
        tc_fence_after();
        const uint32_t s_addr = lane_addr + S_COL + 128 * b;
        // pass 1: row max over this thread's 128 tokens, then with the partner lane
        float mx = -INFINITY;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t sr[32];
          tmem_ld32(s_addr + 32 * q4, sr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (tok0 + 32 * q4 + c < vis_t) mx = fmaxf(mx, __uint_as_float(sr[c]));
        }
        red[(gi & 1) * 128 + L] = mx;
        named_bar_sync(1, 128);
        mx = fmaxf(mx, red[(gi & 1) * 128 + (L ^ 64)]);
        bool rescale = false;
        float alpha = 1.f;
        if (i == 0) {
          m_ref = mx;
        } else {
          const bool need = (mx - m_ref) * c2 > RESCALE_LOG2;
          rescale = __any_sync(0xffffffffu, need);
          if (need) {
            alpha = ex2_approx((m_ref - mx) * c2);
            m_ref = mx;
          }
        }
        // pass 2: p = exp2((s - m) * scale * log2 e) as bf16 pairs. Chunk q4 holds
        // K groups 4 q4 .. 4 q4 + 3; a group is 8 tokens of each half of the tile,
        // the first half in columns 8 g + 0..3 and the second in 8 g + 4..7, in
        // both lanes of the row. The partner lane (L ^ 64) holds the other half.
        const float mo = m_ref * c2;
        float ps = 0.f;
        uint4 *xb = reinterpret_cast<uint4 *>(smem + OFF_XBUF);
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t sr[32];
          tmem_ld32(s_addr + 32 * q4, sr);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int t = tok0 + 32 * q4 + 2 * c;
            const float p0 = t < vis_t ? ex2_approx(fmaf(__uint_as_float(sr[2 * c]), c2, -mo)) : 0.f;
            const float p1 = t + 1 < vis_t ? ex2_approx(fmaf(__uint_as_float(sr[2 * c + 1]), c2, -mo)) : 0.f;
            ps += p0 + p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) xb[L * 4 + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          named_bar_sync(1, 128);
          uint32_t pw[32];
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const uint4 o = xb[(L ^ 64) * 4 + gg];
            const uint32_t mine[4] = {pk[4 * gg], pk[4 * gg + 1], pk[4 * gg + 2], pk[4 * gg + 3]};
            const uint32_t theirs[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              pw[8 * gg + e] = half == 0 ? mine[e] : theirs[e];
              pw[8 * gg + 4 + e] = half == 0 ? theirs[e] : mine[e];
            }
          }
          tmem_st32(s_addr + 32 * q4, pw);
          named_bar_sync(1, 128);  // the exchange buffer is reused by the next chunk
        }
        tmem_wait_st();
        // O is rescaled only after the previous tile's PV has finished with it
        if (gi > 0) mbar_wait_warp(bar(BAR_O_FULL), (gi - 1) & 1, abort_flag);
        tc_fence_after();
        if (rescale) {
#pragma unroll 1
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
        }
        lsum = lsum * alpha + ps;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(bar(BAR_P_FULL), rank);
        // partial block of the last tile: zero its value rows past the end in
        // the two value items (latent halves) that hold it; the MMA thread
        // signals as each one lands
        const int zc = partial_chunk(pc.vis, ti);
        if (zc >= 0) {
          const int valid = vis_t - BLK * zc;
          const int nrow = BLK - valid;
          for (int j = 0; j < 2; ++j) {
            mbar_wait_warp(bar(BAR_V_LANDED), gz & 1, abort_flag);
            ++gz;
            uint8_t *vb = smem + OFF_BIG + ((bbase + value_item(i, n, zc & 1, j)) % NBIG) * BIG + (zc >> 1) * HALF;
            // block slab = [chunk a][64 rows][128 B]: 16 16-byte words per row
            for (int e = L; e < nrow * 16; e += 128) {
              const int r = valid + e / 16, a = (e >> 3) & 1, w16 = e & 7;
              *reinterpret_cast<uint4 *>(vb + a * ATOM + r * 128 + w16 * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) arrive_leader(bar(BAR_ZERO_DONE), rank);
          }
        }
      }
      // ---------------------------------------------------------- epilogue
      mbar_wait_warp(bar(BAR_O_FULL), (gi - 1) & 1, abort_flag);
      tc_fence_after();
      redl[L] = lsum;
      named_bar_sync(1, 128);
      const float ltot = lsum + redl[L ^ 64];
      const float inv = 1.f / ltot;
      const float lse_v = m_ref * p.scale + logf(ltot);
      const int head = HPC * rank + row;
      // A TMEM load gives each thread 32 columns of its own head, so a warp
      // holds 32 heads x 32 columns. It transposes them, 16 columns at a time,
      // through its threads' own 2 KB of the exchange buffer (free here: every
      // thread has passed the last P exchange), so that a store instruction
      // writes 8 heads x 16 contiguous columns rather than 32 heads x 4 or 8.
      // The 16-byte chunk k of row r sits at chunk k ^ ((r >> 1) & 3) of the
      // row's 64 bytes: both the row writes and the column reads are free of
      // bank conflicts.
      float *stg = reinterpret_cast<float *>(smem + OFF_XBUF + 2048 * sp);
      const int head_w = HPC * rank + 32 * (sp & 1);  // head of the warp's row 0
      const int sw_w = (lane >> 1) & 3;
      const int r0 = lane >> 2, c4 = lane & 3;
#pragma unroll 1
      for (int q4 = 0; q4 < 8; ++q4) {
        const int j = q4 >> 2, part = q4 & 3;
        uint32_t o[32];
        tmem_ld32(lane_addr + 128 * j + 32 * part, o);
        tmem_wait_ld();
        const int col = 256 * j + 128 * half + 32 * part;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<float4 *>(stg + 16 * lane + 4 * (k ^ sw_w)) =
                make_float4(__uint_as_float(o[16 * h2 + 4 * k]) * inv, __uint_as_float(o[16 * h2 + 4 * k + 1]) * inv,
                            __uint_as_float(o[16 * h2 + 4 * k + 2]) * inv, __uint_as_float(o[16 * h2 + 4 * k + 3]) * inv);
          __syncwarp();
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const int r = r0 + 8 * k2;
            const float4 v = *reinterpret_cast<const float4 *>(stg + 16 * r + 4 * (c4 ^ ((r >> 1) & 3)));
            const int64_t at = (static_cast<int64_t>(pc.single ? pc.bj : pc.slot) * HEADS + head_w + r) * DC + col +
                               16 * h2 + 4 * c4;
            if (pc.single)
              *reinterpret_cast<uint2 *>(p.o_lat + at) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
            else
              *reinterpret_cast<float4 *>(p.part_o + at) = v;
          }
          __syncwarp();  // the rows are rewritten by the next half
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
      bbase += BIG_PER_TILE * n;
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
  if (warp == WARP_MMA) tmem_dealloc<2>(tmem, 512);
}

// Merge the split partials of every token row that was cut by cluster range
// boundaries: lse = log sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s.
// grid = BJ * 32 blocks of 128 threads: warp w of block g handles head
// 4 (g mod 32) + w of row g / 32, lane l its float4 columns l + 32 c, c < 4.
// The partials of COMBINE_CHUNK pieces (their lse and all four float4) are
// loaded together, one round trip per chunk, and merged with a running max.
constexpr int COMBINE_CHUNK = 2, COMBINE_BLOCKS_PER_ROW = HEADS / 4;
__global__ void __launch_bounds__(128) k_combine(Params p) {
  if (threadIdx.x == 0) griddep_launch_dependents();
  griddep_wait();
  const int bj = blockIdx.x / COMBINE_BLOCKS_PER_ROW;  // token row
  const int head = 4 * (blockIdx.x % COMBINE_BLOCKS_PER_ROW) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int BJ = p.B * p.n_q;
  const int u = unit_of_row(p, bj);
  int first, np;
  if (p.plan[2] == 0) {  // automatic plan: the unit's pieces are its clusters k0 .. k1, slots u + k
    const int G = p.plan[3], ncg = p.plan[4], grp = G > 1 ? u / p.B : 0;
    const int base = G > 1 ? p.plan[plan_tiles(BJ) + grp * p.B] : 0, Qt = p.plan[1];
    const int a = p.plan[plan_tiles(BJ) + u] - base, e = p.plan[plan_tiles(BJ) + u + 1] - base;
    if (e <= a) return;
    const int k0 = grp * ncg + a / Qt, k1 = grp * ncg + (e - 1) / Qt;
    first = u + k0;
    np = k1 - k0 + 1;
  } else {  // forced splits: the unit's pieces are slots piece_off[u] ..
    first = p.plan[plan_pieces(BJ) + u];
    np = p.plan[plan_pieces(BJ) + u + 1] - first;
  }
  if (np <= 1) return;
  const float *pl = p.part_lse + static_cast<int64_t>(first) * HEADS + head;
  const float4 *po =
      reinterpret_cast<const float4 *>(p.part_o + (static_cast<int64_t>(first) * HEADS + head) * DC) + lane;
  constexpr int64_t PIECE4 = static_cast<int64_t>(HEADS) * DC / 4;  // float4 stride between pieces
  float M = -INFINITY, Z = 0.f;
  float4 acc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < np; k += COMBINE_CHUNK) {
    float l[COMBINE_CHUNK];
    float4 x[COMBINE_CHUNK][4];
#pragma unroll
    for (int u = 0; u < COMBINE_CHUNK; ++u) {
      if (k + u < np) {
        l[u] = __ldcg(pl + static_cast<int64_t>(k + u) * HEADS);
#pragma unroll
        for (int c = 0; c < 4; ++c) x[u][c] = __ldcg(po + (k + u) * PIECE4 + 32 * c);
      } else {
        l[u] = -INFINITY;
      }
    }
    float Mn = M;
#pragma unroll
    for (int u = 0; u < COMBINE_CHUNK; ++u) Mn = fmaxf(Mn, l[u]);
    const float r = __expf(M - Mn);  // 0 on the first chunk (M = -inf, Mn finite)
    Z *= r;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      acc[c].x *= r;
      acc[c].y *= r;
      acc[c].z *= r;
      acc[c].w *= r;
    }
#pragma unroll
    for (int u = 0; u < COMBINE_CHUNK; ++u) {
      if (k + u < np) {
        const float wgt = __expf(l[u] - Mn);
        Z += wgt;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[c].x += wgt * x[u][c].x;
          acc[c].y += wgt * x[u][c].y;
          acc[c].z += wgt * x[u][c].z;
          acc[c].w += wgt * x[u][c].w;
        }
      }
    }
    M = Mn;
  }
  const float inv = 1.f / Z;
  uint2 *dst = reinterpret_cast<uint2 *>(p.o_lat + (static_cast<int64_t>(bj) * HEADS + head) * DC) + lane;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint2 out;
    out.x = pack_bf16x2(acc[c].x * inv, acc[c].y * inv);
    out.y = pack_bf16x2(acc[c].z * inv, acc[c].w * inv);
    dst[32 * c] = out;
  }
  if (lane == 0 && p.lse != nullptr) p.lse[static_cast<int64_t>(bj) * HEADS + head] = M + logf(Z);
}

}  // namespace dec

// Workspace: the plan (3 words, tile offsets and piece offsets of the BJ + 1
// row boundaries), then fp32 split partials. Slots: at most BJ + clusters for
// the automatic plan; for S forced splits at most BJ * min(S, tiles of the
// longest row), max_seq_len (0 = unknown) bounding the tiles.
constexpr size_t decode_plan_bytes(size_t BJ) { return ((2 * BJ + 7) * sizeof(int32_t) + 255) & ~size_t(255); }
inline size_t decode_tc_slots(int B, int n_q, int sms, int splits, int64_t max_seq_len) {
  const size_t BJ = static_cast<size_t>(B) * n_q;
  size_t slots = BJ + static_cast<size_t>(sms / 2);
  if (splits > 0) {
    int64_t per_row = splits;
    if (max_seq_len > 0) per_row = std::min<int64_t>(per_row, (max_seq_len + dec::TILE - 1) / dec::TILE);
    slots = std::max(slots, BJ * static_cast<size_t>(per_row));
  }
  return slots;
}
inline size_t decode_tc_ws(int B, int n_q, int sms, int splits = 0, int64_t max_seq_len = 0) {
  const size_t BJ = static_cast<size_t>(B) * n_q;
  const size_t slots = decode_tc_slots(B, n_q, sms, splits, max_seq_len);
  return decode_plan_bytes(BJ) + slots * dec::HEADS * dec::DC * sizeof(float) + slots * dec::HEADS * sizeof(float);
}

}  // namespace mla
