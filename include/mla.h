/*
 * mla.h — C ABI of libmla.so, the B200 (sm_100a) implementation of the
 * absorbed-form decode hot path of Multi-head Latent Attention (MLA,
 * DeepSeek-V2).
 *
 * Notation (MLA walk-through, h.sjds.net, section 1; DeepSeek-V2 MLA
 * explainer, modelers.csdn.net, equations 9-13):
 *   d     model width (5120 for DeepSeek-V2, 7168 for V3)
 *   n_h   heads (128), d_h per-head dim (128)
 *   d_c   KV latent dim (512), d_cq query latent dim d_c' (1536)
 *   d_r   decoupled RoPE dim d_R (64)
 *   D     = d_c + d_r, the width of one cached row [c_KV | k_R] (576)
 *   B     sequences, n_q new tokens per sequence this step, T = B * n_q
 *         token rows; row t = b * n_q + j holds new token j of sequence b.
 *
 * Conventions shared by every entry point:
 *   - All pointers to tensors are DEVICE pointers unless noted; the caller
 *     owns every buffer. No entry point allocates or frees device memory.
 *   - Tensors are dense row-major (C order) with the shapes given below and
 *     16-byte aligned base addresses (the tensor-memory-accelerator loads
 *     need it). Element type is the storage dtype of mla_dims.dtype (bf16 or
 *     fp32) unless stated otherwise; arithmetic accumulates in fp32.
 *   - Weights are stored out x in, as the pages write them (W_DKV is d_c x d,
 *     eq. 9; W_UK, W_UV are n_h*d_h x d_c, eqs. 10-11). Head h owns rows
 *     h*d_h .. h*d_h+d_h-1 of W_UQ, W_UK, W_UV and rows h*d_r .. h*d_r+d_r-1
 *     of W_QR.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and never synchronises, except
 *     mla_get_device_error.
 *   - Arguments are validated on the host before any launch; on an invalid
 *     argument the call returns MLA_ERR_INVALID_ARG (or MLA_ERR_UNSUPPORTED
 *     for valid but unimplemented shapes) and writes nothing.
 *     mla_last_error_message() then describes the problem.
 *   - Contents of device arrays (seq_lens, positions, seq_idx, block tables)
 *     cannot be checked on the host without a synchronisation. Kernels check
 *     them and, on a bad value, skip the access, set the library's device
 *     error word and go on; mla_get_device_error reports it.
 *   - `ws` is caller-owned device scratch of at least
 *     mla_workspace_size(...) bytes (may be NULL when that size is 0); it
 *     must not be shared by calls that run concurrently.
 *   - A CUDA launch failure returns MLA_ERR_CUDA.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,
  MLA_ERR_UNSUPPORTED = 2,
  MLA_ERR_WORKSPACE = 3,
  MLA_ERR_CUDA = 4,
  MLA_ERR_TIMEOUT = 5,   /* a kernel's bounded wait expired (device error word) */
  MLA_ERR_DEVICE_DATA = 6 /* a kernel found an out-of-range index (device error word) */
} mla_status;

typedef enum { MLA_BF16 = 0, MLA_FP32 = 1 } mla_dtype;

/* Layer dimensions. softmax_scale <= 0 selects 1/sqrt(d_h + d_r): the score
 * of step 4 lives in the (d_h + d_r) = 192-dim concatenation of the content
 * and position parts (MLA walk-through, section 1 step 4). RoPE uses
 * RoFormer's interleaved pairs (2i, 2i+1) with theta_i = rope_base^(-2i/d_r). */
typedef struct {
  int32_t d, n_h, d_h, d_c, d_cq, d_r;
  double rope_base;
  float softmax_scale;
  int32_t dtype; /* mla_dtype: storage of h, weights, cache, q, o_lat, o */
} mla_dims;

/* Latent cache (MLA walk-through, section 1 step 1: each token keeps only
 * [c_KV ; k_R], d_c + d_r numbers, no head label and no K/V split).
 *   contiguous (paged = 0): data = [num_seqs][max_len][D]; row of
 *     (b, pos) = b * max_len + pos.
 *   paged (paged = 1): data = [num_blocks][block_size][D] and block_table =
 *     [num_seqs][max_blocks_per_seq] int32 (device); row of (b, pos) =
 *     block_table[b][pos / block_size] * block_size + pos % block_size.
 * The cache struct itself lives in host memory; data and block_table are
 * device pointers. */
typedef struct {
  void *data;
  int32_t paged;
  int32_t block_size;
  const int32_t *block_table;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int64_t max_len;    /* contiguous only */
  int64_t num_blocks; /* paged only */
} mla_cache;

/* Write path (MLA walk-through, section 1 step 1; DeepSeek-V2 explainer,
 * eq. 9): for every new token row t,
 *   c_KV = W_DKV h_t  (d_c),  k_R = RoPE(W_KR h_t, positions[t])  (d_r),
 * rounded once to the storage dtype and stored as the cache row of
 * (seq_idx[t], positions[t]).
 *   h         [T][d]            W_DKV [d_c][d]     W_KR [d_r][d]
 *   seq_idx   [T] int32 device  positions [T] int32 device
 * A row whose (seq_idx, position) falls outside the cache is not written and
 * raises MLA_ERR_DEVICE_DATA in the device error word. */
mla_status mla_cache_append(const mla_dims *dims, const void *h, const void *W_DKV,
                            const void *W_KR, const int32_t *seq_idx, const int32_t *positions,
                            int32_t T, const mla_cache *cache, void *ws, size_t ws_bytes,
                            void *stream);

/* Query path and absorption (MLA walk-through, section 1 step 3 and section
 * 3 order B; DeepSeek-V2 explainer, eqs. 12-13 and the remark that W_UK can
 * be absorbed on the query side):
 *   c_Q = W_DQ h_t (d_cq);  q_C,h = W_UQ_h c_Q (d_h);
 *   q_R,h = RoPE(W_QR_h c_Q, positions[t]) (d_r);  q_lat,h = W_UK_h^T q_C,h (d_c).
 *   h [T][d]  W_DQ [d_cq][d]  W_UQ [n_h*d_h][d_cq]  W_QR [n_h*d_r][d_cq]
 *   W_UK [n_h*d_h][d_c]  positions [T] int32 device
 *   q (output) [T][n_h][D] = [q_lat | q_R] per head, storage dtype.
 * c_Q and q_C are tensor-core operands and are rounded once to the storage
 * dtype: c_Q in the workspace, q_C in shared memory (at most 128 token rows,
 * one CTA per head) or in the workspace (more rows); q is rounded once. */
mla_status mla_absorb_q(const mla_dims *dims, const void *h, const void *W_DQ, const void *W_UQ,
                        const void *W_QR, const void *W_UK, const int32_t *positions, int32_t T,
                        void *q, void *ws, size_t ws_bytes, void *stream);

/* Attention in latent space (MLA walk-through, section 1 step 4 and section
 * 3 order B): for token row t = b*n_q + j, head h, and every cached position
 * i < L_b - n_q + 1 + j (L_b = seq_lens[b] counts cached rows after this
 * step's append; new token j sits at position L_b - n_q + j, causal within
 * the step):
 *   s_i = scale * (q_lat,h . c_KV_i + q_R,h . k_R_i),  p = softmax_i(s),
 *   o_lat[t][h] = sum_i p_i c_KV_i (d_c),  lse[t][h] = log sum_i exp(s_i).
 *   q [B*n_q][n_h][D]   seq_lens [B] int32 device
 *   o_lat (output) [B*n_q][n_h][d_c] storage dtype
 *   lse (output, may be NULL) [B*n_q][n_h] float32 (natural log)
 * num_splits (split-KV): 0 = automatic: the tensor-core path concatenates the
 * 256-token KV tiles of all token rows, cuts that line into one equal share
 * per pair of SMs, and merges every row cut by a share boundary with a
 * log-sum-exp combine. With n_q > 1 (and at least n_q pairs of SMs) the pairs
 * form n_q equal groups, one per query position j; each group cuts the line of
 * the rows of position j into ranges of one common length, so the n_q rows of
 * a sequence read the same cache tiles at about the same time (L2 reuse).
 * S > 0 = forced: every token row is cut into
 * min(S, its tiles) pieces of near-equal tile counts (S = 1: no split), each
 * pair of SMs takes the pieces that start in its equal share of the tile line,
 * and rows of more than one piece are merged by the same combine. The
 * CUDA-core path (fp32 or other dims) never splits and ignores S. Results
 * agree within rounding for every S.
 * seq_lens[b] < n_q or beyond the cache capacity raises MLA_ERR_DEVICE_DATA
 * and that sequence's outputs are left unwritten. */
mla_status mla_decode(const mla_dims *dims, const void *q, const mla_cache *cache,
                      const int32_t *seq_lens, int32_t B, int32_t n_q, void *o_lat, float *lse,
                      int32_t num_splits, void *ws, size_t ws_bytes, void *stream);

/* mla_decode without a caller workspace. The pages have no counterpart: this
 * is a convenience of this library for callers that cannot pass scratch
 * memory. Same computation, arguments (minus num_splits, ws, ws_bytes),
 * outputs and error behaviour as mla_decode.
 *   Scratch: a static device array of this library, sized for at most 64 token
 *   rows (B * n_q <= 64) and 74 decode clusters (one 148-SM B200), about
 *   35 MB, reserved when the library's device code is loaded. Larger calls
 *   return MLA_ERR_UNSUPPORTED with the reason in mla_last_error_message().
 *   The library allocates nothing.
 *   The first call on each device, and the first call after a device reset,
 *   looks up that device's copy of the array (cudaGetSymbolAddress); make that
 *   call before any stream capture.
 *   Nothing in the scratch needs to start at zero: every call writes each
 *   byte it later reads.
 *   The scratch is shared by all callers in the process: calls that can
 *   overlap in time on one device (different streams, or different host
 *   threads) race on it and must be serialised by the caller. */
mla_status mla_decode_noalloc(const mla_dims *dims, const void *q, const mla_cache *cache,
                              const int32_t *seq_lens, int32_t B, int32_t n_q, void *o_lat, float *lse,
                              void *stream);

/* Per-head readout, decompressed once at the end (MLA walk-through, section
 * 3 order B; DeepSeek-V2 explainer, eq. 11):
 *   o[t][h*d_h + i] = sum_j W_UV[h*d_h + i][j] o_lat[t][h][j].
 *   o_lat [T][n_h][d_c]   W_UV [n_h*d_h][d_c]   o (output) [T][n_h*d_h]. */
mla_status mla_out_proj(const mla_dims *dims, const void *o_lat, const void *W_UV, int32_t T,
                        void *o, void *ws, size_t ws_bytes, void *stream);

/* Output projection (MLA walk-through, section 1 step 5: the n_h head outputs
 * of a token, concatenated, are projected back to the model width):
 *   y[t][r] = sum_k W_O[r][k] o[t][k],  k < n_h*d_h.
 *   o [T][n_h*d_h] (the output of mla_out_proj)   W_O [d][n_h*d_h]
 *   y (output) [T][d], storage dtype, rounded once from fp32 sums. */
mla_status mla_o_proj(const mla_dims *dims, const void *o, const void *W_O, int32_t T, void *y, void *ws,
                      size_t ws_bytes, void *stream);

/* W_UV absorbed into the output projection (DeepSeek-V2 explainer, section 3:
 * the remark that W_UV can be folded into W_O; MLA walk-through, section 1
 * step 5 and section 3 order B): since o_h = W_UV_h o_lat,h,
 *   W_OV[r][h*d_c + j] = sum_i W_O[r][h*d_h + i] W_UV[h*d_h + i][j],
 * a d x n_h*d_c matrix, rounded once to the storage dtype. An offline step:
 * W_O [d][n_h*d_h], W_UV [n_h*d_h][d_c], W_OV (output) [d][n_h*d_c]. No
 * workspace. */
mla_status mla_absorb_wo(const mla_dims *dims, const void *W_O, const void *W_UV, void *W_OV, void *stream);

/* Output projection straight from the latent readout, with W_OV from
 * mla_absorb_wo: y[t][r] = sum_k W_OV[r][k] o_lat[t][k], k < n_h*d_c (the same
 * y as mla_out_proj followed by mla_o_proj, up to rounding).
 *   o_lat [T][n_h][d_c]   W_OV [d][n_h*d_c]   y (output) [T][d]. */
mla_status mla_o_proj_latent(const mla_dims *dims, const void *o_lat, const void *W_OV, int32_t T, void *y,
                             void *ws, size_t ws_bytes, void *stream);

/* Merged absorption matrix (MLA walk-through, section 3 order B: the merged
 * matrix can be computed offline): W_UQK_h = W_UK_h^T W_UQ_h, so that
 * q_lat,h = W_UQK_h c_Q in one product.
 *   W_UQK[h*d_c + j][c] = sum_i W_UK[h*d_h + i][j] W_UQ[h*d_h + i][c],
 * n_h*d_c x d_cq, rounded once. W_UQ [n_h*d_h][d_cq], W_UK [n_h*d_h][d_c].
 * No workspace. */
mla_status mla_absorb_merge(const mla_dims *dims, const void *W_UQ, const void *W_UK, void *W_UQK, void *stream);

/* mla_absorb_q with the merged matrix: c_Q = W_DQ h_t, q_lat,h = W_UQK_h c_Q,
 * q_R,h = RoPE(W_QR_h c_Q, positions[t]); same q layout and rounding points
 * as mla_absorb_q (c_Q rounded once to the storage dtype). */
mla_status mla_absorb_q_merged(const mla_dims *dims, const void *h, const void *W_DQ, const void *W_UQK,
                               const void *W_QR, const int32_t *positions, int32_t T, void *q, void *ws,
                               size_t ws_bytes, void *stream);

/* Front end of the step in one call: mla_cache_append and mla_absorb_q over
 * the same h_t (MLA walk-through, section 1 steps 1 and 3: both paths start
 * from h_t). On the tensor-core path h is read once, by one weight-streaming
 * product [W_DKV; W_KR; W_DQ] h whose finalize writes the cache rows and c_Q;
 * the per-head query chain follows. Results, arguments and error behaviour
 * are those of the two calls. */
mla_status mla_front_end(const mla_dims *dims, const void *h, const void *W_DKV, const void *W_KR,
                         const void *W_DQ, const void *W_UQ, const void *W_QR, const void *W_UK,
                         const int32_t *seq_idx, const int32_t *positions, int32_t T, const mla_cache *cache,
                         void *q, void *ws, size_t ws_bytes, void *stream);

/* Per-head queries without absorption, for order A (MLA walk-through,
 * section 1 step 3): c_Q = W_DQ h_t; q_C,h = W_UQ_h c_Q (d_h);
 * q_R,h = RoPE(W_QR_h c_Q, positions[t]) (d_r), written as
 *   qa (output) [T][n_h][d_h + d_r] = [q_C,h | q_R,h], storage dtype
 * (c_Q rounded once to the storage dtype, as in mla_absorb_q). */
mla_status mla_query_heads(const mla_dims *dims, const void *h, const void *W_DQ, const void *W_UQ,
                           const void *W_QR, const int32_t *positions, int32_t T, void *qa, void *ws,
                           size_t ws_bytes, void *stream);

/* Attention in order A, the training form (MLA walk-through, section 3 order
 * A: decompress, then the ordinary dot product): for head h and cached row i
 *   K_h,i = [W_UK_h c_KV_i ; k_R,i] (d_h + d_r),  V_h,i = W_UV_h c_KV_i (d_h),
 * and for token row t = b*n_q + j (new token j of sequence b at position
 * L_b - n_q + j, causal within the chunk of n_q tokens; L_b = seq_lens[b]):
 *   o[t][h] = sum_i softmax_i(scale qa[t][h] . K_h,i) V_h,i,  i <= L_b - n_q + j,
 * the same o as mla_decode followed by mla_out_proj (order B), up to rounding.
 *   qa [B*n_q][n_h][d_h + d_r] (mla_query_heads)   W_UK, W_UV [n_h*d_h][d_c]
 *   o (output) [B*n_q][n_h][d_h], storage dtype.
 * The tensor-core path decompresses K_C and V for every physical cache row
 * into the workspace (bf16, 2 * n_h * rows * d_h * 2 bytes; rows =
 * num_blocks * block_size, or num_seqs * max_len) and stores o rounded once.
 * Bad seq_lens raise MLA_ERR_DEVICE_DATA and leave that sequence unwritten. */
mla_status mla_attend_order_a(const mla_dims *dims, const void *qa, const void *W_UK, const void *W_UV,
                              const mla_cache *cache, const int32_t *seq_lens, int32_t B, int32_t n_q, void *o,
                              void *ws, size_t ws_bytes, void *stream);

/* Self-test of the failure path (no counterpart on the pages). Launches one
 * small projection kernel whose copy engine is told to issue nothing, so that
 * its MMA thread's bounded wait runs out after wait_ns nanoseconds; the kernel
 * then records MLA_ERR_TIMEOUT in the device error word (read it with
 * mla_get_device_error), frees its tensor memory and returns, with no copy in
 * flight. The context stays usable. scratch: >= 65536 bytes of device memory,
 * overwritten. */
mla_status mla_selftest_timeout(uint64_t wait_ns, void *scratch, size_t scratch_bytes, void *stream);

/* Scratch size in bytes for one call of `op` (MLA_OP_*). `rows` is T for
 * append/absorb/out_proj/o_proj and B for decode; n_q, max_seq_len and
 * num_splits are used by decode only. max_seq_len bounds the tiles of a row
 * for forced splits (0 = unknown: the size then covers num_splits pieces for
 * every row); mla_decode itself requires the size for max_seq_len = the
 * cache's capacity (max_len, or max_blocks_per_seq * block_size). For
 * MLA_OP_ATTEND_A, max_seq_len is the number of physical cache rows
 * (num_blocks * block_size, or num_seqs * max_len). */
enum {
  MLA_OP_APPEND = 0, MLA_OP_ABSORB = 1, MLA_OP_DECODE = 2, MLA_OP_OUT_PROJ = 3, MLA_OP_O_PROJ = 4,
  MLA_OP_O_PROJ_LATENT = 5, MLA_OP_ABSORB_MERGED = 6, MLA_OP_FRONT_END = 7, MLA_OP_ABSORB_WO = 8,
  MLA_OP_QUERY_HEADS = 9, MLA_OP_ATTEND_A = 10
};
size_t mla_workspace_size(const mla_dims *dims, int32_t op, int32_t rows, int32_t n_q,
                          int64_t max_seq_len, int32_t num_splits);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns MLA_OK, MLA_ERR_TIMEOUT, MLA_ERR_DEVICE_DATA or MLA_ERR_CUDA. */
mla_status mla_get_device_error(void *stream);

const char *mla_status_string(mla_status s);

/* Text of the last host-side validation or CUDA error on this thread. */
const char *mla_last_error_message(void);

/* Which kernel family serves a call with these dims: 1 = sm_100a tensor
 * cores (tcgen05/TMEM/TMA), 0 = CUDA-core kernels (fp32 storage or dims the
 * tensor-core kernels are not built for). */
int32_t mla_uses_tensor_cores(const mla_dims *dims, int32_t op);

/* Launch overlap (process-wide, off by default). When on, every tensor-core
 * kernel is launched with programmatic stream serialization: it may be
 * scheduled while the kernel ahead of it on the stream is still running, set
 * up its barriers and tensor memory, and start streaming the weight matrices
 * of its call (W_DKV/W_KR, W_DQ, W_UQ/W_QR/W_UK, W_UV); it reads activations,
 * the cache, sequence lengths or positions, and writes any output, only
 * after that kernel has completed. The caller guarantees that the weights of
 * a call are not written by the work enqueued on the stream just before it.
 * Results are identical either way. Returns MLA_OK. No counterpart on the
 * pages: it is a property of how the calls are launched, not of the method. */
mla_status mla_set_launch_overlap(int32_t enable);
int32_t mla_get_launch_overlap(void);

/* Number of kernels this library has launched in this process (all devices,
 * all threads), counted when they are enqueued; a launch captured into a CUDA
 * graph counts once at capture, however often the graph is replayed. Lets
 * callers count launches inside a timed region. */
uint64_t mla_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
