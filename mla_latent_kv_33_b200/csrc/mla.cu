// libmla: host side of the C ABI declared in include/mla.h.
//
// Validates arguments, sizes workspaces, builds TMA tensor maps and launches
// the kernels. Two kernel families serve the calls:
//   - sm_100a tensor-core kernels (tcgen05 MMA into tensor memory, TMA tile
//     loads, mbarrier pipelines) for bf16 storage at the DeepSeek-V2/V3 head
//     geometry (n_h = 128, d_h = 128, d_c = 512, d_r = 64);
//   - CUDA-core kernels for fp32 storage and other dims.
// mla_uses_tensor_cores() reports which family a call will use; the choice
// depends only on dims, never on a runtime failure.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>

#include "../../include/mla.h"
#include "common.cuh"
#include "ptx.cuh"
#include "simt.cuh"
#include "gemm_tc.cuh"
#include "decode_tc.cuh"
#include "prefill_tc.cuh"

namespace {

thread_local std::string g_msg;
std::atomic<uint64_t> g_launches{0};

// Every kernel launch goes through this macro so the count is exact.
#define MLA_LAUNCH(...) (g_launches.fetch_add(1, std::memory_order_relaxed), __VA_ARGS__)

std::atomic<int> g_overlap{0};

// Launch of a tensor-core kernel: plain, or with programmatic stream
// serialization while launch overlap is on (the kernels wait for the grid
// ahead of them with griddepcontrol.wait before touching its outputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_tc(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args &&...args) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_overlap.load(std::memory_order_relaxed) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

mla_status fail(mla_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
mla_status fail(mla_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_msg = buf;
  return s;
}

mla_status cuda_check(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MLA_OK;
}

// Status of a launch_tc() call: its own error, else any pending one.
mla_status launched(cudaError_t e, const char *what) {
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  return cuda_check(what);
}

// cudaFuncSetAttribute applies to the current device: a kernel's dynamic
// shared memory limit is raised once per device (bit `device` of its mask).
enum SmemKernel {
  SMEM_GEMM = 0, SMEM_ABSORB = 1, SMEM_DECODE = 2, SMEM_ATTEND_A = 3, SMEM_DECODE_NQ = 4, SMEM_GEMM_RES = 5, SMEM_KERNELS = 6
};
std::atomic<uint64_t> g_smem_raised[SMEM_KERNELS];

mla_status raise_smem_limit(const void *kernel, SmemKernel which, int bytes, const char *what) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_check(what);
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit != 0 && (g_smem_raised[which].load(std::memory_order_acquire) & bit) != 0) return MLA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return cuda_check(what);
  g_smem_raised[which].fetch_or(bit, std::memory_order_release);
  return MLA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(const mla_dims *d) { return d->dtype == MLA_BF16 ? 2 : 4; }

float softmax_scale(const mla_dims *d) {
  return d->softmax_scale > 0.f ? d->softmax_scale
                                : static_cast<float>(1.0 / std::sqrt(static_cast<double>(d->d_h + d->d_r)));
}

mla_status check_dims(const mla_dims *d) {
  if (d == nullptr) return fail(MLA_ERR_INVALID_ARG, "dims is NULL");
  if (d->d <= 0 || d->n_h <= 0 || d->d_h <= 0 || d->d_c <= 0 || d->d_cq <= 0 || d->d_r <= 0)
    return fail(MLA_ERR_INVALID_ARG, "all dims must be positive");
  if (d->d_r % 2 != 0) return fail(MLA_ERR_INVALID_ARG, "d_r must be even (RoPE pairs)");
  if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32)
    return fail(MLA_ERR_INVALID_ARG, "dtype must be MLA_BF16 or MLA_FP32");
  if (!(d->rope_base > 1.0)) return fail(MLA_ERR_INVALID_ARG, "rope_base must be > 1");
  if (d->d_c + d->d_r > 1024)
    return fail(MLA_ERR_UNSUPPORTED, "d_c + d_r > 1024 is not supported");
  return MLA_OK;
}

mla_status check_cache(const mla_cache *c, int D) {
  (void)D;
  if (c == nullptr || c->data == nullptr) return fail(MLA_ERR_INVALID_ARG, "cache or cache->data is NULL");
  if (!aligned16(c->data)) return fail(MLA_ERR_INVALID_ARG, "cache->data must be 16-byte aligned");
  if (c->num_seqs <= 0) return fail(MLA_ERR_INVALID_ARG, "cache->num_seqs must be positive");
  if (c->paged) {
    if (c->block_table == nullptr) return fail(MLA_ERR_INVALID_ARG, "paged cache needs block_table");
    if (c->block_size <= 0 || c->max_blocks_per_seq <= 0 || c->num_blocks <= 0)
      return fail(MLA_ERR_INVALID_ARG, "paged cache needs block_size, max_blocks_per_seq, num_blocks > 0");
  } else if (c->max_len <= 0) {
    return fail(MLA_ERR_INVALID_ARG, "contiguous cache needs max_len > 0");
  }
  return MLA_OK;
}

mla::CacheView view_of(const mla_cache *c) {
  mla::CacheView v;
  v.data = c->data;
  v.block_table = c->block_table;
  v.max_len = c->max_len;
  v.num_blocks = c->num_blocks;
  v.paged = c->paged;
  v.block_size = c->block_size;
  v.max_blocks_per_seq = c->max_blocks_per_seq;
  v.num_seqs = c->num_seqs;
  return v;
}

// Longest sequence the cache can hold (bounds the tiles of a row).
int64_t cache_capacity(const mla_cache *c) {
  return c->paged ? static_cast<int64_t>(c->max_blocks_per_seq) * c->block_size : c->max_len;
}

bool tc_geometry(const mla_dims *d) {
  return d->dtype == MLA_BF16 && d->n_h == 128 && d->d_h == 128 && d->d_c == 512 && d->d_r == 64 &&
         d->d % 64 == 0 && d->d_cq % 64 == 0;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

// ------------------------------------------------------ CUDA-core variants --

template <typename T>
void launch_linear(const T *W, int64_t w_sb, int64_t w_sn, int64_t w_sk, const void *X, bool x_fp32,
                   int64_t x_sb, int64_t x_st, float *Y, int64_t y_sb, int64_t y_st, int N, int K, int Tn,
                   int batches, cudaStream_t st) {
  dim3 grid((N + 7) / 8, Tn, batches);
  if (x_fp32)
    MLA_LAUNCH(mla::k_simt_linear<T, float><<<grid, 256, 0, st>>>(W, w_sb, w_sn, w_sk, static_cast<const float *>(X),
                                                       x_sb, x_st, Y, y_sb, y_st, N, K));
  else
    MLA_LAUNCH(mla::k_simt_linear<T, T><<<grid, 256, 0, st>>>(W, w_sb, w_sn, w_sk, static_cast<const T *>(X), x_sb,
                                                   x_st, Y, y_sb, y_st, N, K));
}

template <typename T>
mla_status simt_append(const mla_dims *d, const void *h, const void *W_DKV, const void *W_KR,
                       const int32_t *seq_idx, const int32_t *positions, int Tn, const mla_cache *c,
                       void *ws, cudaStream_t st) {
  const int D = d->d_c + d->d_r;
  float *rows = static_cast<float *>(ws);  // [T][D] = [W_DKV h_t | W_KR h_t]
  launch_linear<T>(static_cast<const T *>(W_DKV), 0, d->d, 1, h, false, 0, d->d, rows, 0, D, d->d_c, d->d,
                   Tn, 1, st);
  launch_linear<T>(static_cast<const T *>(W_KR), 0, d->d, 1, h, false, 0, d->d, rows + d->d_c, 0, D, d->d_r,
                   d->d, Tn, 1, st);
  MLA_LAUNCH(mla::k_simt_append_store<T><<<Tn, 128, 0, st>>>(rows, D, d->d_c, d->d_r, d->rope_base, seq_idx,
                                                  positions, view_of(c)));
  return cuda_check("append (CUDA cores)");
}

size_t simt_append_ws(const mla_dims *d, int Tn) {
  return sizeof(float) * static_cast<size_t>(Tn) * (d->d_c + d->d_r);
}

template <typename T>
mla_status simt_absorb(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQ,
                       const void *W_QR, const void *W_UK, const int32_t *positions, int Tn, void *q,
                       void *ws, cudaStream_t st) {
  const int64_t HD = static_cast<int64_t>(d->n_h) * d->d_h;
  const int64_t HR = static_cast<int64_t>(d->n_h) * d->d_r;
  const int64_t HC = static_cast<int64_t>(d->n_h) * d->d_c;
  float *cq = static_cast<float *>(ws);          // [T][d_cq]
  float *qc = cq + static_cast<int64_t>(Tn) * d->d_cq;  // [T][n_h*d_h]
  float *qr = qc + Tn * HD;                      // [T][n_h*d_r]
  float *ql = qr + Tn * HR;                      // [T][n_h][d_c]
  launch_linear<T>(static_cast<const T *>(W_DQ), 0, d->d, 1, h, false, 0, d->d, cq, 0, d->d_cq, d->d_cq, d->d,
                   Tn, 1, st);
  launch_linear<T>(static_cast<const T *>(W_UQ), 0, d->d_cq, 1, cq, true, 0, d->d_cq, qc, 0, HD,
                   static_cast<int>(HD), d->d_cq, Tn, 1, st);
  launch_linear<T>(static_cast<const T *>(W_QR), 0, d->d_cq, 1, cq, true, 0, d->d_cq, qr, 0, HR,
                   static_cast<int>(HR), d->d_cq, Tn, 1, st);
  // q_lat,h[j] = sum_i W_UK[h*d_h + i][j] q_C,h[i]: batch = head, W(h, n=j, k=i)
  launch_linear<T>(static_cast<const T *>(W_UK), static_cast<int64_t>(d->d_h) * d->d_c, 1, d->d_c, qc, true,
                   d->d_h, HD, ql, d->d_c, HC, d->d_c, d->d_h, Tn, d->n_h, st);
  MLA_LAUNCH(mla::k_simt_q_store<T><<<Tn * d->n_h, 128, 0, st>>>(ql, qr, d->n_h, d->d_c, d->d_r, d->rope_base,
                                                      positions, static_cast<T *>(q)));
  return cuda_check("absorb (CUDA cores)");
}

size_t simt_absorb_ws(const mla_dims *d, int Tn) {
  const size_t t = static_cast<size_t>(Tn);
  return sizeof(float) * t * (d->d_cq + static_cast<size_t>(d->n_h) * (d->d_h + d->d_r + d->d_c));
}

template <typename T>
mla_status simt_decode(const mla_dims *d, const void *q, const mla_cache *c, const int32_t *seq_lens, int B,
                       int n_q, void *o_lat, float *lse, cudaStream_t st) {
  const int rows = B * n_q * d->n_h;
  const size_t smem = sizeof(float) * 8 * d->d_c;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(mla::k_simt_decode<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
  MLA_LAUNCH(mla::k_simt_decode<T><<<rows, 256, smem, st>>>(static_cast<const T *>(q), view_of(c), seq_lens, n_q,
                                                 d->n_h, d->d_c, d->d_r, softmax_scale(d),
                                                 static_cast<T *>(o_lat), lse));
  return cuda_check("decode (CUDA cores)");
}

template <typename T>
mla_status simt_out_proj(const mla_dims *d, const void *o_lat, const void *W_UV, int Tn, void *o, void *ws,
                         cudaStream_t st) {
  // o[t][h*d_h + i] = sum_j W_UV[h*d_h+i][j] o_lat[t][h][j]: batch = head
  const int64_t HD = static_cast<int64_t>(d->n_h) * d->d_h;
  float *y = static_cast<float *>(ws);  // [T][n_h*d_h]
  launch_linear<T>(static_cast<const T *>(W_UV), static_cast<int64_t>(d->d_h) * d->d_c, d->d_c, 1, o_lat,
                   false, d->d_c, static_cast<int64_t>(d->n_h) * d->d_c, y, d->d_h, HD, d->d_h, d->d_c, Tn,
                   d->n_h, st);
  const int64_t n = Tn * HD;
  const int64_t blocks = (n + 255) / 256;
  MLA_LAUNCH(mla::k_simt_store<T><<<static_cast<int>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(y, static_cast<T *>(o), n));
  return cuda_check("out_proj (CUDA cores)");
}

template <typename T>
mla_status simt_o_proj(const mla_dims *d, const void *o, const void *W_O, int Tn, void *y, void *ws, cudaStream_t st) {
  // y[t][r] = sum_k W_O[r][k] o[t][k]
  const int64_t HD = static_cast<int64_t>(d->n_h) * d->d_h;
  float *acc = static_cast<float *>(ws);  // [T][d]
  launch_linear<T>(static_cast<const T *>(W_O), 0, HD, 1, o, false, 0, HD, acc, 0, d->d, d->d, static_cast<int>(HD),
                   Tn, 1, st);
  const int64_t n = static_cast<int64_t>(Tn) * d->d;
  const int64_t blocks = (n + 255) / 256;
  MLA_LAUNCH(mla::k_simt_store<T><<<static_cast<int>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(acc, static_cast<T *>(y), n));
  return cuda_check("o_proj (CUDA cores)");
}

size_t simt_o_proj_ws(const mla_dims *d, int Tn) { return sizeof(float) * static_cast<size_t>(Tn) * d->d; }

size_t simt_out_proj_ws(const mla_dims *d, int Tn) {
  return sizeof(float) * static_cast<size_t>(Tn) * d->n_h * d->d_h;
}

// out(h, a, b) = sum_i L(h, i, a) R(h, i, b), i < d_h, rounded once to T.
template <typename T>
void launch_head_product(const void *L, int64_t l_h, int64_t l_i, int64_t l_a, const void *R, int64_t r_h,
                         int64_t r_i, int64_t r_b, void *out, int64_t o_h, int64_t o_a, int64_t o_b, int A, int Bn,
                         int I, int H, cudaStream_t st) {
  dim3 grid((Bn + 255) / 256, A, H);
  MLA_LAUNCH(mla::k_simt_head_product<T><<<grid, 256, 0, st>>>(static_cast<const T *>(L), l_h, l_i, l_a,
                                                                static_cast<const T *>(R), r_h, r_i, r_b,
                                                                static_cast<T *>(out), o_h, o_a, o_b, A, Bn, I));
}

template <typename T>
mla_status simt_absorb_wo(const mla_dims *d, const void *W_O, const void *W_UV, void *W_OV, cudaStream_t st) {
  // W_OV[r][h d_c + j] = sum_i W_O[r][h d_h + i] W_UV[h d_h + i][j]
  const int64_t HD = static_cast<int64_t>(d->n_h) * d->d_h, HC = static_cast<int64_t>(d->n_h) * d->d_c;
  launch_head_product<T>(W_O, d->d_h, 1, HD, W_UV, static_cast<int64_t>(d->d_h) * d->d_c, d->d_c, 1, W_OV, d->d_c,
                         HC, 1, d->d, d->d_c, d->d_h, d->n_h, st);
  return cuda_check("absorb W_UV into W_O (CUDA cores)");
}

template <typename T>
mla_status simt_absorb_merge(const mla_dims *d, const void *W_UQ, const void *W_UK, void *W_UQK, cudaStream_t st) {
  // W_UQK[h d_c + j][c] = sum_i W_UK[h d_h + i][j] W_UQ[h d_h + i][c]
  launch_head_product<T>(W_UK, static_cast<int64_t>(d->d_h) * d->d_c, d->d_c, 1, W_UQ,
                         static_cast<int64_t>(d->d_h) * d->d_cq, d->d_cq, 1, W_UQK,
                         static_cast<int64_t>(d->d_c) * d->d_cq, d->d_cq, 1, d->d_c, d->d_cq, d->d_h, d->n_h, st);
  return cuda_check("merged absorption matrix (CUDA cores)");
}

template <typename T>
mla_status simt_absorb_q_merged(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQK,
                                const void *W_QR, const int32_t *positions, int Tn, void *q, void *ws,
                                cudaStream_t st) {
  const int64_t HR = static_cast<int64_t>(d->n_h) * d->d_r;
  const int64_t HC = static_cast<int64_t>(d->n_h) * d->d_c;
  float *cq = static_cast<float *>(ws);             // [T][d_cq]
  float *qr = cq + static_cast<int64_t>(Tn) * d->d_cq;  // [T][n_h*d_r]
  float *ql = qr + Tn * HR;                         // [T][n_h][d_c]
  launch_linear<T>(static_cast<const T *>(W_DQ), 0, d->d, 1, h, false, 0, d->d, cq, 0, d->d_cq, d->d_cq, d->d, Tn, 1,
                   st);
  launch_linear<T>(static_cast<const T *>(W_QR), 0, d->d_cq, 1, cq, true, 0, d->d_cq, qr, 0, HR, static_cast<int>(HR),
                   d->d_cq, Tn, 1, st);
  // q_lat,h[j] = sum_c W_UQK[h d_c + j][c] c_Q[c]: batch = head
  launch_linear<T>(static_cast<const T *>(W_UQK), static_cast<int64_t>(d->d_c) * d->d_cq, d->d_cq, 1, cq, true, 0,
                   d->d_cq, ql, d->d_c, HC, d->d_c, d->d_cq, Tn, d->n_h, st);
  MLA_LAUNCH(mla::k_simt_q_store<T><<<Tn * d->n_h, 128, 0, st>>>(ql, qr, d->n_h, d->d_c, d->d_r, d->rope_base,
                                                                    positions, static_cast<T *>(q)));
  return cuda_check("merged absorb (CUDA cores)");
}

size_t simt_absorb_merged_ws(const mla_dims *d, int Tn) {
  return sizeof(float) * static_cast<size_t>(Tn) * (d->d_cq + static_cast<size_t>(d->n_h) * (d->d_r + d->d_c));
}

template <typename T>
mla_status simt_o_proj_latent(const mla_dims *d, const void *o_lat, const void *W_OV, int Tn, void *y, void *ws,
                              cudaStream_t st) {
  // y[t][r] = sum_k W_OV[r][k] o_lat[t][k], k < n_h d_c
  const int64_t HC = static_cast<int64_t>(d->n_h) * d->d_c;
  float *acc = static_cast<float *>(ws);  // [T][d]
  launch_linear<T>(static_cast<const T *>(W_OV), 0, HC, 1, o_lat, false, 0, HC, acc, 0, d->d, d->d,
                   static_cast<int>(HC), Tn, 1, st);
  const int64_t n = static_cast<int64_t>(Tn) * d->d;
  const int64_t blocks = (n + 255) / 256;
  MLA_LAUNCH(mla::k_simt_store<T><<<static_cast<int>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(acc, static_cast<T *>(y), n));
  return cuda_check("o_proj (absorbed, CUDA cores)");
}


template <typename T>
mla_status simt_query_heads(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQ, const void *W_QR,
                            const int32_t *positions, int Tn, void *qa, void *ws, cudaStream_t st) {
  const int64_t HD = static_cast<int64_t>(d->n_h) * d->d_h;
  const int64_t HR = static_cast<int64_t>(d->n_h) * d->d_r;
  float *cq = static_cast<float *>(ws);                  // [T][d_cq]
  float *qc = cq + static_cast<int64_t>(Tn) * d->d_cq;  // [T][n_h][d_h]
  float *qr = qc + Tn * HD;                              // [T][n_h][d_r]
  launch_linear<T>(static_cast<const T *>(W_DQ), 0, d->d, 1, h, false, 0, d->d, cq, 0, d->d_cq, d->d_cq, d->d, Tn, 1,
                   st);
  launch_linear<T>(static_cast<const T *>(W_UQ), 0, d->d_cq, 1, cq, true, 0, d->d_cq, qc, 0, HD, static_cast<int>(HD),
                   d->d_cq, Tn, 1, st);
  launch_linear<T>(static_cast<const T *>(W_QR), 0, d->d_cq, 1, cq, true, 0, d->d_cq, qr, 0, HR, static_cast<int>(HR),
                   d->d_cq, Tn, 1, st);
  // qa[t][h] = [q_C (d_h) | RoPE(q_R) (d_r)]: the q store with d_h in place of d_c
  MLA_LAUNCH(mla::k_simt_q_store<T><<<Tn * d->n_h, 128, 0, st>>>(qc, qr, d->n_h, d->d_h, d->d_r, d->rope_base,
                                                                    positions, static_cast<T *>(qa)));
  return cuda_check("query heads (CUDA cores)");
}

size_t simt_query_heads_ws(const mla_dims *d, int Tn) {
  return sizeof(float) * static_cast<size_t>(Tn) * (d->d_cq + static_cast<size_t>(d->n_h) * (d->d_h + d->d_r));
}

template <typename T>
mla_status simt_attend_a(const mla_dims *d, const void *qa, const void *W_UK, const void *W_UV, const mla_cache *c,
                         const int32_t *seq_lens, int B, int n_q, void *o, cudaStream_t st) {
  const int rows = B * n_q * d->n_h;
  MLA_LAUNCH(mla::k_simt_attend_a<T><<<rows, 128, 2 * 128 * sizeof(float), st>>>(
      static_cast<const T *>(qa), static_cast<const T *>(W_UK), static_cast<const T *>(W_UV), view_of(c), seq_lens,
      n_q, d->n_h, d->d_h, d->d_c, d->d_r, softmax_scale(d), static_cast<T *>(o)));
  return cuda_check("order-A attention (CUDA cores)");
}

// ------------------------------------------------------------- TMA maps --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void *ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// bf16 tensor map of rank 2..4 with 128-byte swizzle: dims[0] is the
// contiguous dimension, strides[i] is the byte stride of dims[i + 1]. Encoded
// maps are kept in a small per-thread cache keyed by all of their arguments.
struct TmapKey {
  const void *base;
  int rank;
  uint64_t dims[4], strides[3];
  uint32_t box[4];
  bool operator==(const TmapKey &o) const {
    if (base != o.base || rank != o.rank) return false;
    for (int i = 0; i < rank; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i] || (i + 1 < rank && strides[i] != o.strides[i])) return false;
    return true;
  }
};

mla_status make_tmap_nd(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const uint64_t *strides,
                        const uint32_t *box, const char *what) {
  constexpr int CAP = 64;
  thread_local TmapKey keys[CAP];
  thread_local CUtensorMap maps[CAP];
  thread_local int used = 0, next = 0;
  TmapKey key{};
  key.base = base;
  key.rank = rank;
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides[i];
  }
  for (int i = 0; i < used; ++i)
    if (keys[i] == key) {
      *m = maps[i];
      return MLA_OK;
    }
  auto fn = encode_fn();
  if (fn == nullptr) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t d[4], st[3];
  cuuint32_t bx[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    if (i + 1 < rank) st[i] = strides[i];
  }
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d, st,
                  bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "tensor map for %s: CUresult %d", what, static_cast<int>(r));
  keys[next] = key;
  maps[next] = *m;
  next = (next + 1) % CAP;
  if (used < CAP) ++used;
  return MLA_OK;
}

// 2-D map over a row-major [outer][inner] array with row pitch `pitch_bytes`.
mla_status make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint64_t pitch_bytes,
                          uint32_t box_inner, uint32_t box_outer, const char *what) {
  const uint64_t dims[2] = {inner, outer}, strides[1] = {pitch_bytes};
  const uint32_t box[2] = {box_inner, box_outer};
  return make_tmap_nd(m, base, 2, dims, strides, box, what);
}

// ------------------------------------------------ tensor-core projections --

namespace G = mla::gemm;

struct GemmShape {
  int m_total, m_tiles, n_tile, n_tiles, k_blocks, splits, batches;
};

// split_k = false: one CTA per output tile, epilogue fused into the GEMM.
GemmShape gemm_shape(int m_total, int T, int K, int batches, bool split_k) {
  GemmShape g;
  g.m_total = m_total;
  g.m_tiles = (m_total + G::BM - 1) / G::BM;
  g.n_tile = G::n_tile_for(T);
  g.n_tiles = (T + g.n_tile - 1) / g.n_tile;
  g.k_blocks = K / G::BK;
  g.batches = batches;
  g.splits = split_k ? G::choose_splits(g.m_tiles * g.n_tiles * batches, g.k_blocks, sm_count()) : 1;
  return g;
}

size_t gemm_part_bytes(const GemmShape &g, int T) {
  return sizeof(float) * static_cast<size_t>(g.batches) * g.splits * T * g.m_total;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Operands of one GEMM launch: up to three A maps stacked along m (rows
// [0, m_split) from a, [m_split, m_split2) from a2, the rest from a3), the B
// map, their majors and per-batch offsets.
struct GemmOperands {
  const CUtensorMap *a, *a2, *a3, *b;
  int m_split, m_split2;
  bool a_mn_major, b_mn_major;
  int a_batch_rows, b_batch_cols;
};

GemmOperands operands(const CUtensorMap &a, const CUtensorMap &b) {
  return GemmOperands{&a, &a, &a, &b, 1 << 30, 1 << 30, false, false, 0, 0};
}

mla_status launch_gemm(const GemmOperands &o, const GemmShape &g, int T, G::Params p, cudaStream_t st) {
  const int m_split = o.m_split;
  const bool a_mn_major = o.a_mn_major;
  const int a_batch_rows = o.a_batch_rows, b_batch_cols = o.b_batch_cols;
  p.m_total = g.m_total;
  p.m_split = m_split;
  p.m_split2 = o.m_split2;
  p.b_mn_major = o.b_mn_major ? 1 : 0;
  p.n_total = T;
  p.n_tile = g.n_tile;
  p.k_total = g.k_blocks * G::BK;
  p.k_blocks_per_split = (g.k_blocks + g.splits - 1) / g.splits;
  p.splits = g.splits;
  p.a_mn_major = a_mn_major ? 1 : 0;
  p.a_batch_rows = a_batch_rows;
  p.b_batch_cols = b_batch_cols;
  p.stages = G::stages_for(g.n_tile, g.m_tiles * g.n_tiles * g.batches * g.splits, sm_count());
  p.prefetch = g_overlap.load(std::memory_order_relaxed);  // the kernel is correct either way
  const size_t smem = G::smem_for(g.n_tile, p.stages);
  mla_status s = raise_smem_limit(reinterpret_cast<const void *>(G::k_gemm), SMEM_GEMM, 232448,
                                  "gemm: set shared memory size");
  if (s != MLA_OK) return s;
  dim3 grid(g.m_tiles, g.n_tiles, g.batches * g.splits);
  return launched(launch_tc(G::k_gemm, grid, dim3(G::NUM_THREADS), smem, st, *o.a, *o.a2, *o.a3, *o.b, p),
                  "projection GEMM (tensor cores)");
}

GemmShape append_shape(const mla_dims *d, int T) { return gemm_shape(d->d_c + d->d_r, T, d->d, 1, true); }

size_t tc_append_ws(const mla_dims *d, int T) { return gemm_part_bytes(append_shape(d, T), T); }

mla_status tc_append(const mla_dims *d, const void *h, const void *W_DKV, const void *W_KR, const int32_t *seq_idx,
                     const int32_t *positions, int T, const mla_cache *c, void *ws, cudaStream_t st) {
  const GemmShape g = append_shape(d, T);
  CUtensorMap ta, ta2, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_DKV, d->d, d->d_c, d->d * 2ull, 64, 128, "W_DKV")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&ta2, W_KR, d->d, d->d_r, d->d * 2ull, 64, 128, "W_KR")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, h, d->d, T, d->d * 2ull, 64, g.n_tile, "h")) != MLA_OK) return s;
  float *part = static_cast<float *>(ws);
  G::Params p{};
  p.epi = G::EPI_PARTIAL;
  p.out = part;
  GemmOperands op = operands(ta, tb);
  op.a2 = &ta2;
  op.m_split = d->d_c;
  if ((s = launch_gemm(op, g, T, p, st)) != MLA_OK) return s;
  const int D = d->d_c + d->d_r;
  return launched(launch_tc(G::k_fin_append, dim3((D / 2 + 127) / 128, T), dim3(128), 0, st, part, g.splits, T,
                            d->d_c, d->d_r, d->rope_base, seq_idx, positions, view_of(c)),
                  "append finalize");
}

struct AbsorbPlan {
  GemmShape cq, uq, uk;
  size_t cq_off, qc_off, total;
};

AbsorbPlan absorb_plan(const mla_dims *d, int T) {
  AbsorbPlan a;
  a.cq = gemm_shape(d->d_cq, T, d->d, 1, true);
  a.uq = gemm_shape(d->n_h * (d->d_h + d->d_r), T, d->d_cq, 1, false);
  a.uk = gemm_shape(d->d_c, T, d->d_h, d->n_h, false);
  a.cq_off = align256(gemm_part_bytes(a.cq, T));
  a.qc_off = a.cq_off + align256(static_cast<size_t>(T) * d->d_cq * 2);
  a.total = a.qc_off + static_cast<size_t>(T) * d->n_h * d->d_h * 2;
  return a;
}

size_t tc_absorb_ws(const mla_dims *d, int T) { return absorb_plan(d, T).total; }

// q = [W_UK_h^T W_UQ_h c_Q | RoPE(W_QR_h c_Q)] from a c_Q already stored (bf16
// [T][d_cq]): one CTA per head with q_C in shared memory (T <= 128), or
// [W_UQ; W_QR] then W_UK^T with q_C in the workspace (qc, T * n_h * d_h bf16).
mla_status tc_absorb_from_cq(const mla_dims *d, const __nv_bfloat16 *cq, const void *W_UQ, const void *W_QR,
                             const void *W_UK, const int32_t *positions, int T, void *q, __nv_bfloat16 *qc,
                             cudaStream_t st) {
  const AbsorbPlan a = absorb_plan(d, T);
  const int HD = d->n_h * d->d_h;
  const int64_t Dq = d->d_c + d->d_r;
  CUtensorMap ta, ta2, tb;
  mla_status s;
  if (a.uq.n_tile <= 128) {
    // one CTA per head: q_C,h = W_UQ_h c_Q, q_R,h = RoPE(W_QR_h c_Q), q_lat,h = W_UK_h^T q_C,h
    CUtensorMap tq, tr, tc, tk;
    if ((s = make_tmap_bf16(&tq, W_UQ, d->d_cq, HD, d->d_cq * 2ull, 64, 128, "W_UQ")) != MLA_OK) return s;
    if ((s = make_tmap_bf16(&tr, W_QR, d->d_cq, d->n_h * d->d_r, d->d_cq * 2ull, 64, 64, "W_QR")) != MLA_OK) return s;
    if ((s = make_tmap_bf16(&tc, cq, d->d_cq, T, d->d_cq * 2ull, 64, a.uq.n_tile, "c_Q")) != MLA_OK) return s;
    if ((s = make_tmap_bf16(&tk, W_UK, d->d_c, HD, d->d_c * 2ull, 64, 64, "W_UK")) != MLA_OK) return s;
    G::ab::Params ap{};
    ap.T = T;
    ap.n_tile = a.uq.n_tile;
    ap.n_h = d->n_h;
    ap.d_c = d->d_c;
    ap.d_r = d->d_r;
    ap.k_blocks = d->d_cq / G::BK;
    ap.stages = G::ab::stages(ap.n_tile);
    ap.stage_bytes = G::ab::stage_bytes(ap.n_tile);
    ap.col_stride = (ap.n_tile + 31) / 32 * 32;
    ap.q = static_cast<__nv_bfloat16 *>(q);
    ap.positions = positions;
    ap.rope_base = d->rope_base;
    ap.prefetch = g_overlap.load(std::memory_order_relaxed);  // the kernel is correct either way
    const size_t smem = G::ab::smem(ap.n_tile, ap.stages);
    if ((s = raise_smem_limit(reinterpret_cast<const void *>(G::k_absorb_head), SMEM_ABSORB, 232448,
                              "absorb: set shared memory size")) != MLA_OK)
      return s;
    return launched(launch_tc(G::k_absorb_head, dim3(d->n_h), dim3(G::ab::NUM_THREADS), smem, st, tq, tr, tc, tk, ap),
                    "fused per-head absorb (tensor cores)");
  }
  // [q_C ; q_R] = [W_UQ ; W_QR] c_Q: q_C to the workspace, q_R rotated into q
  if ((s = make_tmap_bf16(&ta, W_UQ, d->d_cq, HD, d->d_cq * 2ull, 64, 128, "W_UQ")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&ta2, W_QR, d->d_cq, d->n_h * d->d_r, d->d_cq * 2ull, 64, 128, "W_QR")) != MLA_OK)
    return s;
  if ((s = make_tmap_bf16(&tb, cq, d->d_cq, T, d->d_cq * 2ull, 64, a.uq.n_tile, "c_Q")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_UQ;
  p.dst = qc;
  p.e_split = HD;
  p.q = static_cast<__nv_bfloat16 *>(q);
  p.n_h = d->n_h;
  p.d_c = d->d_c;
  p.d_r = d->d_r;
  p.rope_base = d->rope_base;
  p.positions = positions;
  GemmOperands op = operands(ta, tb);
  op.a2 = &ta2;
  op.m_split = HD;
  if ((s = launch_gemm(op, a.uq, T, p, st)) != MLA_OK) return s;
  // q_lat,h = W_UK_h^T q_C,h: A(m = latent j, k = i) = W_UK[h*d_h + i][j], m contiguous
  if ((s = make_tmap_bf16(&ta, W_UK, d->d_c, HD, d->d_c * 2ull, 64, 64, "W_UK")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, qc, HD, T, HD * 2ull, 64, a.uk.n_tile, "q_C")) != MLA_OK) return s;
  p = G::Params{};
  p.epi = G::EPI_BF16;
  p.dst = static_cast<__nv_bfloat16 *>(q);
  p.e_bs = Dq;
  p.e_ns = d->n_h * Dq;
  op = operands(ta, tb);
  op.a_mn_major = true;
  op.a_batch_rows = d->d_h;
  op.b_batch_cols = d->d_h;
  return launch_gemm(op, a.uk, T, p, st);
}

// c_Q = W_DQ h (split K, fp32 partials, then rounded to bf16 in the workspace).
mla_status tc_query_latent(const mla_dims *d, const void *h, const void *W_DQ, int T, void *ws, size_t cq_off,
                           cudaStream_t st) {
  const GemmShape g = gemm_shape(d->d_cq, T, d->d, 1, true);
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_DQ, d->d, d->d_cq, d->d * 2ull, 64, 128, "W_DQ")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, h, d->d, T, d->d * 2ull, 64, g.n_tile, "h")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_PARTIAL;
  p.out = static_cast<float *>(ws);
  if ((s = launch_gemm(operands(ta, tb), g, T, p, st)) != MLA_OK) return s;
  __nv_bfloat16 *cq = reinterpret_cast<__nv_bfloat16 *>(static_cast<uint8_t *>(ws) + cq_off);
  const int64_t pairs = static_cast<int64_t>(T) * d->d_cq / 2;
  return launched(launch_tc(G::k_fin_store, dim3(static_cast<int>(std::min<int64_t>(1024, (pairs + 255) / 256))),
                            dim3(256), 0, st, static_cast<float *>(ws), g.splits, T, d->d_cq, cq,
                            static_cast<int64_t>(d->d_cq)),
                  "c_Q finalize");
}

mla_status tc_absorb(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQ, const void *W_QR,
                     const void *W_UK, const int32_t *positions, int T, void *q, void *ws, cudaStream_t st) {
  const AbsorbPlan a = absorb_plan(d, T);
  mla_status s = tc_query_latent(d, h, W_DQ, T, ws, a.cq_off, st);
  if (s != MLA_OK) return s;
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  return tc_absorb_from_cq(d, reinterpret_cast<__nv_bfloat16 *>(w8 + a.cq_off), W_UQ, W_QR, W_UK, positions, T, q,
                           reinterpret_cast<__nv_bfloat16 *>(w8 + a.qc_off), st);
}

// ---- fused front end: one weight-streaming GEMM over [W_DKV; W_KR; W_DQ] ----
// Rows of the stacked product: [0, d_c) W_DKV, [d_c, d_c + kr_tiles * 128)
// W_KR (d_r valid rows, the rest of its tiles zero-filled), then W_DQ.
struct FrontPlan {
  GemmShape g;
  int kr_rows, cq_row;
  size_t cq_off, qc_off, total;
};

FrontPlan front_plan(const mla_dims *d, int T) {
  FrontPlan f;
  f.kr_rows = (d->d_r + G::BM - 1) / G::BM * G::BM;
  f.cq_row = d->d_c + f.kr_rows;
  f.g = gemm_shape(f.cq_row + d->d_cq, T, d->d, 1, true);
  f.cq_off = align256(gemm_part_bytes(f.g, T));
  f.qc_off = f.cq_off + align256(static_cast<size_t>(T) * d->d_cq * 2);
  f.total = f.qc_off + static_cast<size_t>(T) * d->n_h * d->d_h * 2;
  return f;
}

size_t tc_front_ws(const mla_dims *d, int T) { return front_plan(d, T).total; }

mla_status tc_front_end(const mla_dims *d, const void *h, const void *W_DKV, const void *W_KR, const void *W_DQ,
                        const void *W_UQ, const void *W_QR, const void *W_UK, const int32_t *seq_idx,
                        const int32_t *positions, int T, const mla_cache *c, void *q, void *ws, cudaStream_t st) {
  const FrontPlan f = front_plan(d, T);
  CUtensorMap ta, ta2, ta3, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_DKV, d->d, d->d_c, d->d * 2ull, 64, 128, "W_DKV")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&ta2, W_KR, d->d, d->d_r, d->d * 2ull, 64, 128, "W_KR")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&ta3, W_DQ, d->d, d->d_cq, d->d * 2ull, 64, 128, "W_DQ")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, h, d->d, T, d->d * 2ull, 64, f.g.n_tile, "h")) != MLA_OK) return s;
  float *part = static_cast<float *>(ws);
  G::Params p{};
  p.epi = G::EPI_PARTIAL;
  p.out = part;
  GemmOperands op = operands(ta, tb);
  op.a2 = &ta2;
  op.a3 = &ta3;
  op.m_split = d->d_c;
  op.m_split2 = f.cq_row;
  if ((s = launch_gemm(op, f.g, T, p, st)) != MLA_OK) return s;
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  __nv_bfloat16 *cq = reinterpret_cast<__nv_bfloat16 *>(w8 + f.cq_off);
  const int pairs = (d->d_c + d->d_r + d->d_cq) / 2;
  if ((s = launched(launch_tc(G::k_fin_front, dim3((pairs + 127) / 128, T), dim3(128), 0, st, part, f.g.splits, T,
                              f.g.m_total, d->d_c, d->d_r, f.cq_row, d->d_cq, d->rope_base, seq_idx, positions,
                              view_of(c), cq),
                    "front-end finalize")) != MLA_OK)
    return s;
  return tc_absorb_from_cq(d, cq, W_UQ, W_QR, W_UK, positions, T, q,
                           reinterpret_cast<__nv_bfloat16 *>(w8 + f.qc_off), st);
}

// ---- merged-matrix absorption: W_UQK_h = W_UK_h^T W_UQ_h (d_c x d_cq per head) ----
mla_status tc_absorb_merge(const mla_dims *d, const void *W_UQ, const void *W_UK, void *W_UQK, cudaStream_t st) {
  // D(m = c, n = j) = sum_i W_UQ[h d_h + i][c] W_UK[h d_h + i][j]: both operands MN-major
  const GemmShape g = gemm_shape(d->d_cq, d->d_c, d->d_h, d->n_h, false);
  const int HD = d->n_h * d->d_h;
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_UQ, d->d_cq, HD, d->d_cq * 2ull, 64, 64, "W_UQ")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, W_UK, d->d_c, HD, d->d_c * 2ull, 64, 64, "W_UK")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_BF16;
  p.dst = static_cast<__nv_bfloat16 *>(W_UQK);
  p.e_bs = static_cast<int64_t>(d->d_c) * d->d_cq;  // head h: rows h d_c ..
  p.e_ns = d->d_cq;                                  // row j, column c = m
  GemmOperands op = operands(ta, tb);
  op.a_mn_major = true;
  op.b_mn_major = true;
  op.a_batch_rows = d->d_h;
  op.b_batch_cols = d->d_h;
  return launch_gemm(op, g, d->d_c, p, st);
}

size_t tc_absorb_merged_ws(const mla_dims *d, int T) {
  const GemmShape cq = gemm_shape(d->d_cq, T, d->d, 1, true);
  return align256(gemm_part_bytes(cq, T)) + static_cast<size_t>(T) * d->d_cq * 2;
}

mla_status tc_absorb_q_merged(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQK, const void *W_QR,
                              const int32_t *positions, int T, void *q, void *ws, cudaStream_t st) {
  const size_t cq_off = align256(gemm_part_bytes(gemm_shape(d->d_cq, T, d->d, 1, true), T));
  mla_status s = tc_query_latent(d, h, W_DQ, T, ws, cq_off, st);
  if (s != MLA_OK) return s;
  const __nv_bfloat16 *cq = reinterpret_cast<const __nv_bfloat16 *>(static_cast<uint8_t *>(ws) + cq_off);
  const int64_t Dq = d->d_c + d->d_r;
  CUtensorMap ta, tb;
  // q_lat,h = W_UQK_h c_Q: batch = head, A rows h d_c .., bf16 into q[t][h][0 .. d_c)
  const GemmShape gl = gemm_shape(d->d_c, T, d->d_cq, d->n_h, false);
  if ((s = make_tmap_bf16(&ta, W_UQK, d->d_cq, static_cast<uint64_t>(d->n_h) * d->d_c, d->d_cq * 2ull, 64, 128,
                          "W_UQK")) != MLA_OK)
    return s;
  if ((s = make_tmap_bf16(&tb, cq, d->d_cq, T, d->d_cq * 2ull, 64, gl.n_tile, "c_Q")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_BF16;
  p.dst = static_cast<__nv_bfloat16 *>(q);
  p.e_bs = Dq;
  p.e_ns = d->n_h * Dq;
  GemmOperands op = operands(ta, tb);
  op.a_batch_rows = d->d_c;
  if ((s = launch_gemm(op, gl, T, p, st)) != MLA_OK) return s;
  // q_R = RoPE(W_QR c_Q): every row of this product is a q_R row
  const GemmShape gr = gemm_shape(d->n_h * d->d_r, T, d->d_cq, 1, false);
  if ((s = make_tmap_bf16(&ta, W_QR, d->d_cq, d->n_h * d->d_r, d->d_cq * 2ull, 64, 128, "W_QR")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, cq, d->d_cq, T, d->d_cq * 2ull, 64, gr.n_tile, "c_Q")) != MLA_OK) return s;
  p = G::Params{};
  p.epi = G::EPI_UQ;
  p.e_split = 0;
  p.q = static_cast<__nv_bfloat16 *>(q);
  p.n_h = d->n_h;
  p.d_c = d->d_c;
  p.d_r = d->d_r;
  p.rope_base = d->rope_base;
  p.positions = positions;
  return launch_gemm(operands(ta, tb), gr, T, p, st);
}

// ---- W_UV absorbed into the output projection ----
mla_status tc_absorb_wo(const mla_dims *d, const void *W_O, const void *W_UV, void *W_OV, cudaStream_t st) {
  // D(m = j, n = r) = sum_i W_UV[h d_h + i][j] W_O[r][h d_h + i]; W_OV[r][h d_c + j]
  const GemmShape g = gemm_shape(d->d_c, d->d, d->d_h, d->n_h, false);
  const int HD = d->n_h * d->d_h;
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_UV, d->d_c, HD, d->d_c * 2ull, 64, 64, "W_UV")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, W_O, HD, d->d, HD * 2ull, 64, g.n_tile, "W_O")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_BF16;
  p.dst = static_cast<__nv_bfloat16 *>(W_OV);
  p.e_bs = d->d_c;
  p.e_ns = static_cast<int64_t>(d->n_h) * d->d_c;
  GemmOperands op = operands(ta, tb);
  op.a_mn_major = true;
  op.a_batch_rows = d->d_h;
  op.b_batch_cols = d->d_h;
  return launch_gemm(op, g, d->d, p, st);
}

GemmShape o_proj_latent_shape(const mla_dims *d, int T) { return gemm_shape(d->d, T, d->n_h * d->d_c, 1, true); }

size_t tc_o_proj_latent_ws(const mla_dims *d, int T) { return gemm_part_bytes(o_proj_latent_shape(d, T), T); }

mla_status tc_o_proj_latent(const mla_dims *d, const void *o_lat, const void *W_OV, int T, void *y, void *ws,
                            cudaStream_t st) {
  const GemmShape g = o_proj_latent_shape(d, T);
  const int HC = d->n_h * d->d_c;
  float *part = static_cast<float *>(ws);
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_OV, HC, d->d, HC * 2ull, 64, 128, "W_OV")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, o_lat, HC, T, HC * 2ull, 64, g.n_tile, "o_lat")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_PARTIAL;
  p.out = part;
  if ((s = launch_gemm(operands(ta, tb), g, T, p, st)) != MLA_OK) return s;
  const int64_t pairs = static_cast<int64_t>(T) * d->d / 2;
  return launched(launch_tc(G::k_fin_store, dim3(static_cast<int>(std::min<int64_t>(1024, (pairs + 255) / 256))),
                            dim3(256), 0, st, part, g.splits, T, d->d, static_cast<__nv_bfloat16 *>(y),
                            static_cast<int64_t>(d->d)),
                  "o_proj (absorbed) finalize");
}

// ---- order A: query heads without absorption, decompression, 192-d attention ----
size_t tc_query_heads_ws(const mla_dims *d, int T) {
  const GemmShape cq = gemm_shape(d->d_cq, T, d->d, 1, true);
  return align256(gemm_part_bytes(cq, T)) + static_cast<size_t>(T) * d->d_cq * 2;
}

mla_status tc_query_heads(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQ, const void *W_QR,
                          const int32_t *positions, int T, void *qa, void *ws, cudaStream_t st) {
  const size_t cq_off = align256(gemm_part_bytes(gemm_shape(d->d_cq, T, d->d, 1, true), T));
  mla_status s = tc_query_latent(d, h, W_DQ, T, ws, cq_off, st);
  if (s != MLA_OK) return s;
  const __nv_bfloat16 *cq = reinterpret_cast<const __nv_bfloat16 *>(static_cast<uint8_t *>(ws) + cq_off);
  const int HD = d->n_h * d->d_h;
  // [q_C ; q_R] = [W_UQ ; W_QR] c_Q: q_C,h into qa[t][h][0, d_h), q_R,h rotated into qa[t][h][d_h, d_h + d_r)
  const GemmShape g = gemm_shape(d->n_h * (d->d_h + d->d_r), T, d->d_cq, 1, false);
  CUtensorMap ta, ta2, tb;
  if ((s = make_tmap_bf16(&ta, W_UQ, d->d_cq, HD, d->d_cq * 2ull, 64, 128, "W_UQ")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&ta2, W_QR, d->d_cq, d->n_h * d->d_r, d->d_cq * 2ull, 64, 128, "W_QR")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, cq, d->d_cq, T, d->d_cq * 2ull, 64, g.n_tile, "c_Q")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_QA;
  p.e_split = HD;
  p.q = static_cast<__nv_bfloat16 *>(qa);
  p.n_h = d->n_h;
  p.d_c = d->d_h;  // the q_C width of a qa row; q_R follows it
  p.d_r = d->d_r;
  p.rope_base = d->rope_base;
  p.positions = positions;
  GemmOperands op = operands(ta, tb);
  op.a2 = &ta2;
  op.m_split = HD;
  return launch_gemm(op, g, T, p, st);
}

int64_t cache_rows_of(const mla_cache *c) {
  return c->paged ? c->num_blocks * c->block_size : static_cast<int64_t>(c->num_seqs) * c->max_len;
}

// decompressed K_C and V: [n_h][rows][d_h] bf16 each
size_t tc_attend_a_ws(const mla_dims *d, int64_t rows) {
  return 2 * align256(static_cast<size_t>(d->n_h) * rows * d->d_h * 2);
}

mla_status tc_attend_a(const mla_dims *d, const void *qa, const void *W_UK, const void *W_UV, const mla_cache *c,
                       const int32_t *seq_lens, int B, int n_q, void *o, void *ws, cudaStream_t st) {
  namespace P = mla::pre;
  const int64_t R = cache_rows_of(c);
  if (c->paged && c->block_size % P::BLK != 0)
    return fail(MLA_ERR_UNSUPPORTED, "order-A attention needs block_size to be a multiple of %d", P::BLK);
  if (R >= 0x7fff0000LL || (R + 255) / 256 > 65535)
    return fail(MLA_ERR_UNSUPPORTED, "order-A attention: too many cache rows");
  const int HD = d->n_h * d->d_h;
  const int64_t D = d->d_c + d->d_r;
  uint8_t *w8 = static_cast<uint8_t *>(ws);
  __nv_bfloat16 *kc = reinterpret_cast<__nv_bfloat16 *>(w8);
  __nv_bfloat16 *vv = reinterpret_cast<__nv_bfloat16 *>(w8 + align256(static_cast<size_t>(d->n_h) * R * d->d_h * 2));
  mla_status s;
  // decompression over every physical cache row, K_C and V in one launch:
  // X_h[r][i] = sum_j W[h d_h + i][j] c_KV[r][j] for W = W_UK, W_UV
  __nv_bfloat16 *dsts[2] = {kc, vv};
  {
    CUtensorMap ta0, ta1, tx;
    if ((s = make_tmap_bf16(&tx, c->data, d->d_c, R, D * 2, 64, G::rs::NHALF, "cache (c_KV)")) != MLA_OK) return s;
    if ((s = make_tmap_bf16(&ta0, W_UK, d->d_c, HD, d->d_c * 2ull, 64, 128, "W_UK")) != MLA_OK) return s;
    if ((s = make_tmap_bf16(&ta1, W_UV, d->d_c, HD, d->d_c * 2ull, 64, 128, "W_UV")) != MLA_OK) return s;
    G::rs::Params rp{};
    rp.batches = 2 * d->n_h;
    rp.split = d->n_h;
    rp.n_tiles = static_cast<int>((R + G::rs::NT - 1) / G::rs::NT);
    rp.N = static_cast<int>(R);
    rp.kblk = d->d_c / G::BK;
    rp.out0 = kc;
    rp.out1 = vv;
    const int grid = 2 * std::max(1, std::min(sm_count() / 2, (rp.batches / 2) * rp.n_tiles));  // clusters of 2
    if ((s = raise_smem_limit(reinterpret_cast<const void *>(G::k_gemm_resident), SMEM_GEMM_RES, G::rs::SMEM_BYTES,
                              "decompression: set shared memory size")) != MLA_OK)
      return s;
    if ((s = launched(launch_tc(G::k_gemm_resident, dim3(grid), dim3(G::rs::NUM_THREADS), G::rs::SMEM_BYTES, st, ta0,
                                ta1, tx, rp),
                      "order-A decompression (tensor cores)")) != MLA_OK)
      return s;
  }
  // attention
  const int T = B * n_q;
  CUtensorMap tm_q, tm_kc, tm_kr, tm_v;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(P::DQK), static_cast<uint64_t>(d->n_h), static_cast<uint64_t>(T)};
    const uint64_t str[2] = {P::DQK * 2ull, static_cast<uint64_t>(d->n_h) * P::DQK * 2};
    const uint32_t box[3] = {64, 1, P::QROWS};
    if ((s = make_tmap_nd(&tm_q, qa, 3, dims, str, box, "qa")) != MLA_OK) return s;
  }
  for (int u = 0; u < 2; ++u) {
    const uint64_t dims[3] = {static_cast<uint64_t>(d->d_h), static_cast<uint64_t>(R), static_cast<uint64_t>(d->n_h)};
    const uint64_t str[2] = {d->d_h * 2ull, static_cast<uint64_t>(R) * d->d_h * 2};
    const uint32_t box[3] = {64, P::BLK, 1};
    if ((s = make_tmap_nd(u == 0 ? &tm_kc : &tm_v, dsts[u], 3, dims, str, box, u == 0 ? "K_C" : "V")) != MLA_OK)
      return s;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(R)}, str[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {64, P::BLK};
    if ((s = make_tmap_nd(&tm_kr, c->data, 2, dims, str, box, "cache (k_R)")) != MLA_OK) return s;
  }
  P::Params pp{};
  pp.seq_lens = seq_lens;
  pp.block_table = c->block_table;
  pp.max_len = c->max_len;
  pp.rows = R;
  pp.paged = c->paged;
  pp.block_size = c->block_size;
  pp.max_blocks_per_seq = c->max_blocks_per_seq;
  pp.num_blocks_i32 = static_cast<int32_t>(c->paged ? c->num_blocks : 0);
  pp.B = B;
  pp.n_q = n_q;
  pp.n_h = d->n_h;
  pp.qblocks = (n_q + P::QROWS - 1) / P::QROWS;
  pp.capacity = cache_capacity(c);
  pp.scale_log2 = softmax_scale(d) * 1.4426950408889634f;
  pp.o = static_cast<__nv_bfloat16 *>(o);
  if ((s = raise_smem_limit(reinterpret_cast<const void *>(P::k_attend_a), SMEM_ATTEND_A, P::SMEM_BYTES,
                            "order-A attention: set shared memory size")) != MLA_OK)
    return s;
  return launched(launch_tc(P::k_attend_a, dim3(d->n_h * B * pp.qblocks), dim3(P::NUM_THREADS), P::SMEM_BYTES, st,
                            tm_q, tm_kc, tm_kr, tm_v, pp),
                  "order-A attention (tensor cores)");
}

// ---- failure-path self-test: a projection GEMM whose producer issues nothing ----
// The MMA thread's first wait runs out after wait_ns; the kernel records the
// timeout in the device error word and unwinds (no copy is in flight; tensor
// memory is freed). scratch: at least SELFTEST_BYTES of device memory.
constexpr size_t SELFTEST_BYTES = 64 * 1024;

mla_status tc_selftest_timeout(uint64_t wait_ns, void *scratch, cudaStream_t st) {
  uint8_t *s8 = static_cast<uint8_t *>(scratch);
  const GemmShape g = gemm_shape(G::BM, 16, G::BK, 1, false);  // one tile: 128 rows, 16 tokens, one K block
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, s8, G::BK, G::BM, G::BK * 2ull, 64, 128, "self-test A")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, s8 + 16384, G::BK, 16, G::BK * 2ull, 64, g.n_tile, "self-test B")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_PARTIAL;
  p.out = reinterpret_cast<float *>(s8 + 32768);
  p.wait_ns = wait_ns;
  p.idle_producer = 1;
  return launch_gemm(operands(ta, tb), g, 16, p, st);
}

GemmShape out_proj_shape(const mla_dims *d, int T) { return gemm_shape(d->d_h, T, d->d_c, d->n_h, false); }

size_t tc_out_proj_ws(const mla_dims *, int) { return 0; }

mla_status tc_out_proj(const mla_dims *d, const void *o_lat, const void *W_UV, int T, void *o, void *,
                       cudaStream_t st) {
  const GemmShape g = out_proj_shape(d, T);
  const int HD = d->n_h * d->d_h, HC = d->n_h * d->d_c;
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_UV, d->d_c, HD, d->d_c * 2ull, 64, 128, "W_UV")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, o_lat, HC, T, HC * 2ull, 64, g.n_tile, "o_lat")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_BF16;
  p.dst = static_cast<__nv_bfloat16 *>(o);
  p.e_bs = d->d_h;
  p.e_ns = HD;
  GemmOperands op = operands(ta, tb);
  op.a_batch_rows = d->d_h;
  op.b_batch_cols = d->d_c;
  return launch_gemm(op, g, T, p, st);
}

// y = W_O o: split-K over the n_h*d_h columns, fp32 partials, then summed to
// bf16 (the c_Q = W_DQ h pattern with W_O in place of W_DQ).
GemmShape o_proj_shape(const mla_dims *d, int T) { return gemm_shape(d->d, T, d->n_h * d->d_h, 1, true); }

size_t tc_o_proj_ws(const mla_dims *d, int T) { return gemm_part_bytes(o_proj_shape(d, T), T); }

mla_status tc_o_proj(const mla_dims *d, const void *o, const void *W_O, int T, void *y, void *ws, cudaStream_t st) {
  const GemmShape g = o_proj_shape(d, T);
  const int HD = d->n_h * d->d_h;
  float *part = static_cast<float *>(ws);
  CUtensorMap ta, tb;
  mla_status s;
  if ((s = make_tmap_bf16(&ta, W_O, HD, d->d, HD * 2ull, 64, 128, "W_O")) != MLA_OK) return s;
  if ((s = make_tmap_bf16(&tb, o, HD, T, HD * 2ull, 64, g.n_tile, "o")) != MLA_OK) return s;
  G::Params p{};
  p.epi = G::EPI_PARTIAL;
  p.out = part;
  if ((s = launch_gemm(operands(ta, tb), g, T, p, st)) != MLA_OK) return s;
  const int64_t pairs = static_cast<int64_t>(T) * d->d / 2;
  return launched(launch_tc(G::k_fin_store, dim3(static_cast<int>(std::min<int64_t>(1024, (pairs + 255) / 256))),
                            dim3(256), 0, st, part, g.splits, T, d->d, static_cast<__nv_bfloat16 *>(y),
                            static_cast<int64_t>(d->d)),
                  "o_proj finalize");
}

// ------------------------------------------------- tensor-core decode ----

// Clusters of two CTAs that can be resident at once (a pair must share a GPC,
// so this can be below SMs / 2). The persistent decode grid uses exactly this
// many so that no cluster waits for a second wave. Occupancy is a property of
// the device, so the count is cached per device ordinal; it never exceeds
// half of that device's SMs, which is what decode_tc_ws() sizes the split
// partials for.
constexpr int MAX_DEVICES = 64;
std::atomic<int> g_decode_clusters[MAX_DEVICES];

int decode_clusters(int sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = -1;
  }
  if (dev >= 0 && dev < MAX_DEVICES) {
    const int c = g_decode_clusters[dev].load(std::memory_order_acquire);
    if (c > 0) return std::min(c, sms / 2);
  }
  namespace D = mla::dec;
  cudaFuncSetAttribute(D::k_decode<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, D::SMEM_BYTES);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
  cfg.blockDim = dim3(D::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = D::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, D::k_decode<false>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sms / 2;
  }
  n = std::max(1, std::min(n, sms / 2));
  if (dev >= 0 && dev < MAX_DEVICES) g_decode_clusters[dev].store(n, std::memory_order_release);
  return n;
}

mla_status decode_tc(const mla_dims *d, const void *q, const mla_cache *c, const int32_t *seq_lens, int B, int n_q,
                     void *o_lat, float *lse, int num_splits, void *ws, size_t ws_bytes, cudaStream_t st) {
  namespace D = mla::dec;
  const int BJ = B * n_q;
  if (BJ > D::MAX_UNITS) return fail(MLA_ERR_UNSUPPORTED, "tensor-core decode supports B*n_q <= %d", D::MAX_UNITS);
  if (c->paged && c->block_size % D::BLK != 0)
    return fail(MLA_ERR_UNSUPPORTED, "tensor-core decode needs block_size to be a multiple of %d", D::BLK);
  const int64_t rows = c->paged ? c->num_blocks * c->block_size : static_cast<int64_t>(c->num_seqs) * c->max_len;
  if (rows >= 0x7fff0000LL) return fail(MLA_ERR_UNSUPPORTED, "cache has too many rows for 32-bit TMA coordinates");
  const int sms = sm_count();
  const int nclusters = decode_clusters(sms);
  if (ws_bytes < mla::decode_tc_ws(B, n_q, sms, num_splits, cache_capacity(c)))
    return fail(MLA_ERR_WORKSPACE, "decode workspace too small");

  // Views of q and the cache (rows of 576 bf16 = 1152 bytes):
  //   q:        (64 cols, row, 9 chunks of 128 B)        box (64, 64 heads, 3): a third of a CTA's Q
  //   score:    (576 cols, row)                          box (64, 64 tokens): one column chunk of a block
  //   value:    (64 cols, row, 2 chunks, 2 halves) at column 128 * rank, half stride 256 cols
  //             box (64, 64 tokens, 2, 1) = 128 of this CTA's latent columns of a block
  CUtensorMap tm_q, tm_k, tm_v[2];
  mla_status s;
  const uint64_t row_b = D::D * 2;
  {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(BJ) * D::HEADS, 9}, str[2] = {row_b, 128};
    const uint32_t box[3] = {64, D::HPC, 3};
    if ((s = make_tmap_nd(&tm_q, q, 3, dims, str, box, "q")) != MLA_OK) return s;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D::D), static_cast<uint64_t>(rows)}, str[1] = {row_b};
    const uint32_t box[2] = {64, D::BLK};
    if ((s = make_tmap_nd(&tm_k, c->data, 2, dims, str, box, "cache (score chunks)")) != MLA_OK) return s;
  }
  for (int r = 0; r < 2; ++r) {
    const uint64_t dims[4] = {64, static_cast<uint64_t>(rows), 2, 2}, str[3] = {row_b, 128, 512};
    const uint32_t box[4] = {64, D::BLK, 2, 1};
    const void *base = static_cast<const uint8_t *>(c->data) + 256 * r;
    if ((s = make_tmap_nd(&tm_v[r], base, 4, dims, str, box, "cache (value slabs)")) != MLA_OK) return s;
  }

  D::Params p{};
  p.seq_lens = seq_lens;
  p.block_table = c->block_table;
  p.max_len = c->max_len;
  p.cache_rows = rows;
  p.paged = c->paged;
  p.block_size = c->block_size;
  p.max_blocks_per_seq = c->max_blocks_per_seq;
  p.num_blocks_i32 = static_cast<int32_t>(c->paged ? c->num_blocks : 0);
  p.B = B;
  p.n_q = n_q;
  p.capacity = c->paged ? static_cast<int64_t>(c->max_blocks_per_seq) * c->block_size : c->max_len;
  p.scale = softmax_scale(d);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.o_lat = static_cast<__nv_bfloat16 *>(o_lat);
  p.lse = lse;
  p.splits = num_splits;
  const size_t plan_bytes = mla::decode_plan_bytes(BJ);
  const size_t slots = mla::decode_tc_slots(B, n_q, sms, num_splits, cache_capacity(c));
  p.plan = static_cast<int32_t *>(ws);
  p.part_o = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + plan_bytes);
  p.part_lse = p.part_o + slots * D::HEADS * D::DC;

  // n_q > 1: the variant whose cluster groups follow the query positions
  const auto kernel = n_q > 1 ? D::k_decode<true> : D::k_decode<false>;
  if ((s = raise_smem_limit(reinterpret_cast<const void *>(kernel), n_q > 1 ? SMEM_DECODE_NQ : SMEM_DECODE,
                            D::SMEM_BYTES, "decode: set shared memory size")) != MLA_OK)
    return s;
  if ((s = launched(launch_tc(kernel, dim3(2 * nclusters), dim3(D::NUM_THREADS), D::SMEM_BYTES, st, tm_q, tm_k, tm_v[0],
                              tm_v[1], p),
                    "decode (tensor cores)")) != MLA_OK)
    return s;
  return launched(launch_tc(D::k_combine, dim3(BJ * D::COMBINE_BLOCKS_PER_ROW), dim3(128), 0, st, p),
                  "decode combine");
}

}  // namespace

// ------------------------------------------- decode without a caller workspace
//
// mla_decode_noalloc runs the same decode as mla_decode, with its scratch in
// a static device array of this translation unit instead of a caller-provided
// workspace. The array is sized for at most NOALLOC_MAX_ROWS token rows
// (B * n_q) and NOALLOC_MAX_CLUSTERS decode clusters (one B200: 148 SMs = 74
// pairs); larger calls are rejected. Its address is looked up once per device
// with cudaGetSymbolAddress (first call on that device).
namespace {

constexpr int32_t NOALLOC_MAX_ROWS = 64;
constexpr int32_t NOALLOC_MAX_CLUSTERS = 74;
// the decode workspace layout: the plan, then fp32 partials [slots][128][512]
// and [slots][128] for slots = rows + clusters (automatic plan)
constexpr size_t NOALLOC_BYTES =
    mla::decode_plan_bytes(NOALLOC_MAX_ROWS) +
    static_cast<size_t>(NOALLOC_MAX_ROWS + NOALLOC_MAX_CLUSTERS) * mla::dec::HEADS * (mla::dec::DC + 1) * sizeof(float);

}  // namespace

static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_BYTES];

namespace {

// Address of the current device's copy of g_noalloc_scratch. It is looked up
// with cudaGetSymbolAddress on the first call in each CUDA context of a
// device and cached with that context's handle: after a device reset the
// library's device code is loaded again, possibly elsewhere, in a new
// context, and the next call looks the address up again.
mla_status noalloc_scratch(void **ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "mla_decode_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= MAX_DEVICES)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_noalloc: device ordinal %d >= %d", dev, MAX_DEVICES);
  // the current context (runtime calls make the device's primary context current)
  static PFN_cuCtxGetCurrent_v4000 ctx_current = [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      fn = nullptr;
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }();
  CUcontext ctx = nullptr;
  if (ctx_current == nullptr || ctx_current(&ctx) != CUDA_SUCCESS)
    return fail(MLA_ERR_CUDA, "mla_decode_noalloc: cannot query the current CUDA context");
  static std::mutex mu;
  static void *addr[MAX_DEVICES] = {};
  static CUcontext addr_ctx[MAX_DEVICES] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || addr_ctx[dev] != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
      return fail(MLA_ERR_CUDA, "mla_decode_noalloc: cudaGetSymbolAddress of the scratch: %s", cudaGetErrorString(e));
    addr[dev] = p;
    addr_ctx[dev] = ctx;
  }
  *ptr = addr[dev];
  return MLA_OK;
}

}  // namespace

// ------------------------------------------------------------------- C ABI --

extern "C" {

const char *mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
    case MLA_ERR_DEVICE_DATA: return "MLA_ERR_DEVICE_DATA";
  }
  return "MLA_ERR_UNKNOWN";
}

const char *mla_last_error_message(void) { return g_msg.c_str(); }

uint64_t mla_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

mla_status mla_set_launch_overlap(int32_t enable) {
  g_overlap.store(enable != 0 ? 1 : 0, std::memory_order_relaxed);
  return MLA_OK;
}

int32_t mla_get_launch_overlap(void) { return g_overlap.load(std::memory_order_relaxed); }

int32_t mla_uses_tensor_cores(const mla_dims *d, int32_t op) {
  if (d == nullptr || !tc_geometry(d)) return 0;
  return (op >= MLA_OP_APPEND && op <= MLA_OP_ATTEND_A) ? 1 : 0;
}

size_t mla_workspace_size(const mla_dims *d, int32_t op, int32_t rows, int32_t n_q, int64_t max_seq_len,
                          int32_t num_splits) {
  if (d == nullptr || rows <= 0 || num_splits < 0) return 0;
  const bool tc = tc_geometry(d);
  switch (op) {
    case MLA_OP_APPEND: return tc ? tc_append_ws(d, rows) : simt_append_ws(d, rows);
    case MLA_OP_ABSORB: return tc ? tc_absorb_ws(d, rows) : simt_absorb_ws(d, rows);
    case MLA_OP_DECODE:
      return tc ? mla::decode_tc_ws(rows, n_q < 1 ? 1 : n_q, sm_count(), num_splits, max_seq_len) : 0;
    case MLA_OP_OUT_PROJ: return tc ? tc_out_proj_ws(d, rows) : simt_out_proj_ws(d, rows);
    case MLA_OP_O_PROJ: return tc ? tc_o_proj_ws(d, rows) : simt_o_proj_ws(d, rows);
    case MLA_OP_O_PROJ_LATENT: return tc ? tc_o_proj_latent_ws(d, rows) : simt_o_proj_ws(d, rows);
    case MLA_OP_ABSORB_MERGED: return tc ? tc_absorb_merged_ws(d, rows) : simt_absorb_merged_ws(d, rows);
    case MLA_OP_FRONT_END:
      return tc ? tc_front_ws(d, rows) : std::max(simt_append_ws(d, rows), simt_absorb_ws(d, rows));
    case MLA_OP_QUERY_HEADS: return tc ? tc_query_heads_ws(d, rows) : simt_query_heads_ws(d, rows);
    case MLA_OP_ATTEND_A: return tc && max_seq_len > 0 ? tc_attend_a_ws(d, max_seq_len) : 0;
  }
  return 0;
}

mla_status mla_get_device_error(void *stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, mla::g_dev_error, sizeof word);
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "read device error word: %s", cudaGetErrorString(e));
  e = cudaMemcpyToSymbol(mla::g_dev_error, &zero, sizeof zero);
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "clear device error word: %s", cudaGetErrorString(e));
  if (word & MLA_DEVERR_TIMEOUT) return fail(MLA_ERR_TIMEOUT, "a kernel's bounded wait expired");
  if (word & MLA_DEVERR_DATA) return fail(MLA_ERR_DEVICE_DATA, "a kernel found an out-of-range index in device data");
  return MLA_OK;
}

mla_status mla_cache_append(const mla_dims *d, const void *h, const void *W_DKV, const void *W_KR,
                            const int32_t *seq_idx, const int32_t *positions, int32_t T, const mla_cache *c,
                            void *ws, size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!h || !W_DKV || !W_KR || !seq_idx || !positions)
    return fail(MLA_ERR_INVALID_ARG, "append: NULL tensor argument");
  if (!aligned16(h) || !aligned16(W_DKV) || !aligned16(W_KR))
    return fail(MLA_ERR_INVALID_ARG, "append: h and weights must be 16-byte aligned");
  if ((s = check_cache(c, d->d_c + d->d_r)) != MLA_OK) return s;
  const size_t need = mla_workspace_size(d, MLA_OP_APPEND, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "append needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_append(d, h, W_DKV, W_KR, seq_idx, positions, T, c, ws, st);
  if (d->dtype == MLA_BF16)
    return simt_append<__nv_bfloat16>(d, h, W_DKV, W_KR, seq_idx, positions, T, c, ws, st);
  return simt_append<float>(d, h, W_DKV, W_KR, seq_idx, positions, T, c, ws, st);
}

mla_status mla_absorb_q(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQ, const void *W_QR,
                        const void *W_UK, const int32_t *positions, int32_t T, void *q, void *ws, size_t ws_bytes,
                        void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!h || !W_DQ || !W_UQ || !W_QR || !W_UK || !positions || !q)
    return fail(MLA_ERR_INVALID_ARG, "absorb: NULL tensor argument");
  if (!aligned16(h) || !aligned16(W_DQ) || !aligned16(W_UQ) || !aligned16(W_QR) || !aligned16(W_UK) ||
      !aligned16(q))
    return fail(MLA_ERR_INVALID_ARG, "absorb: tensors must be 16-byte aligned");
  const size_t need = mla_workspace_size(d, MLA_OP_ABSORB, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "absorb needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_absorb(d, h, W_DQ, W_UQ, W_QR, W_UK, positions, T, q, ws, st);
  if (d->dtype == MLA_BF16)
    return simt_absorb<__nv_bfloat16>(d, h, W_DQ, W_UQ, W_QR, W_UK, positions, T, q, ws, st);
  return simt_absorb<float>(d, h, W_DQ, W_UQ, W_QR, W_UK, positions, T, q, ws, st);
}

mla_status mla_decode(const mla_dims *d, const void *q, const mla_cache *c, const int32_t *seq_lens, int32_t B,
                      int32_t n_q, void *o_lat, float *lse, int32_t num_splits, void *ws, size_t ws_bytes,
                      void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (B <= 0 || n_q <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_q must be positive");
  if (!q || !seq_lens || !o_lat) return fail(MLA_ERR_INVALID_ARG, "decode: NULL tensor argument");
  if (!aligned16(q) || !aligned16(o_lat)) return fail(MLA_ERR_INVALID_ARG, "decode: q and o_lat must be 16-byte aligned");
  if ((s = check_cache(c, d->d_c + d->d_r)) != MLA_OK) return s;
  if (B > c->num_seqs) return fail(MLA_ERR_INVALID_ARG, "B exceeds cache->num_seqs");
  if (num_splits < 0) return fail(MLA_ERR_INVALID_ARG, "num_splits must be >= 0");
  const size_t need = mla_workspace_size(d, MLA_OP_DECODE, B, n_q, cache_capacity(c), num_splits);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "decode needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return decode_tc(d, q, c, seq_lens, B, n_q, o_lat, lse, num_splits, ws, ws_bytes, st);
  if (d->dtype == MLA_BF16) return simt_decode<__nv_bfloat16>(d, q, c, seq_lens, B, n_q, o_lat, lse, st);
  return simt_decode<float>(d, q, c, seq_lens, B, n_q, o_lat, lse, st);
}

mla_status mla_decode_noalloc(const mla_dims *d, const void *q, const mla_cache *c, const int32_t *seq_lens,
                              int32_t B, int32_t n_q, void *o_lat, float *lse, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (B <= 0 || n_q <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_q must be positive");
  if (static_cast<int64_t>(B) * n_q > NOALLOC_MAX_ROWS)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_noalloc serves at most %d token rows (B * n_q), got %lld",
                NOALLOC_MAX_ROWS, static_cast<long long>(B) * n_q);
  const size_t need = mla_workspace_size(d, MLA_OP_DECODE, B, n_q, 0, 0);
  if (need > NOALLOC_BYTES)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_noalloc: this call needs %zu scratch bytes, %zu are reserved", need,
                NOALLOC_BYTES);
  void *scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != MLA_OK) return s;
  return mla_decode(d, q, c, seq_lens, B, n_q, o_lat, lse, 0, scratch, NOALLOC_BYTES, stream);
}

mla_status mla_out_proj(const mla_dims *d, const void *o_lat, const void *W_UV, int32_t T, void *o, void *ws,
                        size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!o_lat || !W_UV || !o) return fail(MLA_ERR_INVALID_ARG, "out_proj: NULL tensor argument");
  if (!aligned16(o_lat) || !aligned16(W_UV) || !aligned16(o))
    return fail(MLA_ERR_INVALID_ARG, "out_proj: tensors must be 16-byte aligned");
  const size_t need = mla_workspace_size(d, MLA_OP_OUT_PROJ, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "out_proj needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_out_proj(d, o_lat, W_UV, T, o, ws, st);
  if (d->dtype == MLA_BF16) return simt_out_proj<__nv_bfloat16>(d, o_lat, W_UV, T, o, ws, st);
  return simt_out_proj<float>(d, o_lat, W_UV, T, o, ws, st);
}

mla_status mla_o_proj(const mla_dims *d, const void *o, const void *W_O, int32_t T, void *y, void *ws,
                      size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!o || !W_O || !y) return fail(MLA_ERR_INVALID_ARG, "o_proj: NULL tensor argument");
  if (!aligned16(o) || !aligned16(W_O) || !aligned16(y))
    return fail(MLA_ERR_INVALID_ARG, "o_proj: tensors must be 16-byte aligned");
  if (d->d % 2 != 0) return fail(MLA_ERR_UNSUPPORTED, "o_proj: d must be even");
  const size_t need = mla_workspace_size(d, MLA_OP_O_PROJ, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "o_proj needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_o_proj(d, o, W_O, T, y, ws, st);
  if (d->dtype == MLA_BF16) return simt_o_proj<__nv_bfloat16>(d, o, W_O, T, y, ws, st);
  return simt_o_proj<float>(d, o, W_O, T, y, ws, st);
}

mla_status mla_absorb_wo(const mla_dims *d, const void *W_O, const void *W_UV, void *W_OV, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (!W_O || !W_UV || !W_OV) return fail(MLA_ERR_INVALID_ARG, "absorb_wo: NULL tensor argument");
  if (!aligned16(W_O) || !aligned16(W_UV) || !aligned16(W_OV))
    return fail(MLA_ERR_INVALID_ARG, "absorb_wo: tensors must be 16-byte aligned");
  if (d->d > 65535) return fail(MLA_ERR_UNSUPPORTED, "absorb_wo: d > 65535");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_absorb_wo(d, W_O, W_UV, W_OV, st);
  if (d->dtype == MLA_BF16) return simt_absorb_wo<__nv_bfloat16>(d, W_O, W_UV, W_OV, st);
  return simt_absorb_wo<float>(d, W_O, W_UV, W_OV, st);
}

mla_status mla_o_proj_latent(const mla_dims *d, const void *o_lat, const void *W_OV, int32_t T, void *y, void *ws,
                             size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!o_lat || !W_OV || !y) return fail(MLA_ERR_INVALID_ARG, "o_proj_latent: NULL tensor argument");
  if (!aligned16(o_lat) || !aligned16(W_OV) || !aligned16(y))
    return fail(MLA_ERR_INVALID_ARG, "o_proj_latent: tensors must be 16-byte aligned");
  if (d->d % 2 != 0) return fail(MLA_ERR_UNSUPPORTED, "o_proj_latent: d must be even");
  const size_t need = mla_workspace_size(d, MLA_OP_O_PROJ_LATENT, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "o_proj_latent needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_o_proj_latent(d, o_lat, W_OV, T, y, ws, st);
  if (d->dtype == MLA_BF16) return simt_o_proj_latent<__nv_bfloat16>(d, o_lat, W_OV, T, y, ws, st);
  return simt_o_proj_latent<float>(d, o_lat, W_OV, T, y, ws, st);
}

mla_status mla_absorb_merge(const mla_dims *d, const void *W_UQ, const void *W_UK, void *W_UQK, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (!W_UQ || !W_UK || !W_UQK) return fail(MLA_ERR_INVALID_ARG, "absorb_merge: NULL tensor argument");
  if (!aligned16(W_UQ) || !aligned16(W_UK) || !aligned16(W_UQK))
    return fail(MLA_ERR_INVALID_ARG, "absorb_merge: tensors must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_absorb_merge(d, W_UQ, W_UK, W_UQK, st);
  if (d->dtype == MLA_BF16) return simt_absorb_merge<__nv_bfloat16>(d, W_UQ, W_UK, W_UQK, st);
  return simt_absorb_merge<float>(d, W_UQ, W_UK, W_UQK, st);
}

mla_status mla_absorb_q_merged(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQK,
                               const void *W_QR, const int32_t *positions, int32_t T, void *q, void *ws,
                               size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!h || !W_DQ || !W_UQK || !W_QR || !positions || !q)
    return fail(MLA_ERR_INVALID_ARG, "absorb_q_merged: NULL tensor argument");
  if (!aligned16(h) || !aligned16(W_DQ) || !aligned16(W_UQK) || !aligned16(W_QR) || !aligned16(q))
    return fail(MLA_ERR_INVALID_ARG, "absorb_q_merged: tensors must be 16-byte aligned");
  const size_t need = mla_workspace_size(d, MLA_OP_ABSORB_MERGED, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws))
    return fail(MLA_ERR_WORKSPACE, "absorb_q_merged needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_absorb_q_merged(d, h, W_DQ, W_UQK, W_QR, positions, T, q, ws, st);
  if (d->dtype == MLA_BF16)
    return simt_absorb_q_merged<__nv_bfloat16>(d, h, W_DQ, W_UQK, W_QR, positions, T, q, ws, st);
  return simt_absorb_q_merged<float>(d, h, W_DQ, W_UQK, W_QR, positions, T, q, ws, st);
}

mla_status mla_front_end(const mla_dims *d, const void *h, const void *W_DKV, const void *W_KR, const void *W_DQ,
                         const void *W_UQ, const void *W_QR, const void *W_UK, const int32_t *seq_idx,
                         const int32_t *positions, int32_t T, const mla_cache *c, void *q, void *ws, size_t ws_bytes,
                         void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!h || !W_DKV || !W_KR || !W_DQ || !W_UQ || !W_QR || !W_UK || !seq_idx || !positions || !q)
    return fail(MLA_ERR_INVALID_ARG, "front_end: NULL tensor argument");
  if (!aligned16(h) || !aligned16(W_DKV) || !aligned16(W_KR) || !aligned16(W_DQ) || !aligned16(W_UQ) ||
      !aligned16(W_QR) || !aligned16(W_UK) || !aligned16(q))
    return fail(MLA_ERR_INVALID_ARG, "front_end: tensors must be 16-byte aligned");
  if ((s = check_cache(c, d->d_c + d->d_r)) != MLA_OK) return s;
  const size_t need = mla_workspace_size(d, MLA_OP_FRONT_END, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "front_end needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d))
    return tc_front_end(d, h, W_DKV, W_KR, W_DQ, W_UQ, W_QR, W_UK, seq_idx, positions, T, c, q, ws, st);
  // CUDA-core dims: the two calls one after the other (each reads h)
  if ((s = mla_cache_append(d, h, W_DKV, W_KR, seq_idx, positions, T, c, ws, ws_bytes, stream)) != MLA_OK) return s;
  return mla_absorb_q(d, h, W_DQ, W_UQ, W_QR, W_UK, positions, T, q, ws, ws_bytes, stream);
}

mla_status mla_query_heads(const mla_dims *d, const void *h, const void *W_DQ, const void *W_UQ, const void *W_QR,
                           const int32_t *positions, int32_t T, void *qa, void *ws, size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (T <= 0) return fail(MLA_ERR_INVALID_ARG, "T must be positive");
  if (!h || !W_DQ || !W_UQ || !W_QR || !positions || !qa)
    return fail(MLA_ERR_INVALID_ARG, "query_heads: NULL tensor argument");
  if (!aligned16(h) || !aligned16(W_DQ) || !aligned16(W_UQ) || !aligned16(W_QR) || !aligned16(qa))
    return fail(MLA_ERR_INVALID_ARG, "query_heads: tensors must be 16-byte aligned");
  const size_t need = mla_workspace_size(d, MLA_OP_QUERY_HEADS, T, 1, 0, 0);
  if (ws_bytes < need || (need && !ws)) return fail(MLA_ERR_WORKSPACE, "query_heads needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_query_heads(d, h, W_DQ, W_UQ, W_QR, positions, T, qa, ws, st);
  if (d->dtype == MLA_BF16) return simt_query_heads<__nv_bfloat16>(d, h, W_DQ, W_UQ, W_QR, positions, T, qa, ws, st);
  return simt_query_heads<float>(d, h, W_DQ, W_UQ, W_QR, positions, T, qa, ws, st);
}

mla_status mla_attend_order_a(const mla_dims *d, const void *qa, const void *W_UK, const void *W_UV,
                              const mla_cache *c, const int32_t *seq_lens, int32_t B, int32_t n_q, void *o, void *ws,
                              size_t ws_bytes, void *stream) {
  mla_status s = check_dims(d);
  if (s != MLA_OK) return s;
  if (B <= 0 || n_q <= 0) return fail(MLA_ERR_INVALID_ARG, "B and n_q must be positive");
  if (!qa || !W_UK || !W_UV || !seq_lens || !o) return fail(MLA_ERR_INVALID_ARG, "attend_order_a: NULL tensor argument");
  if (!aligned16(qa) || !aligned16(W_UK) || !aligned16(W_UV) || !aligned16(o))
    return fail(MLA_ERR_INVALID_ARG, "attend_order_a: tensors must be 16-byte aligned");
  if ((s = check_cache(c, d->d_c + d->d_r)) != MLA_OK) return s;
  if (B > c->num_seqs) return fail(MLA_ERR_INVALID_ARG, "B exceeds cache->num_seqs");
  if (d->d_h > 128 || d->d_r > 128) return fail(MLA_ERR_UNSUPPORTED, "attend_order_a: d_h and d_r must be <= 128");
  const size_t need = mla_workspace_size(d, MLA_OP_ATTEND_A, B, n_q, cache_rows_of(c), 0);
  if (ws_bytes < need || (need && !ws))
    return fail(MLA_ERR_WORKSPACE, "attend_order_a needs %zu workspace bytes", need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_geometry(d)) return tc_attend_a(d, qa, W_UK, W_UV, c, seq_lens, B, n_q, o, ws, st);
  if (d->dtype == MLA_BF16) return simt_attend_a<__nv_bfloat16>(d, qa, W_UK, W_UV, c, seq_lens, B, n_q, o, st);
  return simt_attend_a<float>(d, qa, W_UK, W_UV, c, seq_lens, B, n_q, o, st);
}

mla_status mla_selftest_timeout(uint64_t wait_ns, void *scratch, size_t scratch_bytes, void *stream) {
  if (wait_ns == 0) return fail(MLA_ERR_INVALID_ARG, "selftest_timeout: wait_ns must be positive");
  if (scratch == nullptr || !aligned16(scratch) || scratch_bytes < SELFTEST_BYTES)
    return fail(MLA_ERR_INVALID_ARG, "selftest_timeout: needs %zu bytes of 16-byte aligned device scratch",
                SELFTEST_BYTES);
  return tc_selftest_timeout(wait_ns, scratch, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
