// Shared device helpers of libmla: the device error word, storage-type loads
// and stores, and RoPE angles.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#define MLA_DEVERR_DATA 1u     // an index from device memory was out of range
#define MLA_DEVERR_TIMEOUT 2u  // a bounded wait expired

namespace mla {

// One word per device, read and cleared by mla_get_device_error().
__device__ unsigned int g_dev_error;

__device__ __forceinline__ void dev_error(unsigned int code) { atomicOr(&g_dev_error, code); }

template <typename T>
__device__ __forceinline__ float ld_f(const T *p);
template <>
__device__ __forceinline__ float ld_f<float>(const float *p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Pack two floats into one bf16x2 word (round to nearest even), low = a.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

// RoPE (RoFormer, interleaved pairs): the pair (x0, x1) = (x[2i], x[2i+1]) is
// rotated by the angle pos * theta_i, theta_i = base^(-2i/d_r).
__device__ __forceinline__ double rope_theta(int pair, int d_r, double base) {
  return exp2(-2.0 * static_cast<double>(pair) / static_cast<double>(d_r) * log2(base));
}

// The angle is formed and reduced to [-pi, pi] in double (so positions up to
// 2^17 and beyond keep full accuracy); on that range the fast hardware sine
// and cosine (__sincosf: absolute error below 2^-21.4 there) are far more
// accurate than the bf16 results, and they keep the unrolled epilogues small.
__device__ __forceinline__ void rope_cos_sin(int pos, double theta, float &c, float &s) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  const double a = static_cast<double>(pos) * theta;
  const double k = rint(a * (1.0 / kTwoPi));
  __sincosf(static_cast<float>(fma(-k, kTwoPi, a)), &s, &c);
}
__device__ __forceinline__ void rope_apply(float &x0, float &x1, float c, float s) {
  const float y0 = x0 * c - x1 * s;
  const float y1 = x0 * s + x1 * c;
  x0 = y0;
  x1 = y1;
}
__device__ __forceinline__ void rope_rotate(float &x0, float &x1, int pos, double theta) {
  float c, s;
  rope_cos_sin(pos, theta, c, s);
  rope_apply(x0, x1, c, s);
}

__device__ __forceinline__ void rope_pair(float &x0, float &x1, int pair, int d_r, int pos, double base) {
  rope_rotate(x0, x1, pos, rope_theta(pair, d_r, base));
}

// Physical cache row of logical (b, pos); returns -1 when out of range.
struct CacheView {
  void *data;
  const int32_t *block_table;
  int64_t max_len;
  int64_t num_blocks;
  int32_t paged;
  int32_t block_size;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
};

__device__ __forceinline__ int64_t cache_row(const CacheView &c, int b, int64_t pos) {
  if (b < 0 || b >= c.num_seqs || pos < 0) return -1;
  if (!c.paged) return pos < c.max_len ? static_cast<int64_t>(b) * c.max_len + pos : -1;
  const int64_t blk_idx = pos / c.block_size;
  if (blk_idx >= c.max_blocks_per_seq) return -1;
  const int64_t blk = c.block_table[static_cast<int64_t>(b) * c.max_blocks_per_seq + blk_idx];
  if (blk < 0 || blk >= c.num_blocks) return -1;
  return blk * c.block_size + pos % c.block_size;
}

}  // namespace mla
