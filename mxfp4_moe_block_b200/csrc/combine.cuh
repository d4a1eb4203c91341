// combine.cuh -- weighted combine of the k expert outputs of each token
// (plus an optional residual), and the parameter-free RMSNorm used between
// stacked layers.  Both are row kernels bound by HBM: 16-byte loads, one
// CTA per token row.
#pragma once
#include "common.cuh"

namespace moe {

// out[t] = bf16( sum_j w[t,j] * y[pair_row[t*k+j]] + residual[t] ), float,
// slots in order j = 0..k-1, residual last.  H % 4 == 0.  grid (T, column
// blocks of 4*blockDim elements): each thread keeps k 16-byte loads in flight.
__global__ void __launch_bounds__(256)
combine_kernel(const float *__restrict__ y, const int32_t *__restrict__ pair_row,
               const float *__restrict__ topk_w, int T, int k, int H,
               const uint16_t *residual, uint16_t *out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  if (t >= T) return;
  const int cbeg = blockIdx.y * blockDim.x * 4;
  __shared__ const float *rows[32];
  __shared__ float wts[32];
  if (threadIdx.x < k) {
    rows[threadIdx.x] =
        y + (size_t)checked_index(__ldg(pair_row + (size_t)t * k + threadIdx.x), (long)T * k) * H;
    wts[threadIdx.x] = __ldg(topk_w + (size_t)t * k + threadIdx.x);
  }
  __syncthreads();
  for (int c = cbeg + threadIdx.x * 4; c < H && c < cbeg + (int)blockDim.x * 4;
       c += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(rows[j] + c));
      const float w = wts[j];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    if (residual) {
      const uint2 r = *reinterpret_cast<const uint2 *>(residual + (size_t)t * H + c);
      acc.x += bf16_lo(r.x);
      acc.y += bf16_hi(r.x);
      acc.z += bf16_lo(r.y);
      acc.w += bf16_hi(r.y);
    }
    uint2 o;
    o.x = (uint32_t)f32_to_bf16_bits(acc.x) | ((uint32_t)f32_to_bf16_bits(acc.y) << 16);
    o.y = (uint32_t)f32_to_bf16_bits(acc.z) | ((uint32_t)f32_to_bf16_bits(acc.w) << 16);
    *reinterpret_cast<uint2 *>(out + (size_t)t * H + c) = o;
  }
}

// out[t] = bf16( x[t] / sqrt(mean(x[t]^2) + eps) ).  H % 8 == 0.
__global__ void __launch_bounds__(256)
rms_norm_kernel(const uint16_t *x, int T, int H, float eps, uint16_t *out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  if (t >= T) return;
  const uint16_t *row = x + (size_t)t * H;
  float ss = 0.f;
  for (int c = threadIdx.x * 8; c < H; c += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4 *>(row + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float a = bf16_lo(w[u]), b = bf16_hi(w[u]);
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float s = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    s = warp_sum(s);
    if (threadIdx.x == 0) red[0] = s;
  }
  __syncthreads();
  const float inv = 1.f / sqrtf(red[0] / (float)H + eps);
  for (int c = threadIdx.x * 8; c < H; c += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4 *>(row + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      o[u] = (uint32_t)f32_to_bf16_bits(bf16_lo(w[u]) * inv) |
             ((uint32_t)f32_to_bf16_bits(bf16_hi(w[u]) * inv) << 16);
    *reinterpret_cast<uint4 *>(out + (size_t)t * H + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace moe
