// ffn_fma.cuh -- MXFP4 expert FFN on the CUDA cores: dequantise to
// registers, float FMA.  The variant for few tokens per expert, where the
// step is a stream of weight bytes (the memory-bound regime that
// "mimo-tilert-1000tps-trillion-parameter-inference", section
// "万亿参数推理为什么特别难", describes: token rate = bandwidth / bytes per token).
//
// Work layout: one warp owns a group of NR weight rows of one expert and the
// whole K range.  Lane l takes the 16-byte chunks l, l+32, ... of every row
// (16 bytes = 32 E2M1 codes = exactly one MX block with one scale byte), so
// each warp-wide load moves 512 contiguous bytes of a row.  Per chunk the
// lane decodes two codes at a time (hardware E2M1x2 -> f16x2 conversion, then
// to float), multiplies the pair by the block's E8M0 scale (an exact power of
// two: the dequantised weights) and accumulates even/odd products with packed
// f32x2 FMAs; the warp reduces at the end.  Activations are read as
// float (converted once by x_to_f32_kernel; GEMM-1 stores h in float too).
// Items (expert, row group) are dealt to warps in contiguous runs, so a
// warp's consecutive items share the expert and its activations stay in L1.
#pragma once
#include "common.cuh"

namespace moe {

struct FfnArgs {
  const uint16_t *x;        // [T, H] bf16
  int T, H, I, E, k;
  const uint8_t *w13c;      // [E, 2I, H/2]
  const uint8_t *w13s;      // [E, 2I, H/32]
  const uint8_t *w2c;       // [E, H, I/2]
  const uint8_t *w2s;       // [E, H, I/32]
  const int32_t *off;       // [E+1]
  const int32_t *sp;        // [P]
  uint16_t *h;              // [P, I] bf16 workspace (SwiGLU output)
  float *y;                 // [P, H]
  float *x32;               // [T, H] float workspace
  float *h32;               // [P, I] float workspace (h, exactly)
};

constexpr int FMA_THREADS = 384;

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra = *reinterpret_cast<unsigned long long *>(&a);
  unsigned long long rb = *reinterpret_cast<unsigned long long *>(&b);
  unsigned long long rc = *reinterpret_cast<unsigned long long *>(&c);
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(ra), "l"(rb), "l"(rc));
  return *reinterpret_cast<float2 *>(&d);
}

// x [T, H] bf16 -> float.
__global__ void __launch_bounds__(256)
x_to_f32_kernel(const uint16_t *__restrict__ x, size_t n8, float *__restrict__ x32) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x) + i);
    float4 *o = reinterpret_cast<float4 *>(x32) + 2 * i;
    o[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    o[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
}

// Active-expert list of one CTA: experts with at least one row, ascending.
// Built by warp 0; returns the count after a __syncthreads.
__device__ __forceinline__ int build_active(const int32_t *__restrict__ off, int E, long P,
                                            int *s_act, int *s_n) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int n = 0;
    if (!offsets_ok(off, E, P)) E = 0;           // checked build: bad offsets, no work
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const bool on = e < E && __ldg(off + e + 1) > __ldg(off + e);
      const unsigned b = __ballot_sync(FULL, on);
      if (on) s_act[n + __popc(b & lanemask_lt())] = e;
      n += __popc(b);
    }
    if (lane == 0) *s_n = n;
  }
  __syncthreads();
  return *s_n;
}

// Lane-partial dot products of NR weight rows with NT float activation rows.
// wc / ws point at the expert's first row; row r's codes start at
// wc + rowoff[r] * (kdim/2), its scales at ws + rowoff[r] * (kdim/32).
template <int NR, int NT>
__device__ __forceinline__ void fma_rows(const uint8_t *__restrict__ wc,
                                         const uint8_t *__restrict__ ws,
                                         const uint32_t (&rowoff)[NR], int kdim,
                                         const float *const (&xr)[NT], int lane,
                                         float (&acc)[NR][NT]) {
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[r][j] = 0.f;
  const int nchunks = kdim >> 5;
  const uint32_t cstride = (uint32_t)kdim >> 1, sstride = (uint32_t)kdim >> 5;

  for (int c = lane; c < nchunks; c += 32) {
    uint4 q[NR];
    uint32_t sc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      q[r] = ld_stream16(wc + (rowoff[r] * cstride + (uint32_t)c * 16));
      sc[r] = __ldg(ws + (rowoff[r] * sstride + (uint32_t)c));
    }
    float2 xv[NT][16];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const float4 *p = reinterpret_cast<const float4 *>(xr[j] + (size_t)c * 32);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 f = __ldg(p + u);
        xv[j][2 * u] = make_float2(f.x, f.y);
        xv[j][2 * u + 1] = make_float2(f.z, f.w);
      }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      // each code pair times the block's scale (exact: a power of two) is
      // the dequantised weight pair, so every product is weight x activation
      // -- no block partial sum outside the range of the result
      float2 part[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) part[j] = make_float2(0.f, 0.f);
      const uint32_t qw[4] = {q[r].x, q[r].y, q[r].z, q[r].w};
#pragma unroll
      for (int b = 0; b < 16; ++b) {
        const float s = e8m0_to_f32(sc[r]);
        float2 wv = e2m1x2_to_f32x2(qw[b >> 2] >> (8 * (b & 3)));
        wv.x *= s;
        wv.y *= s;
#pragma unroll
        for (int j = 0; j < NT; ++j) part[j] = ffma2(wv, xv[j][b], part[j]);
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) acc[r][j] += part[j].x + part[j].y;
    }
  }
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[r][j] = warp_sum(acc[r][j]);
}

// GEMM-1 + SwiGLU for NT tokens starting at sorted row r0 + t0: RG gate rows
// from n0 and the matching RG up rows.
template <int RG, int NT>
__device__ __forceinline__ void ffn1_group(const FfnArgs &a, int e, int n0, int r0, int t0,
                                           int lane) {
  uint32_t rowoff[2 * RG];
#pragma unroll
  for (int r = 0; r < 2 * RG; ++r) rowoff[r] = (uint32_t)(r < RG ? n0 + r : a.I + n0 + r - RG);
  const size_t erows = (size_t)e * 2 * a.I;
  const float *xr[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j)
    xr[j] = a.x32 + (size_t)(checked_index(__ldg(a.sp + r0 + t0 + j), (long)a.T * a.k) / a.k) * a.H;
  float acc[2 * RG][NT];
  fma_rows<2 * RG, NT>(a.w13c + erows * (a.H / 2), a.w13s + erows * (a.H / 32), rowoff, a.H,
                       xr, lane, acc);
#pragma unroll
  for (int r = 0; r < RG; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (lane == r * NT + j) {
        const float g = acc[r][j], u = acc[RG + r][j];
        const uint16_t hb = f32_to_bf16_bits(g / (1.f + expf(-g)) * u);
        const size_t o = (size_t)(r0 + t0 + j) * a.I + n0 + r;
        a.h[o] = hb;
        a.h32[o] = __uint_as_float((uint32_t)hb << 16);
      }
    }
}

template <int RG>
__global__ void __launch_bounds__(FMA_THREADS, 1)
ffn1_fma_kernel(FfnArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_act[1024];
  __shared__ int s_n;
  const int n_act = build_active(a.off, a.E, (long)a.T * a.k, s_act, &s_n);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int gpe = a.I / RG;                       // row groups per expert
  const long total = (long)n_act * gpe;
  const long per = (total + nw - 1) / nw;
  const long i0 = (long)gw * per, i1 = min(total, i0 + per);
  for (long it = i0; it < i1; ++it) {
    const int e = s_act[it / gpe];
    const int n0 = (int)(it % gpe) * RG;
    const int r0 = __ldg(a.off + e), ne = __ldg(a.off + e + 1) - r0;
    int t0 = 0;
    for (; t0 + 2 <= ne; t0 += 2) ffn1_group<RG, 2>(a, e, n0, r0, t0, lane);
    if (t0 < ne) ffn1_group<RG, 1>(a, e, n0, r0, t0, lane);
  }
}

// GEMM-2 (down projection): RD rows of W2 of one expert, NT tokens.
template <int RD, int NT>
__device__ __forceinline__ void ffn2_group(const FfnArgs &a, int e, int m0, int r0, int t0,
                                           int lane) {
  uint32_t rowoff[RD];
#pragma unroll
  for (int r = 0; r < RD; ++r) rowoff[r] = (uint32_t)(m0 + r);
  const size_t erows = (size_t)e * a.H;
  const float *hr[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) hr[j] = a.h32 + (size_t)(r0 + t0 + j) * a.I;
  float acc[RD][NT];
  fma_rows<RD, NT>(a.w2c + erows * (a.I / 2), a.w2s + erows * (a.I / 32), rowoff, a.I, hr,
                   lane, acc);
#pragma unroll
  for (int r = 0; r < RD; ++r)
#pragma unroll
    for (int j = 0; j < NT; ++j)
      if (lane == j * RD + r) a.y[(size_t)(r0 + t0 + j) * a.H + m0 + r] = acc[r][j];
}

template <int RD>
__global__ void __launch_bounds__(FMA_THREADS, 1)
ffn2_fma_kernel(FfnArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_act[1024];
  __shared__ int s_n;
  const int n_act = build_active(a.off, a.E, (long)a.T * a.k, s_act, &s_n);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int gpe = a.H / RD;
  const long total = (long)n_act * gpe;
  const long per = (total + nw - 1) / nw;
  const long i0 = (long)gw * per, i1 = min(total, i0 + per);
  for (long it = i0; it < i1; ++it) {
    const int e = s_act[it / gpe];
    const int m0 = (int)(it % gpe) * RD;
    const int r0 = __ldg(a.off + e), ne = __ldg(a.off + e + 1) - r0;
    int t0 = 0;
    for (; t0 + 2 <= ne; t0 += 2) ffn2_group<RD, 2>(a, e, m0, r0, t0, lane);
    if (t0 < ne) ffn2_group<RD, 1>(a, e, m0, r0, t0, lane);
  }
}

}  // namespace moe
