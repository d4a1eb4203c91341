// quantize.cuh -- bf16 weights -> OCP MXFP4 (E2M1 codes + E8M0 block scales).
//
// The expert weights the verify step streams are MXFP4 ("MiMo-v2.5-Pro-
// UltraSpeed - infra 架构解读", section "FP4 Expert 量化";
// "mimo-tilert-1000tps-trillion-parameter-inference", section "第一层：FP4
// 选择性量化").  This kernel produces that format from bf16 weights by the
// OCP MX v1.0 conversion: per 32 consecutive elements of a row the shared
// scale is 2^(floor(log2 amax) - 2) (2 = the largest E2M1 exponent), and each
// element becomes the nearest E2M1 value of v / scale, ties to the even
// code, saturating at +-6, its sign kept -- the hardware conversion
// (cvt.rn.satfinite.e2m1x2.f32) applies exactly that rule to the exactly
// scaled value.
//
// HBM-bound: 2 bytes read and 17/32 byte written per element.  Each thread
// takes 8 consecutive elements (one 16-byte load, one 4-byte store of codes);
// four neighbouring threads hold a 32-element block and meet by shuffles.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int QUANT_THREADS = 256;

// Quantise one group of 8 bf16 (w4 = its 16 bytes) of a 32-element block
// whose other three groups sit in lanes lane^1, lane^2, lane^3: returns the
// packed codes, and the block's scale byte in *sb.
__device__ __forceinline__ uint32_t quantize_group8(const uint4 v, uint32_t *sb) {
  const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
  // largest magnitude of the block: bf16 bit patterns without the sign
  // compare like the magnitudes they encode
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(wd[i] & 0x7fffu, (wd[i] >> 16) & 0x7fffu));
  m = max(m, __shfl_xor_sync(FULL, m, 1));
  m = max(m, __shfl_xor_sync(FULL, m, 2));
  // scale byte = floor(log2 amax) - 2 + 127 = (biased exponent of amax) - 2,
  // at least 0 (all-zero and tiny blocks); bf16 exponents stop at 254, so
  // the byte never exceeds 252
  const int be = (int)(m >> 7);
  const uint32_t s = (uint32_t)max(0, be - 2);
  const float inv = __uint_as_float((254u - s) << 23);   // 2^(127 - s), exact
  // v * 2^(127 - s) is exact wherever it can reach 0.25 (and stays below 8);
  // the conversion rounds it to the nearest E2M1 value, ties to the even
  // code (the IEEE rule: mantissa bit 0), saturating at +-6 and keeping the
  // sign (-0 -> code 8); two codes per instruction, the first in the low
  // nibble
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = make_float2(bf16_lo(wd[i]) * inv, bf16_hi(wd[i]) * inv);
    const uint32_t byte =
        (uint32_t)__nv_cvt_float2_to_fp4x2(f, __NV_E2M1, cudaRoundNearest) & 0xffu;
    word |= byte << (8 * i);
  }
  *sb = s;
  return word;
}

// w: n8 groups of 8 bf16 (n8 = R*K/8); codes: 4 bytes per group; scales: one
// byte per 4 groups.  Each warp takes QUANT_UNROLL runs of 32 consecutive
// groups per trip, all loads first, so that each thread keeps QUANT_UNROLL
// 16-byte loads in flight (8: 0.95 of the copy bandwidth, against 0.77 with 4;
// the run offsets are added to per-trip pointers, which keeps the 8 runs in
// registers).
constexpr int QUANT_UNROLL = 8;

__global__ void __launch_bounds__(QUANT_THREADS)
mxfp4_quantize_kernel(const uint16_t *__restrict__ w, size_t n8, uint8_t *__restrict__ codes,
                      uint8_t *__restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const unsigned lane = threadIdx.x & 31;
  const size_t warps = ((size_t)gridDim.x * blockDim.x) >> 5;
  const size_t wid = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  // the loop bound is warp-uniform (every lane takes part in the shuffles);
  // n8 is a multiple of 4, so the four threads of a block are valid together
  for (size_t r0 = wid * QUANT_UNROLL; r0 * 32 < n8; r0 += warps * QUANT_UNROLL) {
    // this lane's first group of the trip; run u is 32u groups further on
    const size_t g0 = r0 * 32 + lane;
    const uint4 *src = reinterpret_cast<const uint4 *>(w) + g0;
    const unsigned left = (unsigned)min((size_t)(32 * QUANT_UNROLL), n8 - r0 * 32);
    uint4 v[QUANT_UNROLL];
#pragma unroll
    for (int u = 0; u < QUANT_UNROLL; ++u)
      v[u] = 32u * u + lane < left ? ld_stream16(src + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t *dst = reinterpret_cast<uint32_t *>(codes) + g0;
    uint8_t *sdst = scales + (g0 >> 2);
#pragma unroll
    for (int u = 0; u < QUANT_UNROLL; ++u) {
      uint32_t sb;
      const uint32_t word = quantize_group8(v[u], &sb);
      if (32u * u + lane < left) {
        dst[32 * u] = word;
        if ((lane & 3) == 0) sdst[8 * u] = (uint8_t)sb;
      }
    }
  }
}

}  // namespace moe
