// common.cuh -- device helpers shared by the kernels of the MXFP4 MoE
// block-verify library (sm_100a).  Built as one translation unit with
// mxfp4_moe.cu, so __device__ globals here are visible to every kernel.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>
#include <utility>

#include "../../include/mxfp4_moe.h"

namespace moe {

// Sticky device status word: the first error detail wins.
__device__ int g_status;

__device__ __forceinline__ void raise_status(int detail) {
  atomicCAS(&g_status, 0, detail);
}

// Checked build (-DMOE_CHECKS, libmxfp4_moe_checks.so): every index read
// from a caller's array -- the pair ids of sorted_pair and pair_row, the
// expert offsets -- is checked before it addresses memory; a bad one sets
// MOE_DEV_BAD_INDEX and is replaced by 0 (offsets: the call's experts are
// left empty).  No trap, no access outside the arrays.  Off in the normal
// build, where those arrays are trusted to come from moe_permute.
#ifdef MOE_CHECKS
constexpr bool kChecks = true;
__device__ __forceinline__ int checked_index(int i, long n) {
  if (i < 0 || i >= n) {
    raise_status(MOE_DEV_BAD_INDEX);
    return 0;
  }
  return i;
}
#else
constexpr bool kChecks = false;
__device__ __forceinline__ int checked_index(int i, long) { return i; }
#endif

// Checked build: expert offsets off[0..E] non-decreasing from >= 0 to <= P,
// tested by one warp (all lanes get the verdict); false sets MOE_DEV_BAD_INDEX.
__device__ __forceinline__ bool offsets_ok(const int32_t *off, int E, long P) {
  if (!kChecks) return true;
  bool bad = false;
  for (int e = (int)(threadIdx.x & 31); e < E; e += 32) {
    const int a = __ldg(off + e), b = __ldg(off + e + 1);
    bad |= a < 0 || b < a || b > P;
  }
  bad = __any_sync(0xffffffffu, bad);
  if (bad && (threadIdx.x & 31) == 0) raise_status(MOE_DEV_BAD_INDEX);
  return !bad;
}

constexpr unsigned FULL = 0xffffffffu;

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation, so the next kernel on the stream
// may become resident (and run its prologue) while this one finishes.
// pdl_wait() blocks until the preceding kernel on the stream has completed
// and its writes are visible; a kernel calls it before it reads anything a
// preceding kernel may have written, and before its first global write.
// pdl_trigger() lets the next kernel launch; kernels call it after their
// wait, so a kernel that starts early finds everything two launches back
// complete.  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host: launch `kernel` with programmatic stream serialisation allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same for clusters of `cluster_x` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                      size_t smem, unsigned cluster_x, cudaStream_t stream,
                                      Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// bf16 bit patterns packed two per 32-bit word -> float.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&b);
}

// E8M0 scale byte -> 2^(e-127) as float (0 -> 2^-127, a subnormal; 255 -> NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  if (e == 0u) return __uint_as_float(0x00400000u);
  if (e == 255u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float(e << 23);
}

// Two E2M1 codes of one byte (low nibble = even element) -> two floats, exact.
__device__ __forceinline__ float2 e2m1x2_to_f32x2(uint32_t byte) {
  __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xffu), __NV_E2M1);
  return __half22float2(*reinterpret_cast<__half2 *>(&r));
}

// 16-byte streaming load that bypasses L1 (weights are read exactly once).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

// (value, index) argmax order: larger value first, then the lower index.
// idx < 0 marks "no candidate".
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return bi < 0 || (i >= 0 && (v > bv || (v == bv && i < bi)));
}

__device__ __forceinline__ void warp_argmax(float &v, int &i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(FULL, v, o);
    int oi = __shfl_xor_sync(FULL, i, o);
    if (better(ov, oi, v, i)) { v = ov; i = oi; }
  }
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace moe
