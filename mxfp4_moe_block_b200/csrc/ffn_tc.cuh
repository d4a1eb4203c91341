// ffn_tc.cuh -- MXFP4 expert FFN on the 5th-generation tensor cores.
//
// The expert weights stay in their MXFP4 form all the way into the tensor
// core: the block-scaled tcgen05.mma takes A = E2M1 codes with one E8M0
// scale per 32 elements -- exactly the OCP MX block the pages name for the
// experts ("MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section "FP4 Expert
// 量化"; "mimo-tilert-1000tps-trillion-parameter-inference", section
// "第一层：FP4 选择性量化").  Nothing is dequantised on the CUDA cores.
//
// The activations (bf16) become the B operand as a short sum of narrow terms
// (see "activation block encodings" below): eight E2M1 terms with one scale
// per row and term for kind::mxf4 (exact for bf16), or two E4M3 terms with
// E8M0 block scales for kind::mxf8f6f4 (two B columns per token where tiles
// are wide).
//
// One persistent CTA per SM takes tiles (expert, 128-row block of the weight
// matrix, block of B rows): its first from blockIdx.x, the rest from an
// atomic counter.  Warp roles, after the tile-pipelining and
// warp-specialisation ideas the pages describe for TileRT (prior art):
//   warp 0     TMA producer: the weight tile (one box) and the activation tile
//              of each stage,
//              and the tile index ring every other role reads;
//   warp 1     scale loader: the scale bytes into shared memory -- by TMA,
//              16 bytes of each row per four stages (kind::mxf8f6f4, K a
//              multiple of 512), else by cp.async in the 32-row x 16-byte
//              layout of the scale-factor columns;
//   warp 2     TMEM allocation and the single MMA-issuing thread;
//   warp 3     constant B block scales (kind::mxf4);
//   warps 4-7  epilogue: TMEM -> registers -> SwiGLU (GEMM-1) or y (GEMM-2);
//   warps 8-11 scale writers: tcgen05.st of the stage's scale factors
//              (weights, and kind::mxf8f6f4's activation block scales);
//   warps 12-15 a second epilogue group (kind::mxf8f6f4).
// Every wait is bounded; on time-out the kernel records MOE_DEV_TIMEOUT,
// drains what it issued, frees its TMEM and returns.
#pragma once
#include <cuda.h>
#include <atomic>
#include <mutex>
#include "common.cuh"
#include "ffn_fma.cuh"

namespace moe {

// ------------------------------------------------------------ PTX wrappers --

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded waits.  The pipeline's waits give up after g_wait_limit_ns (2 s
// unless moe_set_wait_limit_ns lowered it): the waiting role sets the CTA's
// abort flag and the status word (MOE_DEV_TIMEOUT), and every role then
// leaves its loop.  The drain at the end of the kernel -- for copies and MMAs
// already issued -- has its own fixed limit, so that a lowered pipeline limit
// never cuts a drain short.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;
constexpr uint64_t kDrainLimitNs = 2000000000ull;

__device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  const uint64_t limit = *(volatile unsigned long long *)&g_wait_limit_ns;
  // each try_wait may itself suspend the thread for a while, so the flag
  // and the clock are checked after every one of them
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 >= limit) {
      raise_status(MOE_DEV_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// Wait for the completion of work already issued (abort flag ignored).
__device__ __noinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 >= kDrainLimitNs) {
      raise_status(MOE_DEV_TIMEOUT);
      return false;
    }
  }
}

// Flags in global memory between the CTAs of one launch (the fused FFN):
// release / acquire at GPU scope, and a bounded wait like the barrier waits.
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// atomic add with acquire-release semantics at GPU scope; returns the old value
__device__ __forceinline__ int atom_add_acq_rel_gpu(int *p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}
__device__ __forceinline__ float ld_weak_f32(const float *p) {
  float v;
  asm volatile("ld.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}
// 16 bytes through the coherent path (rows this CTA wrote in this launch)
__device__ __forceinline__ uint4 ld_global_v4(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int *p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Generic-proxy writes before, async-proxy (TMA) reads after -- or the other
// way round -- of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __noinline__ bool wait_flag(const int *f, volatile int *abort) {
  if (ld_acquire_gpu(f)) return true;
  const uint64_t t0 = global_ns();
  const uint64_t limit = *(volatile unsigned long long *)&g_wait_limit_ns;
  for (;;) {
    __nanosleep(128);
    if (ld_acquire_gpu(f)) return true;
    if (*abort) return false;
    if (global_ns() - t0 >= limit) {
      raise_status(MOE_DEV_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// Inline first try; the bounded slow path only when the phase is not done.
__device__ __forceinline__ bool mbar_wait_fast(uint64_t *bar, uint32_t parity,
                                               volatile int *abort) {
  return mbar_try_wait(bar, parity) || mbar_wait(bar, parity, abort);
}

// The same with acquire at cluster scope: barriers that the other CTA of a
// pair arrives on (release at cluster scope).
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __noinline__ bool mbar_wait_cl(uint64_t *bar, uint32_t parity, volatile int *abort) {
  const uint64_t t0 = global_ns();
  const uint64_t limit = *(volatile unsigned long long *)&g_wait_limit_ns;
  for (;;) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 >= limit) {
      raise_status(MOE_DEV_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait_fast_cl(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort) {
  return mbar_try_wait_cl(bar, parity) || mbar_wait_cl(bar, parity, abort);
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// 3-D box: c0 innermost
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (K-major).  Fields: start address >> 4,
// leading and stride byte offsets >> 4, version 1, swizzle mode in [61,64).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
  return (uint64_t)((saddr >> 4) & 0x3fff) | ((uint64_t)((lbo >> 4) & 0x3fff) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3fff) << 32) | (1ull << 46) | ((uint64_t)swizzle << 61);
}
constexpr uint32_t kSwizzle128B = 2, kSwizzleNone = 0;

// Instruction descriptor of a block-scaled MMA with E8M0 scales, M = 128,
// K-major A and B: a/b formats (mxf8f6f4: 5 = E2M1, 0 = E4M3; mxf4: 1 =
// E2M1), N, and the byte of the scale word each operand's scales start at.
__device__ __forceinline__ uint32_t idesc_block_scaled(uint32_t afmt, uint32_t bfmt, int n,
                                                       uint32_t sf_id, uint32_t m = 128) {
  return (sf_id << 4) | (afmt << 7) | (bfmt << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) |
         ((m >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void mma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate));
}

__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate));
}

__device__ __forceinline__ void tc_cp_32x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ---- CTA pairs (tcgen05 cta_group::2): one M = 256 MMA over two SMs ----
// The even CTA of a cluster of two issues the MMAs; each CTA holds its own
// 128 weight rows, half of the B rows and, in its tensor memory, its rows'
// accumulators (every column) and scale factors (A: its rows; B: all rows).
__device__ __forceinline__ void mma_mxf8f6f4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                  uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate));
}
// completion of the pair's MMAs, signalled on the barrier at the same offset
// in both CTAs
__device__ __forceinline__ void tc_commit_pair_both(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// the same shared-memory variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_rank(const void *p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on the other CTA's barrier.  The default semantics (release at CTA
// scope): the signal only orders this thread's completed tensor-memory
// stores and barrier waits, and a cluster-scope release measured ~0.9 us per
// arrive, stalling the pipeline.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// every thread of both CTAs
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// 32 lanes x 16 columns of 32-bit accumulator -> 16 registers per thread;
// the registers are valid after tc_wait_ld().
__device__ __forceinline__ void tc_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x N columns of 32-bit words from registers (this warp's lane quarter).
__device__ __forceinline__ void tc_st_x4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void tc_st_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Named barrier of one epilogue warp group (ids 1 and 2, 128 threads each);
// constant ids keep the kernel's barrier count small.
__device__ __forceinline__ void group_sync(int grp) {
  if (grp) asm volatile("bar.sync 2, 128;" ::: "memory");
  else asm volatile("bar.sync 1, 128;" ::: "memory");
}

// The same barrier, returning true iff `v` holds on every thread of the
// group: the group's warps take each leave-or-stay decision together, so no
// warp can wait at group_sync for one that has left.
__device__ __forceinline__ bool group_all(int grp, bool v) {
  uint32_t r;
  __syncwarp();
  if (grp)
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, 2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"((uint32_t)v) : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"((uint32_t)v) : "memory");
  return r != 0;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

// ------------------------------------------------ activation block encodings --
//
// The tensor cores take the activations (bf16 x, and GEMM-1's bf16 output h)
// as a short sum of narrow terms, v = sum_t 2^(s_t) * c_t, term t encoding
// what terms 0..t-1 left over.
//  * kind::mxf8f6f4: two E4M3 terms with an E8M0 scale per 32 elements
//    (what is lost is below ~2^-18 of the block's largest element);
//    warp-cooperative, lane l holds element l of one 32-element block.
//  * kind::mxf4: eight E2M1 terms with ONE scale per row and term, chosen
//    from the row's largest remaining magnitude.  The MMA then sees a
//    constant block scale of 1.0 for B (copied to tensor memory once per
//    CTA), and the epilogue multiplies each term's column by its exact power
//    of two.  Each term takes about two more significant bits of the
//    largest remainder, so eight terms give bf16 rows back to ~1e-9
//    relative (all but a few elements in 10^4 exactly), and each term
//    column's fp32 sum over K -- products of E2M1 values and powers of two --
//    rarely rounds: the FFN meets the oracle to ~1e-7.

__device__ __forceinline__ float pow2f(int s) { return __uint_as_float((uint32_t)(127 + s) << 23); }

// E4M3 term: scale exponent with amax / 2^s in [128, 256) (E4M3 max 448).
__device__ __forceinline__ int e4m3_block_exp(float amax) {
  const int be = (int)((__float_as_uint(amax) >> 23) & 0xff);
  const int e = (be == 0 ? -126 : be - 127) - 7;
  return max(-126, min(126, e));
}

// E2M1 term: scale exponent with amax / 2^s in (3, 6] (E2M1 max 6).
__device__ __forceinline__ int e2m1_block_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int be = (int)((b >> 23) & 0xff);
  int e = (be == 0 ? -126 : be - 127) - 2;
  if ((b & 0x7fffffu) > 0x400000u) e += 1;     // mantissa above 1.5: use 2^(e+1)
  return max(-126, min(125, e));
}

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float from_e4m3(uint8_t q) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
  return __half2float(*reinterpret_cast<__half *>(&h));
}
__device__ __forceinline__ uint32_t to_e2m1(float v) {
  return (uint32_t)__nv_cvt_float_to_fp4(v, __NV_E2M1, cudaRoundNearest) & 0xfu;
}

// Largest |v| over the warp: non-negative floats order like their bit
// patterns, so one integer max reduction (redux.sync) replaces a chain of
// five shuffles.
__device__ __forceinline__ float warp_absmax(float v) {
  return __uint_as_float(__reduce_max_sync(FULL, __float_as_uint(fabsf(v))));
}

// Kind of tensor-core MMA used by the FFN (KIND_F4_FUSED: kind::mxf4, both
// GEMMs in one launch -- a host-side choice only; the kernels see KIND_F4).
enum TcKind { KIND_F8 = 0, KIND_F4 = 1, KIND_F4_FUSED = 2, KIND_F8_PAIR = 3 };
constexpr int kF4Terms = 8;     // E2M1 terms per activation row (kind::mxf4)

template <int KIND>
struct TcKindCfg {
  static constexpr int kTerms = KIND == KIND_F4 ? kF4Terms : 2;  // B rows per token
  static constexpr int kStageK = KIND == KIND_F4 ? 256 : 128;   // K elements per stage
  static constexpr int kKGroups = kStageK / 128;                // 4-scale groups per stage
  static constexpr uint32_t kABytes = 128u * kStageK / 2;       // packed weight bytes per stage
  static constexpr int kBRowBytesPerK2 = KIND == KIND_F4 ? 1 : 2;  // B row bytes = K * this / 2
  // Epilogue warp groups (alternating 16-column chunks): two where tiles are
  // wide and the SwiGLU work per tile is large; one for kind::mxf4, whose
  // narrow tiles leave room for the encode kernels' CTAs beside the GEMM CTA.
  static constexpr int kEpiGroups = KIND == KIND_F8 ? 2 : 1;
  static constexpr int kThreads = (8 + 4 * kEpiGroups) * 32;
  static constexpr int kRingReaders = 1 + 1 + 4 * kEpiGroups + 4;
  static constexpr bool kRowScaledB = KIND == KIND_F4;          // B scales per row, not block
};

// Four E4M3 codes (the first in the lowest byte) and back: the paired
// hardware conversions, round to nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xffffu) | ((hi & 0xffffu) << 16);
}
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// One whole 32-element block of an activation row, held by one thread: its
// two E4M3 terms (32 code bytes each, written as two 16-byte stores to q0 and
// q1) and their scale bytes.  Term t takes the scale 2^s with the block's
// largest remaining magnitude / 2^s in [128, 256) (scale byte 127 + s; an
// all-zero block gets 127), codes round to nearest, saturating at +-448, and
// the next term encodes what the codes leave over.
__device__ __forceinline__ void encode_block_f8(float (&v)[32], uint8_t *q0, uint8_t *q1,
                                                uint8_t *s0, uint8_t *s1) {
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    uint32_t mb = 0;
#pragma unroll
    for (int e = 0; e < 32; ++e) mb = max(mb, __float_as_uint(fabsf(v[e])));
    const float amax = __uint_as_float(mb);
    const int s = amax > 0.f ? e4m3_block_exp(amax) : 0;
    const float inv = pow2f(-s), sc = pow2f(s);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i] = e4m3x4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv, v[4 * i + 3] * inv);
      const float2 lo = e4m3x2_to_f32(w[i]), hi = e4m3x2_to_f32(w[i] >> 16);
      v[4 * i] -= lo.x * sc;
      v[4 * i + 1] -= lo.y * sc;
      v[4 * i + 2] -= hi.x * sc;
      v[4 * i + 3] -= hi.y * sc;
    }
    uint4 *q = reinterpret_cast<uint4 *>(t ? q1 : q0);
    q[0] = make_uint4(w[0], w[1], w[2], w[3]);
    q[1] = make_uint4(w[4], w[5], w[6], w[7]);
    *(t ? s1 : s0) = (uint8_t)(127 + s);
  }
}

// kind::mxf8f6f4 activation operand of GEMM-1: for every sorted row r (token
// sp[r]/k) the two E4M3 terms of x[token] as B rows 2r, 2r+1, and their scale
// bytes.  One thread per 32-element block (four 16-byte loads when x is
// 16-byte aligned), its maximum taken over its own values: no warp
// reductions, so the loads of many blocks are in flight at once.
__global__ void __launch_bounds__(256)
split_x_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ sp, int P, int k,
               int H, uint8_t *__restrict__ xq, uint8_t *__restrict__ xs, int *counters) {
  pdl_wait();
  pdl_trigger();
  if (counters && blockIdx.x == 0 && threadIdx.x < 2) counters[threadIdx.x] = 0;
  const int nb = H / 32;
  const long total = (long)P * nb;
  const bool vec = (reinterpret_cast<uintptr_t>(x) & 15) == 0;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total;
       i += (long)gridDim.x * blockDim.x) {
    const int r = (int)(i / nb), b = (int)(i % nb);
    const int t = checked_index(__ldg(sp + r), P) / k;
    const uint16_t *src = x + (size_t)t * H + b * 32;
    float v[32];
    if (vec) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(src) + q);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * q + 2 * j] = bf16_lo(ww[j]);
          v[8 * q + 2 * j + 1] = bf16_hi(ww[j]);
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __uint_as_float((uint32_t)__ldg(src + e) << 16);
    }
    const size_t r2 = 2 * (size_t)r;
    encode_block_f8(v, xq + r2 * H + 32 * b, xq + (r2 + 1) * H + 32 * b, xs + r2 * nb + b,
                    xs + (r2 + 1) * nb + b);
  }
}

// kind::mxf4 activation operand: row r of the source (x[sp[r]/k] when sp is
// given, else src row r) as NT E2M1 terms, B rows NT*r + t (packed, K/2
// bytes each), and the NT per-row scales 2^(s_t) as floats.  One CTA per
// row; each thread keeps its elements (pairs 2i, 2i+1 for i = tid + 256j) in
// registers; K <= 2 * 256 * ENC_MAX_PAIRS.
constexpr int ENC_THREADS = 256;
constexpr int ENC_MAX_PAIRS = 16;

template <int NT>
__global__ void __launch_bounds__(ENC_THREADS)
encode_rows_f4_kernel(const uint16_t *__restrict__ src, const int32_t *__restrict__ sp, int k,
                      int K, uint8_t *__restrict__ q, float *__restrict__ rs, int early_trigger,
                      int *counters, int ncounters) {
  // early_trigger: the next kernel (GEMM-2) may start streaming its weights
  // while this one still waits for GEMM-1; it reads our output only after
  // its own wait, and nothing of GEMM-1's before it
  if (early_trigger) pdl_trigger();
  pdl_wait();
  if (!early_trigger) pdl_trigger();
  // the GEMMs' tile counters for this call, and the fused FFN's B-tile
  // counters and flags (GEMM-1 reads its own only after this kernel
  // completed; GEMM-2 after the next one did)
  if (counters && blockIdx.x == 0)
    for (int i = threadIdx.x; i < ncounters; i += blockDim.x) counters[i] = 0;
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const uint16_t *row =
      src + (size_t)(sp ? checked_index(__ldg(sp + r), gridDim.x) / k : r) * K;
  __shared__ float red[ENC_THREADS / 32];
  const int npairs = K / 2;
  float v[2 * ENC_MAX_PAIRS];
#pragma unroll
  for (int j = 0; j < ENC_MAX_PAIRS; ++j) {
    const int i = tid + ENC_THREADS * j;
    uint32_t pr = 0;
    if (i < npairs) pr = __ldg(reinterpret_cast<const uint32_t *>(row) + i);
    v[2 * j] = bf16_lo(pr);
    v[2 * j + 1] = bf16_hi(pr);
  }
#pragma unroll 1
  for (int t = 0; t < NT; ++t) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 2 * ENC_MAX_PAIRS; ++j) m = fmaxf(m, fabsf(v[j]));
    m = warp_max(m);
    __syncthreads();                       // red[] reuse across terms
    if (lane == 0) red[w] = m;
    __syncthreads();
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < ENC_THREADS / 32; ++i) amax = fmaxf(amax, red[i]);
    const int sexp = amax > 0.f ? e2m1_block_exp(amax) : 0;
    const float inv = pow2f(-sexp), sc = pow2f(sexp);
    uint8_t *qrow = q + (size_t)(NT * r + t) * (K / 2);
#pragma unroll
    for (int j = 0; j < ENC_MAX_PAIRS; ++j) {
      const int i = tid + ENC_THREADS * j;
      const uint32_t c0 = to_e2m1(v[2 * j] * inv), c1 = to_e2m1(v[2 * j + 1] * inv);
      const float2 d = e2m1x2_to_f32x2(c0 | (c1 << 4));
      v[2 * j] -= d.x * sc;
      v[2 * j + 1] -= d.y * sc;
      if (i < npairs) qrow[i] = (uint8_t)(c0 | (c1 << 4));
    }
    if (tid == 0) rs[NT * r + t] = sc;
  }
}

// The same encoding with one warp per row, for rows of K = 64 * PPL <= 2048
// elements (PPL pairs per lane in registers, the row maximum by shuffles, no
// block barrier): four rows per CTA (small CTAs stay resident beside a GEMM
// CTA).  Same outputs as the kernel above.
template <int NT, int PPL>
__global__ void __launch_bounds__(128)
encode_rows_f4_warp_kernel(const uint16_t *__restrict__ src, const int32_t *__restrict__ sp,
                           int k, int P, uint8_t *__restrict__ q, float *__restrict__ rs,
                           int early_trigger, int *counters, int ncounters) {
  if (early_trigger) pdl_trigger();
  pdl_wait();
  if (!early_trigger) pdl_trigger();
  if (counters && blockIdx.x == 0)
    for (int i = threadIdx.x; i < ncounters; i += blockDim.x) counters[i] = 0;
  constexpr int K = 64 * PPL;
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (r >= P) return;
  const uint32_t *row =
      reinterpret_cast<const uint32_t *>(src + (size_t)(sp ? checked_index(__ldg(sp + r), P) / k : r) * K);
  float v[2 * PPL];
#pragma unroll
  for (int j = 0; j < PPL; ++j) {
    const uint32_t pr = __ldg(row + lane + 32 * j);
    v[2 * j] = bf16_lo(pr);
    v[2 * j + 1] = bf16_hi(pr);
  }
#pragma unroll 1
  for (int t = 0; t < NT; ++t) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 2 * PPL; ++j) m = fmaxf(m, fabsf(v[j]));
    const float amax = warp_max(m);
    const int sexp = amax > 0.f ? e2m1_block_exp(amax) : 0;
    const float inv = pow2f(-sexp), sc = pow2f(sexp);
    uint8_t *qrow = q + (size_t)(NT * r + t) * (K / 2);
#pragma unroll
    for (int j = 0; j < PPL; ++j) {
      const uint32_t c0 = to_e2m1(v[2 * j] * inv), c1 = to_e2m1(v[2 * j + 1] * inv);
      const float2 d = e2m1x2_to_f32x2(c0 | (c1 << 4));
      v[2 * j] -= d.x * sc;
      v[2 * j + 1] -= d.y * sc;
      qrow[lane + 32 * j] = (uint8_t)(c0 | (c1 << 4));
    }
    if (lane == 0) rs[NT * r + t] = sc;
  }
}

// The same encoding of one bf16 row of K <= 4096 elements by the 128 threads
// of one epilogue warp group (the fused FFN's last GEMM-1 tile of a B tile
// encodes that tile's h rows).  The row is read through L2 (ld.global.cg):
// other CTAs of the same launch wrote parts of it.  red: 8 floats of shared
// memory (two sets of four, alternating by term).
constexpr int GRP_ENC_MAX_PAIRS = 16;
template <int NT>
__device__ __forceinline__ void encode_row_f4_group(const uint16_t *row, int K, uint8_t *q,
                                                    float *rs, int grp, float *red) {
  const int tid = (threadIdx.x & 127), lane = tid & 31, w = tid >> 5;
  const int npairs = K / 2;
  float v[2 * GRP_ENC_MAX_PAIRS];
#pragma unroll
  for (int j = 0; j < GRP_ENC_MAX_PAIRS; ++j) {
    const int i = tid + 128 * j;
    const uint32_t pr = i < npairs ? __ldcg(reinterpret_cast<const unsigned int *>(row) + i) : 0u;
    v[2 * j] = bf16_lo(pr);
    v[2 * j + 1] = bf16_hi(pr);
  }
#pragma unroll 1
  for (int t = 0; t < NT; ++t) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < 2 * GRP_ENC_MAX_PAIRS; ++j) m = fmaxf(m, fabsf(v[j]));
    m = warp_absmax(m);
    if (lane == 0) red[(t & 1) * 4 + w] = m;
    group_sync(grp);
    const float *rr = red + (t & 1) * 4;
    const float amax = fmaxf(fmaxf(rr[0], rr[1]), fmaxf(rr[2], rr[3]));
    const int sexp = amax > 0.f ? e2m1_block_exp(amax) : 0;
    const float inv = pow2f(-sexp), sc = pow2f(sexp);
    uint8_t *qrow = q + (size_t)t * (K / 2);
#pragma unroll
    for (int j = 0; j < GRP_ENC_MAX_PAIRS; ++j) {
      const int i = tid + 128 * j;
      const uint32_t c0 = to_e2m1(v[2 * j] * inv), c1 = to_e2m1(v[2 * j + 1] * inv);
      const float2 d = e2m1x2_to_f32x2(c0 | (c1 << 4));
      v[2 * j] -= d.x * sc;
      v[2 * j + 1] -= d.y * sc;
      if (i < npairs) qrow[i] = (uint8_t)(c0 | (c1 << 4));
    }
    if (tid == 0) rs[t] = sc;
  }
}

// Launch a row encoder: a CTA per row (shortest latency: a row's work
// spread over 256 threads) for a few rows, a warp per row (no barriers, the
// most rows per SM) once there are hundreds.
constexpr size_t ENC_WARP_MIN_ROWS = 512;
template <int NT>
inline cudaError_t launch_encode_f4(const uint16_t *src, const int32_t *sp, int k, int K,
                                   size_t P, uint8_t *q, float *rs, int early_trigger,
                                   int *counters, int ncounters, cudaStream_t s) {
  const unsigned g4 = (unsigned)((P + 3) / 4);
  switch (P >= ENC_WARP_MIN_ROWS ? K : 0) {
    case 256:
      return launch_pdl(encode_rows_f4_warp_kernel<NT, 4>, g4, 128, 0, s, src, sp, k, (int)P, q,
                        rs, early_trigger, counters, ncounters);
    case 512:
      return launch_pdl(encode_rows_f4_warp_kernel<NT, 8>, g4, 128, 0, s, src, sp, k, (int)P, q,
                        rs, early_trigger, counters, ncounters);
    case 1024:
      return launch_pdl(encode_rows_f4_warp_kernel<NT, 16>, g4, 128, 0, s, src, sp, k, (int)P, q,
                        rs, early_trigger, counters, ncounters);
    case 2048:
      return launch_pdl(encode_rows_f4_warp_kernel<NT, 32>, g4, 128, 0, s, src, sp, k, (int)P, q,
                        rs, early_trigger, counters, ncounters);
    default:
      return launch_pdl(encode_rows_f4_kernel<NT>, (unsigned)P, ENC_THREADS, 0, s, src, sp, k, K,
                        q, rs, early_trigger, counters, ncounters);
  }
}

// ------------------------------------------------------------- the kernel --

struct TcMaps {
  // weights, box 128 (padded E2M1) or 128 B (packed) wide: GEMM-1's [E*2I, K]
  // as [2E][I][K], a box of 64 rows of both halves (gate, then up); GEMM-2's
  // [E*H, K], a box of 128 rows -- one TMA per stage either way
  CUtensorMap a;
  CUtensorMap b[4];     // activation terms [T*P, row bytes]: box 128 B x {16, 32, 64, 128} rows
  // scale bytes in 16-byte groups (TcArgs::sf_tma): weights [E*rows, K/32]
  // (16 B of the same rows as map a); activation terms [T*P, K/32], box 16 B
  // x the B boxes' rows
  CUtensorMap sa;
  CUtensorMap sb[4];
};

struct TcArgs {
  const uint8_t *a_scales;   // [E*rows, K/32]
  const uint8_t *b_scales;   // kind::mxf8f6f4: [T*P, K/32] block scale bytes
  const float *b_rowscale;   // kind::mxf4: [T*P] per-row, per-term scales
  const int32_t *off;        // [E+1]
  int E, K, rows_per_expert, P;
  int I;                     // GEMM-1: the gate/up split
  int H;                     // y row length (GEMM-2)
  int b_box[4];              // rows of each B box (clamped to T*P)
  // GEMM-1 outputs
  uint16_t *h;               // [P, I] bf16
  uint8_t *hq;               // activation terms of h
  uint8_t *hs;               // their scale bytes
  // GEMM-2 output
  float *y;                  // [P, H]
  // tiles past the first wave are handed out by this counter (zeroed by the
  // encode kernel that runs first in the call)
  int *tile_counter;
  // fused FFN: per B tile, GEMM-1 tiles finished and the GEMM-2 operand's
  // readiness flag (zeroed by the same encode kernel)
  int *bt_done;
  int *bt_ready;
  // kind::mxf8f6f4, K % 512 == 0 (16 scale bytes per row cover four
  // stages): the scale bytes come by TMA through maps sa / sb
  int sf_tma;
};

constexpr int kMaxStages = 12;

// PAIR: the stage holds this CTA's half of the B rows (the other CTA of the
// pair holds the other half).
template <int KIND, int BN, int PAIR = 0>
struct TcCfg {
  using Kd = TcKindCfg<KIND>;
  static constexpr int kRowChunks = (BN + 127) / 128;               // 128-row scale chunks of B
  static constexpr int kA = 128 * 128;                              // smem bytes of one A stage
  static constexpr int kB = (PAIR ? BN / 2 : BN) * 128;
  static constexpr int kSfa = 512 * Kd::kKGroups;
  static constexpr int kSfb = Kd::kRowScaledB ? 0 : 512 * Kd::kKGroups * kRowChunks;
  static constexpr int kSfbConst = Kd::kRowScaledB ? 512 * kRowChunks : 0;  // all 1.0
  // kind::mxf8f6f4: the scale bytes have a ring of their own, refilled as
  // soon as the writer warps have moved a slot into tensor memory (not when
  // the MMAs release the stage), so the scale loads run that much further
  // ahead; sized to leave the operand stages as many as before.  Else one
  // scale slot per operand stage.
  static constexpr int kSfRing = KIND == KIND_F8 ? (PAIR ? 8 : 4) : 0;
  // With TcArgs::sf_tma (kind::mxf8f6f4) the scale bytes come instead in
  // groups of kSfGroup stages (16 bytes of each A and B row) by TMA, into one
  // of kSftSlots slots of [128 A rows][16] then [BN B rows][16] bytes.
  static constexpr int kSfGroup = 16 / (4 * Kd::kKGroups);
  static constexpr int kSftA = 128 * 16;               // A part of a slot; the B part follows
  static constexpr int kSft = KIND == KIND_F8 ? kSftA + 16 * BN : 0;   // all B rows (PAIR too)
  static constexpr int kSftSlots = 2;
  static constexpr int kRingBytes =
      !kSfRing ? 0
               : (kSfRing * (kSfa + kSfb) > kSftSlots * kSft ? kSfRing * (kSfa + kSfb)
                                                              : kSftSlots * kSft);
  static constexpr int kStageBytes = kA + kB + (kSfRing ? 0 : kSfa + kSfb);
  static constexpr int kFixed = 1024 + Kd::kEpiGroups * 64 * (16 / Kd::kTerms) * 4 + 1026 * 2 +
                                 2 * 1025 * 4 + 128 + 1024 + kSfbConst;
  static constexpr int kStages0 = (227 * 1024 - kFixed - kRingBytes) / kStageBytes;
  static constexpr int kStages = kStages0 > kMaxStages ? kMaxStages : kStages0;
  static constexpr int kSfSlots = kSfRing ? kSfRing : kStages;
  static constexpr int kSfCols =                                    // TMEM columns per stage
      4 * Kd::kKGroups * (Kd::kRowScaledB ? 1 : 1 + kRowChunks);
  // Independent accumulation chains per buffer: with few B columns each MMA
  // is tiny and a single chain would run at MMA latency; MMA kk of a stage
  // accumulates into chain kk % kChains and the epilogue adds the chains.
  static constexpr int kChains = BN <= 32 ? 4 : BN <= 64 ? 2 : 1;
  static constexpr int kSfbConstCols = Kd::kRowScaledB ? 4 * kRowChunks : 0;
  // Two accumulator buffers (the epilogue drains one while the MMAs fill the
  // other) wherever tensor memory holds them beside the scale columns.
  static constexpr int kAcc =
      2 * kChains * BN + kStages * kSfCols + kSfbConstCols <= 512 ? 2 : 1;
  static constexpr int kAccCols = kAcc * kChains * BN;
  static constexpr int kUsed = kAccCols + kStages * kSfCols + kSfbConstCols;
  static constexpr int kTmemCols = kUsed <= 128 ? 128 : kUsed <= 256 ? 256 : 512;
  static_assert(kUsed <= 512, "TMEM budget");
  static constexpr int kOffB = kStages * kA;
  static constexpr int kOffSfa = kOffB + kStages * kB;
  static constexpr int kOffSfb = kOffSfa + kSfSlots * kSfa;
  static constexpr int kOffBar = kSfRing ? kOffSfa + kRingBytes : kOffSfb + kSfSlots * kSfb;
  // SwiGLU exchange: 64 rows x (tokens per 16-column chunk) floats per
  // epilogue warp group
  static constexpr int kXchgFloats = 64 * (16 / Kd::kTerms);
  static constexpr int kOffXchg = kOffBar + 1024;
  static constexpr int kOffTab = kOffXchg + Kd::kEpiGroups * kXchgFloats * 4;  // tile table
  // tile table: expert ids (16-bit), tile prefix and first sorted row (32-bit)
  static constexpr int kTabBytes = 1026 * 2 + 2 * 1025 * 4;
  static constexpr int kOffSfbConst = (kOffTab + kTabBytes + 127) & ~127;  // 16B-aligned for tcgen05.cp
  static constexpr int kSmem = kOffSfbConst + kSfbConst + 1024;   // + alignment slack
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kOffSfa % 1024 == 0 && kOffSfb % 128 == 0 && kOffSfbConst % 128 == 0 &&
                    kSft % 128 == 0,
                "descriptor and TMA destination alignment");
};

// B rows of a tile (N = ncol, a multiple of 16): one box of 16, 32, 64 or
// 128 rows, or a 128-row box and a second one for the rest.  Box class
// (0..3) | (class of the second box + 1) << 3.
__device__ __forceinline__ int b_box_class(int n) { return n <= 16 ? 0 : n <= 32 ? 1 : n <= 64 ? 2 : 3; }
__device__ __forceinline__ int b_box_sel(int ncol) {
  return ncol <= 128 ? b_box_class(ncol) : 3 | ((b_box_class(ncol - 128) + 1) << 3);
}

// warps: 0 TMA producer, 1 scale loader, 2 TMEM + MMA issuer, 3 constant B
// scales, 4-7 epilogue, 8-11 scale writers (one per TMEM lane quarter),
// 12-15 second epilogue group (kind::mxf8f6f4)
constexpr int kRing = 4;                        // tile indices published ahead

// Reader side of the tile ring: tile i of this CTA's sequence (all lanes of
// the calling warp wait; `arrive` is the one lane that releases the slot).
__device__ __forceinline__ int ring_read(uint64_t *ring_full, uint64_t *ring_empty,
                                         volatile int *ring, int i, bool arrive,
                                         volatile int *abort, int sentinel) {
  const int slot = i % kRing;
  if (!mbar_wait_fast(&ring_full[slot], (uint32_t)(i / kRing) & 1u, abort)) return sentinel;
  const int t = ring[slot];
  __syncwarp(__activemask());
  if (arrive) mbar_arrive(&ring_empty[slot]);
  return t;
}

// MODE 1: GEMM-1 + SwiGLU (maps, a); MODE 2: GEMM-2 (maps, a); MODE 3: the
// fused FFN, one launch over every GEMM-1 tile (maps, a) and then every
// GEMM-2 tile (maps2, a2) -- phase 0 and phase 1 of the tile sequence.  The
// last GEMM-1 tile of a B tile (the rows of one expert in one B-tile slot)
// encodes those h rows into the GEMM-2 operand and raises the B tile's
// readiness flag; a GEMM-2 tile's producer waits for the flag (bounded)
// before loading its B operand.  Every CTA is resident at once (one per SM)
// and tiles are taken in increasing order, so every GEMM-1 tile a waiting
// GEMM-2 tile needs is held by a running CTA.
// Register budget: the compiler's own choice for the two GEMMs (no
// minimum-blocks hint, which let it take up to 168); at most 136 for the
// fused launch, so that the x encoder's CTAs (256 threads x 48 registers)
// stay resident beside a GEMM CTA under programmatic dependent launch.
// PAIR (kind::mxf8f6f4, MODES 1 and 2): clusters of two CTAs, each tile two
// m-blocks of one B tile -- rank r of the pair takes m-block 2m + r and half
// of the B rows; the even CTA issues M = 256 MMAs (cta_group::2) over both.
// Each CTA's own loads complete on its own full barrier; its scale writers
// then tell the even CTA (ready), whose MMAs release both CTAs' stages and
// accumulators with multicast commits.  Tiles are dealt out statically, pair
// p taking p, p + pairs, ...
template <int KIND, int MODE, int BN, int PAIR = 0>
__global__ void __launch_bounds__(TcKindCfg<KIND>::kThreads) __maxnreg__(MODE == 3 ? 136 : 168)
tc_gemm_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ TcArgs a,
               const __grid_constant__ TcMaps maps2, const __grid_constant__ TcArgs a2) {
  static_assert(!PAIR || (KIND == KIND_F8 && MODE != 3 && BN >= 64), "CTA pairs: mxf8f6f4 GEMMs");
  using C = TcCfg<KIND, BN, PAIR>;
  using Kd = TcKindCfg<KIND>;
  constexpr int T = Kd::kTerms;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *empty = full + C::kStages;
  uint64_t *acc_full = empty + C::kStages;     // [2]
  uint64_t *acc_empty = acc_full + 2;          // [2]
  volatile int *abort = reinterpret_cast<volatile int *>(acc_empty + 2);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 3);
  uint64_t *sfs_full = acc_empty + 4;          // [kSfSlots] scale bytes landed in smem
  // tile ring: the producer publishes each tile index it takes; every other
  // role reads the same sequence
  uint64_t *ring_full = sfs_full + C::kSfSlots;  // [kRing]
  uint64_t *ring_empty = ring_full + kRing;     // [kRing]
  volatile int *ring = reinterpret_cast<volatile int *>(ring_empty + kRing);   // [kRing]
  // end of the kernel: the MMA thread's last commit, and the number of
  // stages the producer issued (the abort path drains them)
  uint64_t *drain_bar = ring_empty + kRing + 2;
  volatile int *s_issued = reinterpret_cast<volatile int *>(drain_bar + 1);
  // PAIR, even CTA: a stage's operands and scale factors are in place in
  // both CTAs (the 4 + 4 scale-writer warps)
  uint64_t *ready = drain_bar + 2;              // [kStages]
  // kSfRing: a scale slot moved to tensor memory (4 writer warps)
  uint64_t *sfs_empty = ready + C::kStages;     // [kSfSlots]
  static_assert(8 * (3 * C::kStages + 2 * C::kSfSlots + 2 * kRing + 10) <= 960, "barrier region");
  float *xchg = reinterpret_cast<float *>(smem + C::kOffXchg);
  // The table stays small: a GEMM CTA leaves a few KB of the SM's shared
  // memory free, so that the encode kernels' CTAs can become resident beside
  // it under programmatic dependent launch.
  uint16_t *s_act = reinterpret_cast<uint16_t *>(smem + C::kOffTab);   // [1025] (+ count)
  int *s_pre = reinterpret_cast<int *>(smem + C::kOffTab + 1026 * 2);   // tile prefix
  int *s_r0 = s_pre + 1025;        // first sorted row of each active expert (+ total)

  // the fused FFN's encode scratch: the last-tile flag and the row maxima
  volatile int *s_last = reinterpret_cast<volatile int *>(smem + C::kOffBar + 960);
  float *s_red = reinterpret_cast<float *>(smem + C::kOffBar + 960 + 16);   // [8]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t crank = PAIR ? cluster_rank() : 0u;   // rank in the pair
  const bool leader = crank == 0;
  const int pair_id = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // m-blocks of a B tile and K stages, per phase (phase 1: MODE 3 only)
  const int mt1 = MODE == 2 ? a.rows_per_expert / 128 : a.I / 64;
  const int mt2 = a2.rows_per_expert / 128;
  const int ks1 = a.K / Kd::kStageK, ks2 = a2.K / Kd::kStageK;
  // the table's prefix is in tiles (MODES 1, 2; PAIR: tiles of two
  // m-blocks) or in B tiles (MODE 3)
  const int mtiles = MODE == 3 ? 1 : PAIR ? mt1 / 2 : mt1;
  // scale bytes by TMA in 16-byte groups (kind::mxf8f6f4)
  const bool sft = KIND == KIND_F8 && MODE != 3 && a.sf_tma != 0;
  const int n_sfslots = sft ? C::kSftSlots : C::kSfSlots;

  // tile table: active experts and the prefix of their tile counts (none
  // where the checked build finds the offsets bad)
  if (warp == 0) {
    int n = 0, acc = 0;
    const int n_e = offsets_ok(a.off, a.E, a.P) ? a.E : 0;
    for (int e0 = 0; e0 < n_e; e0 += 32) {
      const int e = e0 + lane;
      const int r0 = e < n_e ? __ldg(a.off + e) : 0;
      const int cnt = e < n_e ? __ldg(a.off + e + 1) - r0 : 0;
      const int nt = cnt > 0 ? (T * cnt + BN - 1) / BN : 0;
      const unsigned b = __ballot_sync(FULL, nt > 0);
      int sc = nt * mtiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, sc, o);
        if (lane >= o) sc += y;
      }
      if (nt > 0) {
        const int pos = n + __popc(b & lanemask_lt());
        s_act[pos] = (uint16_t)e;
        s_pre[pos] = acc + sc - nt * mtiles;   // exclusive
        s_r0[pos] = r0;
      }
      n += __popc(b);
      acc += __shfl_sync(FULL, sc, 31);
    }
    if (lane == 0) {
      s_act[1024] = (uint16_t)n;
      s_pre[n] = acc;
      s_r0[n] = n_e ? __ldg(a.off + a.E) : 0;   // rows of inactive experts are empty: the next
                                       // active expert's first row ends the previous one
    }
  } else if (warp == 1 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // producer expect_tx + 4 A-scale writer warps (PAIR: the producer's
      // expect_tx alone; the writers report to the even CTA's ready)
      mbar_init(&full[s], PAIR ? 1 : 1 + 4);
      mbar_init(&empty[s], 1);         // MMA commit
      if (PAIR) mbar_init(&ready[s], 8);
    }
    for (int s = 0; s < C::kSfSlots; ++s) {
      mbar_init(&sfs_full[s], sft ? 1 : 32);   // the loader's expect_tx, or 32 cp.async lanes
      if (C::kSfRing) mbar_init(&sfs_empty[s], 4);   // 4 scale-writer warps
    }
    for (int r = 0; r < kRing; ++r) {
      mbar_init(&ring_full[r], 1);             // producer
      mbar_init(&ring_empty[r], Kd::kRingReaders); // scale loader, MMA, epilogue, 4 writers
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      // one arrival per epilogue warp (PAIR: of both CTAs)
      mbar_init(&acc_empty[b], (PAIR ? 8 : 4) * Kd::kEpiGroups);
    }
    mbar_init(drain_bar, 1);           // the MMA thread's final commit
    *abort = 0;
    *s_issued = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  } else if (warp == 2) {
    if (PAIR) {
      // both CTAs' warp 2: the same columns in each CTA's tensor memory
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(C::kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  if (Kd::kRowScaledB && warp == 3) {
    // constant B block scales (byte 127 = 1.0), copied to tensor memory once
    uint32_t *cst = reinterpret_cast<uint32_t *>(smem + C::kOffSfbConst);
    for (int i = lane; i < C::kSfbConst / 4; i += 32) cst[i] = 0x7f7f7f7fu;
    fence_proxy_async();
  }
  tc_fence_before();
  __syncthreads();
  // a pair's barriers are initialised before either CTA signals the other's
  if (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_act = s_act[1024];
  const int n_bt = s_pre[n_act];
  const int n1 = MODE == 3 ? n_bt * mt1 : n_bt;          // tiles of phase 0
  const int n_tiles = MODE == 3 ? n1 + n_bt * mt2 : n_bt;
  auto phase_of = [&](int t) { return (MODE == 3 && t >= n1) ? 1 : 0; };
  auto mode_of = [&](int ph) { return MODE == 3 ? 1 + ph : MODE; };
  auto ksteps_of = [&](int ph) { return ph ? ks2 : ks1; };

  // tile index -> (expert, m-block, first B row, B rows in the tile, phase,
  // global B-tile index).  Every role walks its tiles in increasing order,
  // so within a phase the active-expert index only moves forward: a linear
  // advance from the last position, all from shared memory.
  struct Tile {
    int e, mt, rowB, nB, ph, g;
  };
  int dpos = 0, dph = 0;
  auto decode = [&](int t) {
    Tile r;
    r.ph = phase_of(t);
    const int tl = r.ph ? t - n1 : t;
    const int mtl = MODE == 3 ? (r.ph ? mt2 : mt1) : 1;
    if (r.ph != dph) {
      dpos = 0;
      dph = r.ph;
    }
    int lo = dpos;
    while (lo + 1 < n_act && s_pre[lo + 1] * mtl <= tl) ++lo;
    dpos = lo;
    r.e = s_act[lo];
    const int r0 = s_r0[lo];
    const int ne = s_r0[lo + 1] - r0;
    const int nt_cnt = (T * ne + BN - 1) / BN;
    const int local = tl - s_pre[lo] * mtl;
    r.mt = PAIR ? 2 * (local / nt_cnt) + (int)crank : local / nt_cnt;
    const int nt = local % nt_cnt;
    r.g = s_pre[lo] + nt;
    r.rowB = T * r0 + nt * BN;
    r.nB = min(BN, T * ne - nt * BN);
    return r;
  };

  int w_arrived = 0;   // stages an A-scale writer warp has released (abort drain)
  int l_signaled = 0;  // stages the scale loader has signalled (abort drain)
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer --
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      // B rows of a tile: b_box_sel's boxes, so a stage loads at most 15
      // rows more than the tile's N.  PAIR: N rounded up to 32, this CTA's
      // half (a multiple of 16 rows) in one box of up to 64 rows or a 64-row
      // box and a second one.
      auto tile_geom = [&](int t, int &ac1, int &ac2, int &rowB, int &bsel, int &ph, int &g) {
        const Tile tl = decode(t);
        if (PAIR) {
          const int half = ((tl.nB + 31) & ~31) / 2;
          bsel = half <= 64 ? b_box_class(half) : 2 | ((b_box_class(half - 64) + 1) << 3);
          rowB = tl.rowB + (int)crank * half;
        } else {
          bsel = b_box_sel((tl.nB + 15) & ~15);
          rowB = tl.rowB;
        }
        ph = tl.ph;
        g = tl.g;
        const int rpe = ph ? a2.rows_per_expert : a.rows_per_expert;
        // the weight box: GEMM-1 rows m*64.. of halves 2e, 2e + 1; GEMM-2 rows
        // e*H + m*128..
        ac1 = mode_of(ph) == 1 ? tl.mt * 64 : tl.e * rpe + tl.mt * 128;
        ac2 = 2 * tl.e;
      };
      auto b_bytes = [&](int bsel) {
        const int tail = bsel >> 3;
        return (uint32_t)(a.b_box[bsel & 7] + (tail ? a.b_box[tail - 1] : 0)) * 128u;
      };
      // the box's inner coordinate is in elements (padded E2M1) or bytes
      // (packed E2M1); both are kt * 128.  One box of the tile's 128 rows
      // (GEMM-1: 64 gate rows, then 64 up rows)
      auto load_a = [&](int st, int ac1, int ac2, int kt, int ph) {
        uint8_t *sa = smem + st * C::kA;
        const CUtensorMap *m = ph ? &maps2.a : &maps.a;
        if (mode_of(ph) == 1)
          tma_load_3d(sa, m, kt * 128, ac1, ac2, &full[st], pol_w);
        else
          tma_load_2d(sa, m, kt * 128, ac1, &full[st], pol_w);
      };
      auto load_b = [&](int st, int bsel, int rowB, int kt, int ph) {
        uint8_t *sb = smem + C::kOffB + st * C::kB;
        const CUtensorMap *mb = ph ? maps2.b : maps.b;
        constexpr int kFirst = PAIR ? 64 : 128;   // rows of the first box when there are two
        tma_load_2d(sb, &mb[bsel & 7], kt * 128, rowB, &full[st], pol_x);
        if (bsel >> 3)
          tma_load_2d(sb + kFirst * 128, &mb[(bsel >> 3) - 1], kt * 128, rowB + kFirst, &full[st],
                      pol_x);
      };
      // a GEMM-2 tile of the fused FFN: its B operand (h rows encoded by the
      // last GEMM-1 tile of the same B tile) is published by a flag.  On a
      // failed wait the loads still go out (the kernel is aborting; what they
      // read does not matter, and every expect_tx gets its bytes).
      auto b_ready = [&](int ph, int g) {
        if (MODE != 3 || !ph) return true;
        const bool ok = wait_flag(a.bt_ready + g, abort);
        fence_proxy_async_global();
        return ok;
      };
      // Tile sequence: blockIdx.x first, then gridDim.x + (the counter's next
      // value) -- a CTA whose tiles went fast takes more (PAIR: pair p takes
      // p, p + pairs, ..., the same in both CTAs).  Each index is published
      // into the ring as soon as it is known.
      int published = 0;
      auto publish = [&](int t) {
        const int slot = published % kRing;
        if (published >= kRing &&
            !mbar_wait_fast(&ring_empty[slot], (uint32_t)(published / kRing - 1) & 1u, abort))
          return false;
        ring[slot] = t;
        mbar_arrive(&ring_full[slot]);        // release: the index is visible
        ++published;
        return true;
      };
      publish(pair_id);
      // Weights depend on no earlier kernel: the first tile's leading stages
      // of A stream in before the wait for the activation operand.
      int npre = 0;
      if (pair_id < n_tiles) {
        int ac1, ac2, rowB, bsel, ph, g;
        tile_geom(pair_id, ac1, ac2, rowB, bsel, ph, g);
        npre = min(C::kStages, ksteps_of(ph));
        for (int kt = 0; kt < npre; ++kt) {
          mbar_expect_tx(&full[kt], Kd::kABytes + b_bytes(bsel));
          load_a(kt, ac1, ac2, kt, ph);
        }
        pdl_wait();
        pdl_trigger();
        b_ready(ph, g);
        for (int kt = 0; kt < npre; ++kt) load_b(kt, bsel, rowB, kt, ph);
        issued = npre;
        stage = npre % C::kStages;
        phase = npre == C::kStages ? 1u : 0u;
      } else {
        pdl_wait();
        pdl_trigger();
      }
      for (int t = pair_id; t < n_tiles && !*abort;) {
        // the next tile, published before this one's stages are issued
        const int t_next = PAIR ? t + n_units : n_units + atomicAdd(a.tile_counter, 1);
        if (!publish(t_next < n_tiles ? t_next : n_tiles)) break;
        int ac1, ac2, rowB, bsel, ph, g;
        tile_geom(t, ac1, ac2, rowB, bsel, ph, g);
        const uint32_t bbytes = b_bytes(bsel);
        if (t != pair_id && !b_ready(ph, g)) break;
        const int ksteps = ksteps_of(ph);
        for (int kt = t == pair_id ? npre : 0; kt < ksteps; ++kt) {
          if (!mbar_wait_fast(&empty[stage], phase ^ 1, abort)) break;
          mbar_expect_tx(&full[stage], Kd::kABytes + bbytes);
          load_a(stage, ac1, ac2, kt, ph);
          load_b(stage, bsel, rowB, kt, ph);
          ++issued;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        t = t_next;
      }
      if (*abort) publish(n_tiles);            // release readers still waiting
      *s_issued = issued;                      // read after the role loops end
    }
  } else if (warp == 1) {
    // --------------------------------------------------- scale loader --
    // cp.async path: per stage and 4-scale group g, the scale bytes of the
    // 128 A rows (and of the B rows) go straight into the 32 x 16-byte layout
    // of the scale-factor columns: byte 16*(row%32) + 4*(row/32) + (k-block
    // within the group).
    if (!Kd::kRowScaledB) pdl_wait();        // B block scales come from the previous kernel
    if (sft) {
      // 16 bytes of every A row and B row of the tile -- the scale bytes of
      // kSfGroup stages -- per TMA group: the weight tile's 128 rows, then the
      // B tile's boxes, into a slot of [row][16] bytes.  A row's
      // later groups read the rest of the line its first group brought into
      // L2, so the weight scales are not marked evict-first as the weights
      // are.  The writer warps free a slot as soon as they have read it, at
      // the group's first stage.
      const uint64_t pol_w = policy_evict_normal(), pol_x = policy_evict_last();
      int slot = 0;
      uint32_t sph = 0;
      bool ok = true;
      for (int ti = 0; ok; ++ti) {
        const int t = ring_read(ring_full, ring_empty, ring, ti, lane == 0, abort, n_tiles);
        if (!__all_sync(FULL, t < n_tiles && !*abort)) break;
        const Tile tl = decode(t);
        const TcArgs &ap = tl.ph ? a2 : a;       // this phase's operands
        const TcMaps &mp = tl.ph ? maps2 : maps;
        const bool m1 = mode_of(tl.ph) == 1;
        const int arow = m1 ? tl.mt * 64 : tl.e * ap.rows_per_expert + tl.mt * 128;
        const int bsel = b_box_sel((tl.nB + 15) & ~15);
        const int tail = bsel >> 3;
        const uint32_t bytes =
            (uint32_t)(C::kSftA + 16 * (a.b_box[bsel & 7] + (tail ? a.b_box[tail - 1] : 0)));
        const int groups = ksteps_of(tl.ph) / C::kSfGroup;
        for (int gi = 0; gi < groups; ++gi) {
          if (!__all_sync(FULL, mbar_wait_fast(&sfs_empty[slot], sph ^ 1, abort))) {
            ok = false;
            break;
          }
          if (lane == 0) {
            uint8_t *dst = smem + C::kOffSfa + slot * C::kSft;
            mbar_expect_tx(&sfs_full[slot], bytes);
            if (m1)   // the weight tile's rows, as map a: 64 gate, then 64 up
              tma_load_3d(dst, &mp.sa, 16 * gi, arow, 2 * tl.e, &sfs_full[slot], pol_w);
            else
              tma_load_2d(dst, &mp.sa, 16 * gi, arow, &sfs_full[slot], pol_w);
            tma_load_2d(dst + C::kSftA, &mp.sb[bsel & 7], 16 * gi, tl.rowB, &sfs_full[slot],
                        pol_x);
            if (tail)
              tma_load_2d(dst + C::kSftA + 128 * 16, &mp.sb[tail - 1], 16 * gi, tl.rowB + 128,
                          &sfs_full[slot], pol_x);
          }
          ++l_signaled;
          if (++slot == C::kSftSlots) { slot = 0; sph ^= 1; }
        }
      }
    } else {
      // Leave-or-stay decisions are warp-wide, so that every stage this warp
      // signals gets all 32 lanes' arrivals.
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int ti = 0; ok; ++ti) {
        const int t = ring_read(ring_full, ring_empty, ring, ti, lane == 0, abort, n_tiles);
        if (!__all_sync(FULL, t < n_tiles && !*abort)) break;
        const Tile tl = decode(t);
        const int mt = tl.mt, rowB = tl.rowB, nB = tl.nB;
        const TcArgs &ap = tl.ph ? a2 : a;       // this phase's operands
        const uint32_t kb = ap.K / 32;           // scale bytes per row
        const int ebase = tl.e * ap.rows_per_expert;
        // this lane's four A rows (lane + 32q) for the whole tile
        const uint8_t *src_a[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = lane + 32 * q;
          const int row = mode_of(tl.ph) == 1
                              ? ebase + (i < 64 ? mt * 64 + i : a.I + mt * 64 + i - 64)
                              : ebase + mt * 128 + i;
          src_a[q] = ap.a_scales + (size_t)row * kb;
        }
        const int ksteps = ksteps_of(tl.ph);
        for (int kt = 0; kt < ksteps; ++kt) {
          // the slot is free: its last bytes are in tensor memory (kSfRing), or
          // the MMAs that read its stage's columns are done
          if (!__all_sync(FULL, C::kSfRing ? mbar_wait_fast(&sfs_empty[stage], phase ^ 1, abort)
                                           : mbar_wait_fast(&empty[stage], phase ^ 1, abort))) {
            ok = false;
            break;
          }
          uint8_t *sfa = smem + C::kOffSfa + stage * C::kSfa;
          uint8_t *sfb = smem + C::kOffSfb + stage * C::kSfb;
#pragma unroll
          for (int g = 0; g < Kd::kKGroups; ++g) {
            const uint32_t koff = (uint32_t)(kt * Kd::kKGroups + g) * 4;
#pragma unroll
            for (int q = 0; q < 4; ++q)         // A rows lane + 32q
              cp_async4(sfa + 512 * g + 16 * lane + 4 * q, src_a[q] + koff);
#pragma unroll
            for (int q = 0; q < 4 * C::kRowChunks; ++q) {
              const int i = lane + 32 * q;
              if (!Kd::kRowScaledB && i < nB)
                cp_async4(sfb + 512 * (g * C::kRowChunks + (q >> 2)) + 16 * lane + 4 * (q & 3),
                          ap.b_scales + (size_t)(rowB + i) * kb + koff);
            }
          }
          cp_async_arrive_noinc(&sfs_full[stage]);
          ++l_signaled;
          if (++stage == C::kSfSlots) { stage = 0; phase ^= 1; }
        }
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
  } else if (warp == 2) {
    // ----------------------------------------------------- MMA issuer --
    if (PAIR && !leader && lane == 0) {
      // the odd CTA of a pair issues no MMAs; it only takes its turn in the
      // tile ring
      for (int it = 0;; ++it) {
        const int t = ring_read(ring_full, ring_empty, ring, it, true, abort, n_tiles);
        if (t >= n_tiles || *abort) break;
      }
    } else if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t sf_col0 = (uint32_t)C::kAccCols;
      const uint32_t sfb_const_t = tmem + sf_col0 + C::kStages * C::kSfCols;
      if (Kd::kRowScaledB) {
#pragma unroll
        for (int c = 0; c < C::kRowChunks; ++c)
          tc_cp_32x128b(sfb_const_t + 4 * c,
                        smem_desc(smem_u32(smem + C::kOffSfbConst + 512 * c), 0, 128,
                                  kSwizzleNone));
      }
      // Descriptors of stage 0.  A stage's operands, and each MMA's K slice,
      // sit at fixed byte offsets from these, and the start-address field
      // (address >> 4, 14 bits; shared memory is below 256 KB) takes such an
      // offset by plain addition -- the single issuing thread does little
      // more per MMA than the instruction itself.
      const uint64_t a_desc0 = smem_desc(smem_u32(smem), 16, 1024, kSwizzle128B);
      const uint64_t b_desc0 = smem_desc(smem_u32(smem + C::kOffB), 16, 1024, kSwizzle128B);
      int it = 0;
      for (int t = ring_read(ring_full, ring_empty, ring, it, true, abort, n_tiles);
           t < n_tiles && !*abort; t = ring_read(ring_full, ring_empty, ring, ++it, true, abort, n_tiles)) {
        const Tile tl = decode(t);
        const int ncol = PAIR ? (tl.nB + 31) & ~31 : (tl.nB + 15) & ~15;
        const int ksteps = ksteps_of(tl.ph);
        // the tile's instruction descriptor; MMA kk or-s in its scale byte
        // selector (sf_id, bits 4-5 and 29-30)
        const uint32_t idesc0 = KIND == KIND_F4 ? idesc_block_scaled(1, 1, ncol, 0)
                                                : idesc_block_scaled(5, 0, ncol, 0, PAIR ? 256 : 128);
        const int buf = it % C::kAcc;
        const uint32_t use = (uint32_t)(it / C::kAcc);
        if (!(PAIR ? mbar_wait_fast_cl(&acc_empty[buf], (use & 1) ^ 1, abort)
                   : mbar_wait_fast(&acc_empty[buf], (use & 1) ^ 1, abort)))
          break;
        tc_fence_after();
        const uint32_t acc_t = tmem + (uint32_t)(buf * C::kChains * BN);
        bool ok = true;
        for (int kt = 0; kt < ksteps; ++kt) {
          if (!(PAIR ? mbar_wait_fast_cl(&ready[stage], phase, abort)
                     : mbar_wait_fast(&full[stage], phase, abort))) {
            ok = false;
            break;
          }
          // The full barrier completes once the stage's TMA bytes have landed
          // and the writer warps have stored its scale factors into tensor
          // memory (tcgen05.wait::st + fence before their arrive); PAIR: the
          // ready barrier, once the writer warps of both CTAs have seen their
          // CTA's bytes land and stored its scale factors.
          tc_fence_after();
          // TMEM: per stage, the A scale groups then, per group, the B row
          // chunks (all written by the scale-writer warps)
          const uint32_t sfa_t = tmem + sf_col0 + stage * C::kSfCols;
          const uint32_t sfb_t = sfa_t + 4 * Kd::kKGroups;
          const uint64_t ad = a_desc0 + (uint64_t)((stage * C::kA) >> 4);
          const uint64_t bd = b_desc0 + (uint64_t)((stage * C::kB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // 32 bytes of each 128-byte row per MMA (K = 32 E4M3/E2M1-padded or
            // 64 E2M1): descriptor offset 2 (units of 16 bytes)
            const uint32_t acc = (kt > 0 || kk >= C::kChains) ? 1u : 0u;
            const uint32_t d_t = acc_t + (uint32_t)((kk % C::kChains) * BN);
            if (KIND == KIND_F4) {
              const int g = kk >> 1;                     // scale group of this MMA
              const uint32_t sfid = 2u * (kk & 1);      // two scale bytes per row
              mma_mxf4(d_t, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk),
                       idesc0 | (sfid << 4) | (sfid << 29), (sfa_t + 4 * g) | (sfid << 30),
                       sfb_const_t | (sfid << 30), acc);
            } else {
              const uint32_t sfid = (uint32_t)kk;
              if (PAIR)
                mma_mxf8f6f4_pair(d_t, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk),
                                  idesc0 | (sfid << 4) | (sfid << 29), sfa_t | (sfid << 30),
                                  sfb_t | (sfid << 30), acc);
              else
                mma_mxf8f6f4(d_t, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk),
                             idesc0 | (sfid << 4) | (sfid << 29), sfa_t | (sfid << 30),
                             sfb_t | (sfid << 30), acc);
            }
          }
          if (PAIR) tc_commit_pair_both(&empty[stage]); else tc_commit(&empty[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (PAIR) tc_commit_pair_both(&acc_full[buf]); else tc_commit(&acc_full[buf]);
      }
      // Every MMA and tensor-memory copy this thread issued completes before
      // the CTA frees its tensor memory, on every exit path: one more commit
      // tracks them all.  (On the normal path the epilogue has waited for the
      // last tile already, so this costs nothing.)
      if (PAIR) tc_commit_pair(drain_bar); else tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else if (warp >= 8 && warp < 12) {
    // --------------------------------------------------- scale writers --
    // Warp 8+q stores lane quarter q of every stage's scale-factor columns
    // with tcgen05.st (the scale-factor layout repeats the same 32 lanes in
    // all four quarters), keeping the copies off the MMA issue path: the A
    // (weight) scales and, for kind::mxf8f6f4, the B block scales.  Column
    // 4g + j, lane l = the 4 scale bytes of tile row 32j + l, K-group g: the
    // 16 bytes the scale loader put at 512g + 16l.
    // Each leave-or-stay decision is taken by the whole warp (__all_sync):
    // tcgen05.st and tcgen05.wait::st need all 32 lanes.
    const int q = warp - 8;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int stage = 0;
    uint32_t phase = 0;
    int slot = 0;          // scale slot (the stage itself unless kSfRing)
    uint32_t sph = 0;
    int sub = 0;           // sft: the stage's place in its group
    // sft: the group's 16 bytes of this lane's A rows (32j + lane) and B rows
    // (128c + 32j + lane), taken out of the slot at the group's first stage
    // so that the loader can refill it at once; .x is the current stage's
    uint4 ga[4], gb[C::kRowChunks][4];
    bool ok = true;
    for (int ti = 0; ok; ++ti) {
      const int t = ring_read(ring_full, ring_empty, ring, ti, lane == 0, abort, n_tiles);
      if (!__all_sync(FULL, t < n_tiles && !*abort)) break;
      const int ksteps = ksteps_of(phase_of(t));
      for (int kt = 0; kt < ksteps; ++kt) {
        // the MMAs that read this stage's columns last time are done, and the
        // stage's scale bytes are in shared memory
        const bool rdy = mbar_wait_fast(&empty[stage], phase ^ 1, abort) &&
                         ((sft && sub != 0) || mbar_wait_fast(&sfs_full[slot], sph, abort));
        if (!__all_sync(FULL, rdy)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dst = tmem + lane_base + (uint32_t)C::kAccCols + stage * C::kSfCols;
        if (sft) {
          if (sub == 0) {
            // [row][16] bytes; B rows past the tile's boxes feed no output
            // column
            const uint4 *sv = reinterpret_cast<const uint4 *>(smem + C::kOffSfa + slot * C::kSft);
#pragma unroll
            for (int j = 0; j < 4; ++j) ga[j] = sv[32 * j + lane];
#pragma unroll
            for (int c = 0; c < C::kRowChunks; ++c)
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int row = 128 * c + 32 * j + lane;
                gb[c][j] = row < BN ? sv[C::kSftA / 16 + row] : make_uint4(0u, 0u, 0u, 0u);
              }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfs_empty[slot]);   // after the warp's reads
            if (++slot == C::kSftSlots) { slot = 0; sph ^= 1; }
          }
          uint32_t r[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) r[j] = ga[j].x;
          tc_st_x4(dst, r);
#pragma unroll
          for (int c = 0; c < C::kRowChunks; ++c) {
#pragma unroll
            for (int j = 0; j < 4; ++j) r[j] = gb[c][j].x;
            tc_st_x4(dst + 4 + 4 * c, r);
          }
          // the next stage's bytes move into .x
#pragma unroll
          for (int j = 0; j < 4; ++j) ga[j] = make_uint4(ga[j].y, ga[j].z, ga[j].w, 0u);
#pragma unroll
          for (int c = 0; c < C::kRowChunks; ++c)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              gb[c][j] = make_uint4(gb[c][j].y, gb[c][j].z, gb[c][j].w, 0u);
        } else {
          const uint4 *src =
              reinterpret_cast<const uint4 *>(smem + C::kOffSfa + slot * C::kSfa) + lane;
          if (Kd::kKGroups == 2) {
            const uint4 g0 = src[0], g1 = src[32];
            const uint32_t r[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            tc_st_x8(dst, r);
          } else {
            const uint4 g0 = src[0];
            const uint32_t r[4] = {g0.x, g0.y, g0.z, g0.w};
            tc_st_x4(dst, r);
          }
          if (!Kd::kRowScaledB) {
            // kind::mxf8f6f4's B block scales: the same layout, one 128-row
            // chunk of B after another, behind the A scale columns
            const uint4 *srb =
                reinterpret_cast<const uint4 *>(smem + C::kOffSfb + slot * C::kSfb) + lane;
#pragma unroll
            for (int gc = 0; gc < Kd::kKGroups * C::kRowChunks; ++gc) {
              const uint4 v = srb[32 * gc];
              const uint32_t r[4] = {v.x, v.y, v.z, v.w};
              tc_st_x4(dst + 4 * Kd::kKGroups + 4 * gc, r);
            }
          }
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (sft) {
          if (++sub == C::kSfGroup) sub = 0;
        } else if (C::kSfRing) {
          // the slot's bytes are in registers and stored: the loader may refill it
          if (lane == 0) mbar_arrive(&sfs_empty[slot]);
          if (++slot == C::kSfSlots) { slot = 0; sph ^= 1; }
        } else {
          slot = stage == C::kStages - 1 ? 0 : stage + 1;
          sph = stage == C::kStages - 1 ? phase ^ 1 : phase;
        }
        if (PAIR) {
          // this CTA's operand bytes have landed too; then the even CTA hears
          // of both
          if (!__all_sync(FULL, mbar_wait_fast(&full[stage], phase, abort))) { ok = false; break; }
          if (lane == 0) {
            if (leader) mbar_arrive(&ready[stage]);
            else mbar_arrive_cluster(mapa_rank(&ready[stage], 0));
          }
        } else if (lane == 0) {
          mbar_arrive(&full[stage]);
        }
        ++w_arrived;
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- epilogue --
    // accumulator column T*j + t holds term t of token j of the tile.  Two
    // groups of four warps (4-7 and 12-15, one per TMEM lane quarter each)
    // take alternate 16-column chunks.
    const int q = warp & 3;                     // TMEM lane quarter
    // hand an accumulator buffer back to the MMA thread (PAIR: the even CTA's)
    auto release_acc = [&](int b) {
      if (PAIR && !leader) mbar_arrive_cluster(mapa_rank(&acc_empty[b], 0));
      else mbar_arrive(&acc_empty[b]);
    };
    const int grp = warp >= 12 ? 1 : 0;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    float *gx = xchg + grp * C::kXchgFloats;
    pdl_wait();                                 // row scales in, h / y out
    constexpr int kTokPerLd = 16 / T;           // tokens per 16-column load
    for (int it = 0;; ++it) {
      const int t = ring_read(ring_full, ring_empty, ring, it, lane == 0, abort, n_tiles);
      bool ok = t < n_tiles && !*abort;
      Tile tl{0, 0, 0, 0, 0, 0};
      if (ok) tl = decode(t);
      const int mt = tl.mt, rowB = tl.rowB, nB = tl.nB;
      const int md = mode_of(tl.ph);
      const int buf = it % C::kAcc;
      const uint32_t use = (uint32_t)(it / C::kAcc);
      const int ntok = nB / T;                  // tokens in this tile (>= 1 in a tile)
      const int rtok0 = rowB / T;               // sorted row of the tile's first token
      // Row scales of the B terms.  The fused FFN's GEMM-2 tiles read ones
      // this launch wrote -- after the accumulator wait (which follows the
      // producer's flag wait) and an acquire of the flag, through L2; all
      // other tiles load the first chunk's before the wait, while the MMAs
      // still run.
      const float *rsb = tl.ph ? a2.b_rowscale : a.b_rowscale;
      const bool rs_late = MODE == 3 && tl.ph;
      // scales from an earlier launch: the read-only path; ones this launch
      // wrote: plain loads after the acquire below (the read-only path may
      // hold a line another B tile's rows share, read before they were
      // written)
      auto ld_rs = [&](const float *p) { return rs_late ? ld_weak_f32(p) : __ldg(p); };
      const int cfirst = 16 * grp;              // this group's first chunk
      float rs0[16];
      auto load_rs0 = [&]() {
        // (rows past ntok are discarded; with no tile the index stays at 0)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int tok = max(0, min((cfirst + i) / T, ntok - 1));
          rs0[i] = ld_rs(rsb + (size_t)(rtok0 + tok) * T + i % T);
        }
      };
      if (Kd::kRowScaledB && !rs_late) load_rs0();
      if (ok) ok = mbar_wait_fast(&acc_full[buf], use & 1, abort);
      // the group's four warps leave together: at the end of the tiles, or
      // when any of them saw the abort flag or a wait run out
      if (!group_all(grp, ok)) break;
      tc_fence_after();
      if (Kd::kRowScaledB && rs_late) {
        // one acquire per warp, ordered before the other lanes' reads
        if (lane == 0) (void)ld_acquire_gpu(a.bt_ready + tl.g);
        __syncwarp();
        load_rs0();
      }
      const uint32_t acc_t = tmem + (uint32_t)(buf * C::kChains * BN);
      if (cfirst >= nB) {
        // no chunk for this group: hand the buffer back at once
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(buf);
      }
      for (int c0 = cfirst; c0 < nB; c0 += 16 * Kd::kEpiGroups) {
        float v[16];
        {
          uint32_t r[C::kChains][16];
#pragma unroll
          for (int ch = 0; ch < C::kChains; ++ch)
            tc_ld16_nowait(acc_t + lane_base + (uint32_t)(ch * BN + c0), r[ch]);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float acc = __uint_as_float(r[0][i]);
#pragma unroll
            for (int ch = 1; ch < C::kChains; ++ch) acc += __uint_as_float(r[ch][i]);
            v[i] = acc;
          }
        }
        if (c0 + 16 * Kd::kEpiGroups >= nB) {
          // every accumulator column of the tile is in registers: hand the
          // buffer back to the MMA warp before the arithmetic and the stores
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(buf);
        }
        const int tok0 = c0 / T;
        float tok_sum[kTokPerLd];
#pragma unroll
        for (int j = 0; j < kTokPerLd; ++j) {
          float sum = 0.f;
          if (Kd::kRowScaledB) {
            if (c0 == cfirst) {
#pragma unroll
              for (int u = 0; u < T; ++u) sum = fmaf(v[T * j + u], rs0[T * j + u], sum);
            } else {
              const int tok = min(tok0 + j, ntok - 1);     // rows past ntok are discarded
              const float *rsc = rsb + (size_t)(rtok0 + tok) * T;
#pragma unroll
              for (int u = 0; u < T; ++u) sum = fmaf(v[T * j + u], ld_rs(rsc + u), sum);
            }
          } else {
#pragma unroll
            for (int u = 0; u < T; ++u) sum += v[T * j + u];
          }
          tok_sum[j] = sum;
        }
        if (md == 2) {
          const int m = mt * 128 + 32 * q + lane;
          float *y = MODE == 3 ? a2.y : a.y;
#pragma unroll
          for (int j = 0; j < kTokPerLd; ++j)
            if (tok0 + j < ntok) y[(size_t)(rtok0 + tok0 + j) * a.H + m] = tok_sum[j];
        } else {
          // Rows 0-63 gate (quarters 0,1), 64-127 up (quarters 2,3).  Quarter
          // q and q+2 hold gate and up of the same 32 rows n; the gate warp
          // finishes the chunk's even tokens, the up warp the odd ones, each
          // handing the other its half through disjoint slots of xchg.
          const int qq = q & 1;
          const bool gate = q < 2;
          // Token j = 2 jj + par of the chunk is this warp's (par = 0 for the
          // gate warp); the loops below have no data-dependent branch, so the
          // warp's tokens run as independent chains.
          const int slot0 = (32 * qq + lane) * kTokPerLd;
          const int par = gate ? 0 : 1;
          constexpr int kOwn = kTokPerLd / 2;
#pragma unroll
          for (int jj = 0; jj < kOwn; ++jj)   // the other warp's tokens
            gx[slot0 + 2 * jj + 1 - par] = gate ? tok_sum[2 * jj + 1] : tok_sum[2 * jj];
          group_sync(grp);
          {
            const int n = mt * 64 + 32 * qq + lane;
#pragma unroll
            for (int jj = 0; jj < kOwn; ++jj) {
              const int j = 2 * jj + par;
              const float own = gate ? tok_sum[2 * jj] : tok_sum[2 * jj + 1];
              const float oth = gx[slot0 + j];
              const float g = gate ? own : oth;
              const float u = gate ? oth : own;
              // SiLU(g) * u, rounded to bf16 (the fast exponential and divide
              // are far inside the bf16 rounding step)
              const uint16_t hb = f32_to_bf16_bits(__fdividef(g, 1.f + __expf(-g)) * u);
              if (tok0 + j < ntok) a.h[(size_t)(rtok0 + tok0 + j) * a.I + n] = hb;
            }
          }
          group_sync(grp);
        }
      }
      if (!Kd::kRowScaledB && md == 1) {
        // kind::mxf8f6f4's GEMM-2 operand: two E4M3 terms of h with a scale
        // byte per 32-element block.  Each thread takes whole blocks -- one
        // token's 32 h columns of this tile, read back after the group's
        // barrier -- of the tokens this group finished: chunk k of the group
        // held tokens 16k + 8 grp .. +7.
        group_sync(grp);
        const int nch = nB > 16 * grp ? (nB - 16 * grp + 31) / 32 : 0;
        for (int p = 32 * q + lane; p < 16 * nch; p += 128) {
          const int lt = p >> 1, b = p & 1;
          const int tok = 16 * (lt >> 3) + 8 * grp + (lt & 7);
          if (tok >= ntok) continue;
          const size_t r = (size_t)(rtok0 + tok);
          const int col = mt * 64 + 32 * b;
          const uint4 *src = reinterpret_cast<const uint4 *>(a.h + r * a.I + col);
          float v[32];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 w = ld_global_v4(src + i);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              v[8 * i + 2 * k] = __uint_as_float(ww[k] << 16);
              v[8 * i + 2 * k + 1] = __uint_as_float(ww[k] & 0xffff0000u);
            }
          }
          encode_block_f8(v, a.hq + (2 * r) * a.I + col, a.hq + (2 * r + 1) * a.I + col,
                          a.hs + (2 * r) * (a.I / 32) + col / 32,
                          a.hs + (2 * r + 1) * (a.I / 32) + col / 32);
        }
      }
      if (MODE == 3 && md == 1) {
        // The tile's h columns are written.  Count it; the B tile's last
        // GEMM-1 tile turns the B tile's h rows (complete now) into the
        // GEMM-2 operand and publishes them.
        group_sync(grp);
        if (q == 0 && lane == 0) {
          // release: the group's h stores (ordered before by the barrier);
          // acquire: the other tiles' stores, before this group reads them
          const int done = atom_add_acq_rel_gpu(a.bt_done + tl.g, 1) + 1;
          *s_last = done == mt1;
        }
        group_sync(grp);
        if (*s_last) {
          for (int j = 0; j < ntok; ++j) {
            const size_t r = (size_t)(rtok0 + j);
            encode_row_f4_group<T>(a.h + r * a.I, a.I, a.hq + (size_t)T * r * (a.I / 2),
                                   reinterpret_cast<float *>(a.hs) + (size_t)T * r, grp, s_red);
          }
          fence_proxy_async_global();           // TMA loads of another CTA read the rows
          __threadfence();
          group_sync(grp);
          if (q == 0 && lane == 0) st_release_gpu(a.bt_ready + tl.g, 1);
        }
      }
    }
  }

  // Every role has left its loop, and the MMA thread's issued work is
  // complete.  After an abort, TMA loads may still be in flight into stages
  // the MMA never consumed: the A-scale writers make the arrivals they owe on
  // those stages' full barriers (the producer issued at most kStages ahead of
  // them), so that each barrier's phase now waits for its TMA bytes alone,
  // and the producer waits (bounded) for the last stages it issued to land
  // before the CTA's shared memory is released.  (PAIR: a full barrier waits
  // for the producer and its bytes alone already.)
  __syncthreads();
  if (*abort) {
    const int issued = *s_issued;
    if (!PAIR && warp >= 8 && warp < 12 && lane == 0)
      for (int j = w_arrived; j < issued; ++j) mbar_arrive(&full[j % C::kStages]);
    __syncthreads();
    if (warp == 0 && lane == 0)
      for (int j = max(0, issued - C::kStages); j < issued; ++j)
        mbar_wait_drain(&full[j % C::kStages], (uint32_t)(j / C::kStages) & 1u);
    // the scale loader's last signals: their cp.async arrivals or TMA bytes
    // have landed
    if (warp == 1)
      for (int j = max(0, l_signaled - n_sfslots); j < l_signaled; ++j)
        mbar_wait_drain(&sfs_full[j % n_sfslots], (uint32_t)(j / n_sfslots) & 1u);
    __syncthreads();
  }
  if (PAIR) {
    // An abort ends the other CTA's waits at once; then neither CTA leaves
    // (its barriers and operands are the other's too) before both are done.
    if (*abort && threadIdx.x == 0) st_cluster_u32(mapa_rank((const void *)abort, crank ^ 1u), 1u);
    tc_fence_before();
    cluster_sync_all();
    if (warp == 2) {
      tc_fence_after();
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(C::kTmemCols));
    }
  } else if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols));
  }
}

// ----------------------------------------------------------------- host --

inline size_t align256_tc(size_t n) { return (n + 255) & ~size_t(255); }

// Operands of either kind: the terms of x and of h (kind::mxf8f6f4: 2 rows of
// K bytes per sorted row; kind::mxf4: kTerms rows of K/2 bytes) and their
// scales (block scale bytes [2P, K/32], or kTerms floats per row).
inline size_t tc_term_bytes(size_t P, int K) {
  const size_t f8 = 2 * P * (size_t)K, f4 = kF4Terms * P * (size_t)K / 2;
  return f8 > f4 ? f8 : f4;
}
inline size_t tc_scale_bytes(size_t P, int K) {
  const size_t f8 = 2 * P * (size_t)K / 32, f4 = kF4Terms * P * sizeof(float);
  return f8 > f4 ? f8 : f4;
}
// Counters of one call: the two GEMMs' tile counters (ints 0, 1), then the
// fused FFN's per-B-tile done counts and readiness flags.  A B tile holds at
// least 16 term rows (two tokens) or all of an expert's, so there are at
// most P/2 + (active experts <= 1024) of them.
inline size_t tc_bt_max(size_t P) { return P / 2 + 1025; }
inline size_t tc_counter_ints(size_t P) { return 64 + 2 * tc_bt_max(P); }
inline size_t tc_workspace_bytes(size_t P, int H, int I) {
  return align256_tc(tc_term_bytes(P, H)) + align256_tc(tc_scale_bytes(P, H)) +
         align256_tc(tc_term_bytes(P, I)) + align256_tc(tc_scale_bytes(P, I)) +
         align256_tc(tc_counter_ints(P) * sizeof(int));
}

// The tensor-core variant streams the weights with TMA and needs no
// dequantisation, so it is the default wherever its shape limits allow
// (scale rows of at least 16 bytes: H >= 512).
inline bool tc_prefer(size_t P, int E, int H) {
  (void)P;
  (void)E;
  return H >= 512;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process (a function-
// local static: its initialisation is thread-safe).
inline EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return (EncodeTiledFn) nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D K-major tensor map: inner dimension `inner` elements, `rows` rows,
// row pitch `pitch` bytes, box `box_inner` x `box_rows`, 128-byte swizzle
// (or none: the 16-byte scale groups).
inline bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner,
                     uint64_t rows, uint64_t pitch, uint32_t box_inner, uint32_t box_rows,
                     CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            swz == CU_TENSOR_MAP_SWIZZLE_NONE ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                              : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map: [outer][mid][inner], pitches `pitch` (mid) and `pitch2` (outer)
// bytes, box `box_inner` x `box_mid` x `box_outer`.
inline bool make_map3(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner,
                      uint64_t mid, uint64_t outer, uint64_t pitch, uint64_t pitch2,
                      uint32_t box_inner, uint32_t box_mid, uint32_t box_outer,
                      CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, mid, outer};
  const cuuint64_t strides[2] = {pitch, pitch2};
  const cuuint32_t box[3] = {box_inner, box_mid, box_outer};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            swz == CU_TENSOR_MAP_SWIZZLE_NONE ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                              : CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weight maps: padded E2M1 (box 128 elements) for kind::mxf8f6f4, packed
// bytes (box 128 bytes = 256 codes) for kind::mxf4.  GEMM-1's [E*2I, K] as
// [2E][I][K] with a box of 64 rows x both halves of one expert (its gate and
// up rows of the tile); GEMM-2's [E*H, K] with a box of 128 rows.
template <int KIND>
inline bool make_weight_map_gate_up(CUtensorMap *m, const uint8_t *codes, uint64_t K, uint64_t I,
                                    uint64_t E) {
  const uint64_t pitch = K / 2;
  if (KIND == KIND_F4)
    return make_map3(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, I, 2 * E, pitch, I * pitch,
                     128, 64, 2, CU_TENSOR_MAP_SWIZZLE_128B);
  return make_map3(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, codes, K, I, 2 * E, pitch,
                   I * pitch, 128, 64, 2, CU_TENSOR_MAP_SWIZZLE_128B);
}
template <int KIND>
inline bool make_weight_map(CUtensorMap *m, const uint8_t *codes, uint64_t K, uint64_t rows) {
  if (KIND == KIND_F4)
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, rows, K / 2, 128, 128);
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, codes, K, rows, K / 2, 128, 128);
}

// Maximum dynamic shared memory of the two GEMM kernels of one
// instantiation, set once per device; a failed set is reported and retried
// on the next call.  Guarded by a mutex: host threads may make their first
// call at the same time.
template <int KIND, int MODE, int BN, int PAIR = 0>
inline int tc_attributes(int dev) {
  using C = TcCfg<KIND, BN, PAIR>;
  static std::mutex mu;
  static unsigned long long done = 0;   // one bit per device
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if ((done >> dev) & 1ull) return MOE_OK;
  if (cudaFuncSetAttribute(tc_gemm_kernel<KIND, MODE, BN, PAIR>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  done |= 1ull << dev;
  return MOE_OK;
}

// CTAs of a paired GEMM launch: two per cluster of two that can be resident
// at once (a cluster's two SMs sit in one GPC), asked of the runtime once per
// kernel and process; at most the SM count.
template <int MODE, int BN>
inline int tc_pair_grid(int sms) {
  static std::atomic<int> cached{0};
  int n = cached.load();
  if (n == 0) {
    using C = TcCfg<KIND_F8, BN, 1>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sms & ~1));
    cfg.blockDim = dim3(TcKindCfg<KIND_F8>::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, tc_gemm_kernel<KIND_F8, MODE, BN, 1>, &cfg) !=
            cudaSuccess ||
        clusters <= 0) {
      cudaGetLastError();
      clusters = sms / 2;
    }
    n = 2 * std::min(clusters, sms / 2);
    cached.store(n);
  }
  return n;
}

// The tensor maps of one FFN call depend only on its pointers and sizes;
// callers that run the same problem again (an eager decode loop) find them
// here instead of encoding twelve maps on the host per call.  A handful of
// entries, replaced round-robin, under a mutex.
struct TcMapKey {
  int kind, bn, pair, dev, H, I, E;
  size_t P;
  const void *w13c, *w2c, *w13s, *w2s, *xq, *hq;
  bool operator==(const TcMapKey &o) const {
    return kind == o.kind && bn == o.bn && pair == o.pair && dev == o.dev && H == o.H &&
           I == o.I && E == o.E && P == o.P && w13c == o.w13c && w2c == o.w2c &&
           w13s == o.w13s && w2s == o.w2s && xq == o.xq && hq == o.hq;
  }
};

struct TcMapCache {
  static constexpr int kEntries = 8;
  std::mutex mu;
  TcMapKey key[kEntries];
  TcMaps m1[kEntries], m2[kEntries];
  bool used[kEntries] = {};
  int next = 0;
  bool find(const TcMapKey &k, TcMaps &a, TcMaps &b) {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < kEntries; ++i)
      if (used[i] && key[i] == k) {
        a = m1[i];
        b = m2[i];
        return true;
      }
    return false;
  }
  void put(const TcMapKey &k, const TcMaps &a, const TcMaps &b) {
    std::lock_guard<std::mutex> lk(mu);
    const int i = next;
    next = (next + 1) % kEntries;
    key[i] = k;
    m1[i] = a;
    m2[i] = b;
    used[i] = true;
  }
};

inline TcMapCache &tc_map_cache() {
  static TcMapCache c;
  return c;
}

// One FFN call on the tensor cores: the x encoder, then GEMM-1 + SwiGLU, the
// h encoder and GEMM-2 -- or, FUSED (kind::mxf4), the x encoder and one
// launch of both GEMMs that encodes h itself; PAIR (kind::mxf8f6f4): both
// GEMMs on clusters of two CTAs.
template <int KIND, int BN, bool FUSED, int PAIR = 0>
int tc_run(const FfnArgs &f, uint8_t *ws, int sms, cudaStream_t s) {
  static_assert(!FUSED || KIND == KIND_F4, "the fused FFN takes the kind::mxf4 operands");
  static_assert(!PAIR || (KIND == KIND_F8 && !FUSED), "CTA pairs: kind::mxf8f6f4, two launches");
  using C = TcCfg<KIND, BN, PAIR>;
  using Kd = TcKindCfg<KIND>;
  constexpr int T = Kd::kTerms;
  const size_t P = (size_t)f.T * f.k;
  const int H = f.H, I = f.I, E = f.E;
  const size_t xrow = (size_t)H * Kd::kBRowBytesPerK2 / 2;   // bytes per term row of x
  const size_t hrow = (size_t)I * Kd::kBRowBytesPerK2 / 2;
  uint8_t *xq = ws;
  uint8_t *xs = xq + align256_tc(tc_term_bytes(P, H));
  uint8_t *hq = xs + align256_tc(tc_scale_bytes(P, H));
  uint8_t *hs = hq + align256_tc(tc_term_bytes(P, I));
  int *counters = reinterpret_cast<int *>(hs + align256_tc(tc_scale_bytes(P, I)));

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  int st;
  if constexpr (FUSED) {
    st = tc_attributes<KIND, 3, BN>(dev);
  } else {
    st = tc_attributes<KIND, 1, BN, PAIR>(dev);
    if (st == MOE_OK) st = tc_attributes<KIND, 2, BN, PAIR>(dev);
  }
  if (st != MOE_OK) return st;

  // GEMM-1 (a1): W13 [E*2I, H] x x-terms [T*P, H] -> h; GEMM-2 (a2): W2 [E*H, I]
  // x h-terms [T*P, I] -> y
  TcArgs a1{};
  a1.off = f.off;
  a1.E = E;
  a1.P = (int)P;
  a1.I = I;
  a1.H = H;
  a1.h = f.h;
  a1.hq = hq;
  a1.hs = hs;
  a1.y = f.y;
  // B boxes of 16, 32, 64 and 128 rows (wider tiles load two)
  for (int i = 0; i < 4; ++i) a1.b_box[i] = (int)std::min<size_t>(16u << i, T * P);
  a1.tile_counter = counters;
  a1.bt_done = counters + 64;
  a1.bt_ready = counters + 64 + tc_bt_max(P);
  TcArgs a2 = a1;
  a1.a_scales = f.w13s;
  a1.b_scales = xs;
  a1.b_rowscale = reinterpret_cast<const float *>(xs);
  a1.K = H;
  a1.rows_per_expert = 2 * I;
  a2.a_scales = f.w2s;
  a2.b_scales = hs;
  a2.b_rowscale = reinterpret_cast<const float *>(hs);
  a2.K = I;
  a2.rows_per_expert = H;
  a2.tile_counter = counters + 1;
  // scale bytes by TMA: 16-byte groups of whole rows (K % 512 == 0) from
  // 16-byte aligned scale arrays
  auto al16 = [](const void *q) { return ((uintptr_t)q & 15u) == 0; };
  // (kind::mxf4 keeps its cp.async scale loads: with TMA the HBM-bound
  // kind::mxf4 GEMMs measured 1.3-2 % slower)
  a1.sf_tma = KIND == KIND_F8 && H % 512 == 0 && al16(f.w13s) ? 1 : 0;
  a2.sf_tma = KIND == KIND_F8 && I % 512 == 0 && al16(f.w2s) ? 1 : 0;

  TcMaps maps1{}, maps2{};
  const TcMapKey key{KIND, BN, PAIR, dev, H, I, E, P, f.w13c, f.w2c, f.w13s, f.w2s, xq, hq};
  if (!tc_map_cache().find(key, maps1, maps2)) {
    if (!make_weight_map_gate_up<KIND>(&maps1.a, f.w13c, H, I, E)) return MOE_ERR_CUDA;
    for (int i = 0; i < 4; ++i)
      if (!make_map(&maps1.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, xrow, T * P, xrow, 128,
                    a1.b_box[i]))
        return MOE_ERR_CUDA;
    if (!make_weight_map<KIND>(&maps2.a, f.w2c, I, (uint64_t)E * H)) return MOE_ERR_CUDA;
    for (int i = 0; i < 4; ++i)
      if (!make_map(&maps2.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, hq, hrow, T * P, hrow, 128,
                    a1.b_box[i]))
        return MOE_ERR_CUDA;
    const auto nosw = CU_TENSOR_MAP_SWIZZLE_NONE;
    if (a1.sf_tma) {
      if (!make_map3(&maps1.sa, CU_TENSOR_MAP_DATA_TYPE_UINT8, f.w13s, H / 32, I, 2 * (uint64_t)E,
                     H / 32, (uint64_t)I * (H / 32), 16, 64, 2, nosw))
        return MOE_ERR_CUDA;
      for (int i = 0; i < 4; ++i)
        if (!make_map(&maps1.sb[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, xs, H / 32, T * P, H / 32, 16,
                      a1.b_box[i], nosw))
          return MOE_ERR_CUDA;
    }
    if (a2.sf_tma) {
      if (!make_map(&maps2.sa, CU_TENSOR_MAP_DATA_TYPE_UINT8, f.w2s, I / 32, (uint64_t)E * H,
                    I / 32, 16, 128, nosw))
        return MOE_ERR_CUDA;
      for (int i = 0; i < 4; ++i)
        if (!make_map(&maps2.sb[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, hs, I / 32, T * P, I / 32, 16,
                      a1.b_box[i], nosw))
          return MOE_ERR_CUDA;
    }
    tc_map_cache().put(key, maps1, maps2);
  }

  if (KIND == KIND_F4) {
    const int ncounters = FUSED ? (int)tc_counter_ints(P) : 2;
    if (launch_encode_f4<T>(f.x, f.sp, f.k, H, P, xq, reinterpret_cast<float *>(xs), 0, counters,
                            ncounters, s) != cudaSuccess)
      return MOE_ERR_CUDA;
  } else {
    const long blocks = (long)P * (H / 32);
    const int grid = (int)std::min<long>((blocks + 255) / 256, (long)sms * 16);   // thread per block
    if (launch_pdl(split_x_kernel, grid, 256, 0, s, f.x, f.sp, (int)P, f.k, H, xq, xs, counters) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }

  if constexpr (FUSED) {
    if (launch_pdl(tc_gemm_kernel<KIND, 3, BN>, sms, Kd::kThreads, C::kSmem, s, maps1, a1, maps2,
                   a2) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if constexpr (PAIR != 0) {
    // clusters of two CTAs, as many as are resident at once
    if (launch_pdl_cluster(tc_gemm_kernel<KIND, 1, BN, PAIR>, tc_pair_grid<1, BN>(sms),
                           Kd::kThreads, C::kSmem, 2u, s, maps1, a1, maps1, a1) != cudaSuccess ||
        launch_pdl_cluster(tc_gemm_kernel<KIND, 2, BN, PAIR>, tc_pair_grid<2, BN>(sms),
                           Kd::kThreads, C::kSmem, 2u, s, maps2, a2, maps2, a2) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (launch_pdl(tc_gemm_kernel<KIND, 1, BN>, sms, Kd::kThreads, C::kSmem, s, maps1, a1, maps1,
                 a1) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (KIND == KIND_F4)
    if (launch_encode_f4<T>(f.h, nullptr, 1, I, P, hq, reinterpret_cast<float *>(hs), 1, nullptr,
                            0, s) != cudaSuccess)
      return MOE_ERR_CUDA;
  if (launch_pdl(tc_gemm_kernel<KIND, 2, BN>, sms, Kd::kThreads, C::kSmem, s, maps2, a2, maps2,
                 a2) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// B-tile width wanted for a problem: room for the busier experts (1.5 x
// the average B rows per active expert), and at least 4 tokens.
template <int KIND>
inline size_t tc_want(const FfnArgs &f) {
  const size_t P = (size_t)f.T * f.k;
  const size_t used = P < (size_t)f.E ? P : (size_t)f.E;
  const size_t terms = TcKindCfg<KIND>::kTerms;
  const size_t rows = (terms * P + used - 1) / used;           // B rows per expert, average
  size_t want = rows + rows / 2;
  if (want < 4 * terms) want = 4 * terms;
  return want;
}

template <int KIND, bool FUSED>
inline int tc_dispatch(const FfnArgs &f, uint8_t *ws, int sms, cudaStream_t s) {
  const size_t want = tc_want<KIND>(f);
  if (want <= 16) return tc_run<KIND, 16, FUSED>(f, ws, sms, s);
  if (want <= 32) return tc_run<KIND, 32, FUSED>(f, ws, sms, s);
  if (want <= 64) return tc_run<KIND, 64, FUSED>(f, ws, sms, s);
  if (want <= 128) return tc_run<KIND, 128, FUSED>(f, ws, sms, s);
  if (want <= 192) return tc_run<KIND, 192, FUSED>(f, ws, sms, s);
  return tc_run<KIND, 256, FUSED>(f, ws, sms, s);
}

// kind::mxf8f6f4 on clusters of two CTAs: B tiles of 128, 192 or 256 rows.
inline int tc_dispatch_pair(const FfnArgs &f, uint8_t *ws, int sms, cudaStream_t s) {
  const size_t want = tc_want<KIND_F8>(f);
  if (want <= 128) return tc_run<KIND_F8, 128, false, 1>(f, ws, sms, s);
  if (want <= 192) return tc_run<KIND_F8, 192, false, 1>(f, ws, sms, s);
  return tc_run<KIND_F8, 256, false, 1>(f, ws, sms, s);
}

// kind::mxf4 (packed FP4 weights, 4 activation terms) when K allows 256-wide
// stages, else kind::mxf8f6f4.
inline int tc_ffn(const FfnArgs &f, uint8_t *ws, int sms, cudaStream_t s, int kind) {
  if (f.H < 512 || f.I < 128) return MOE_ERR_UNSUPPORTED;   // scale rows of >= 16 bytes
  if (kind < 0) {
    // kind::mxf4 (exact 8-term activations) while the B tiles stay narrow --
    // at small N the extra term columns cost nothing; with many tokens per
    // expert the 8 terms double the MMA work and kind::mxf8f6f4 (two E4M3
    // terms) is faster.
    const size_t P = (size_t)f.T * f.k;
    const size_t used = P < (size_t)f.E ? P : (size_t)f.E;
    const bool narrow = (size_t)kF4Terms * P <= 128 * used;
    const bool f4_ok = f.H % 256 == 0 && f.I % 256 == 0 &&
                       f.H <= 2 * ENC_THREADS * ENC_MAX_PAIRS &&
                       f.I <= 2 * ENC_THREADS * ENC_MAX_PAIRS;
    kind = (f4_ok && narrow) ? KIND_F4 : KIND_F8;
    // A few tokens per expert (B tiles of at most 32 columns, as in a
    // batch-1 block): both GEMMs in one launch, which saves the h encoder's
    // launch and GEMM-2's ramp (measured 193 vs 200 us at batch 1).  With
    // wider tiles the fused launch's h encoding -- one warp group of the CTA
    // that finishes a B tile -- costs more than it saves (4-6 % slower).
    if (kind == KIND_F4 && tc_want<KIND_F4>(f) <= 32 && f.I <= 2 * 128 * GRP_ENC_MAX_PAIRS)
      kind = KIND_F4_FUSED;
  }
  if (kind == KIND_F4 || kind == KIND_F4_FUSED) {
    if (f.H % 256 || f.I % 256 || f.H > 2 * ENC_THREADS * ENC_MAX_PAIRS ||
        f.I > 2 * ENC_THREADS * ENC_MAX_PAIRS)
      return MOE_ERR_UNSUPPORTED;
    if (kind == KIND_F4_FUSED) {
      // h rows are encoded by one warp group of the fused kernel
      if (f.I > 2 * 128 * GRP_ENC_MAX_PAIRS) return MOE_ERR_UNSUPPORTED;
      return tc_dispatch<KIND_F4, true>(f, ws, sms, s);
    }
    return tc_dispatch<KIND_F4, false>(f, ws, sms, s);
  }
  if (kind == KIND_F8_PAIR) {
    // GEMM-2's m-blocks (H / 128 of them) go to the pair two at a time
    if (f.H % 256 || sms < 2) return MOE_ERR_UNSUPPORTED;
    return tc_dispatch_pair(f, ws, sms, s);
  }
  return tc_dispatch<KIND_F8, false>(f, ws, sms, s);
}

}  // namespace moe
