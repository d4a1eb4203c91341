// ffn_tc.cuh -- MXFP4 expert FFN on the 5th-generation tensor cores.
//
// The expert weights stay in their MXFP4 form all the way into the tensor
// core: tcgen05.mma.kind::mxf8f6f4.block_scale takes A = E2M1 codes with one
// E8M0 scale per 32 elements -- exactly the OCP MX block the pages name for
// the experts ("MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section "FP4 Expert
// 量化"; "mimo-tilert-1000tps-trillion-parameter-inference", section
// "第一层：FP4 选择性量化").  Nothing is dequantised on the CUDA cores.
//
// The activations (bf16) become the B operand as two E4M3 terms with their
// own E8M0 block scales: x = s1*q1 + s2*q2 per 32-element block, q1 the
// nearest E4M3 of x/s1, q2 that of the remainder.  A bf16 value has 8
// significant bits and q1 captures the top 4, so the remainder is exact in
// E4M3 whenever it stays in E4M3's normal range; what is lost is below
// ~2^-18 of the block's largest element.  Each token occupies two adjacent
// B rows (its two terms) and the epilogue adds the two accumulator columns.
//
// One persistent CTA per SM walks a tile list (expert, 128-row block of the
// weight matrix, block of B rows).  Warp roles, after the tile-pipelining and
// warp-specialisation ideas the pages describe for TileRT (prior art):
//   warp 0  TMA producer: weight tile (E2M1, 16U4_ALIGN16B so that each code
//           lands in its own byte lane, 128B swizzle) + activation tile;
//   warp 1  scale loader: cp.async of the scale bytes straight into the
//           32-row x 16-byte layout tcgen05.cp wants;
//   warp 2  TMEM allocation and the single MMA-issuing thread;
//   warps 4-7 epilogue: TMEM -> registers -> SwiGLU (GEMM-1) or y (GEMM-2).
// Every wait is bounded; on time-out the kernel records MOE_DEV_TIMEOUT,
// drains what it issued, frees its TMEM and returns.
#pragma once
#include <cuda.h>
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

// Bounded wait: false (and the status word set) after ~2 s.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 63) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        raise_status(MOE_DEV_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
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

// Instruction descriptor of mxf8f6f4.block_scale: A = E2M1, B = E4M3,
// E8M0 scales, M = 128, K-major A and B.
__device__ __forceinline__ uint32_t idesc_mxf8f6f4(int n, uint32_t sf_id) {
  return (sf_id << 4) | (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) |
         ((128u >> 4) << 24) | (sf_id << 29);
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

__device__ __forceinline__ void tc_cp_32x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 16 columns of 32-bit accumulator -> 16 registers per thread.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

// --------------------------------------------- two-term E4M3 block encoding --

// Exponent s of a block scale 2^s for block maximum amax (> 0): amax / 2^s
// lies in [128, 256), inside E4M3's range (max 448).
__device__ __forceinline__ int block_exp(float amax) {
  const int be = (int)((__float_as_uint(amax) >> 23) & 0xff);
  const int e = (be == 0 ? -126 : be - 127) - 7;
  return max(-126, min(126, e));
}

__device__ __forceinline__ float pow2f(int s) { return __uint_as_float((uint32_t)(127 + s) << 23); }

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float from_e4m3(uint8_t q) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
  return __half2float(*reinterpret_cast<__half *>(&h));
}

// Warp-cooperative: lane l holds element l of one 32-element block.
// Produces the two E4M3 codes of the lane and the two scale bytes.
__device__ __forceinline__ void split2(float v, uint8_t &q1, uint8_t &q2, uint8_t &sb1,
                                       uint8_t &sb2) {
  const float a1 = warp_max(fabsf(v));
  int s1 = 0;
  float r = v;
  if (a1 > 0.f) {
    s1 = block_exp(a1);
    q1 = to_e4m3(v * pow2f(-s1));
    r = v - from_e4m3(q1) * pow2f(s1);
  } else {
    q1 = 0;
  }
  const float a2 = warp_max(fabsf(r));
  int s2 = 0;
  if (a2 > 0.f) {
    s2 = block_exp(a2);
    q2 = to_e4m3(r * pow2f(-s2));
  } else {
    q2 = 0;
  }
  sb1 = (uint8_t)(127 + s1);
  sb2 = (uint8_t)(127 + s2);
}

// Activation operand of GEMM-1: for every sorted row r (token sp[r]/k), the
// two E4M3 terms of x[token] as B rows 2r and 2r+1, [2P, H], and their scale
// bytes [2P, H/32].  One warp per 32-element block.
__global__ void __launch_bounds__(256)
split_x_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ sp, int P, int k,
               int H, uint8_t *__restrict__ xq, uint8_t *__restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int nb = H / 32;
  const long total = (long)P * nb;
  for (long w = (blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5; w < total;
       w += ((long)gridDim.x * blockDim.x) >> 5) {
    const int r = (int)(w / nb), b = (int)(w % nb);
    const int t = __ldg(sp + r) / k;
    const float v = __uint_as_float((uint32_t)__ldg(x + (size_t)t * H + b * 32 + lane) << 16);
    uint8_t q1, q2, s1, s2;
    split2(v, q1, q2, s1, s2);
    xq[(size_t)(2 * r) * H + b * 32 + lane] = q1;
    xq[(size_t)(2 * r + 1) * H + b * 32 + lane] = q2;
    if (lane == 0) {
      xs[(size_t)(2 * r) * nb + b] = s1;
      xs[(size_t)(2 * r + 1) * nb + b] = s2;
    }
  }
}

// ------------------------------------------------------------- the kernel --

struct TcMaps {
  CUtensorMap a;        // weights: [E*rows, K] E2M1 (16U4_ALIGN16B), box 128 x 64 rows
  CUtensorMap b[5];     // activations: [2P, K] E4M3, box 128 x {16,32,64,128,256} rows
};

struct TcArgs {
  const uint8_t *a_scales;   // [E*rows, K/32]
  const uint8_t *b_scales;   // [2P, K/32]
  const int32_t *off;        // [E+1]
  int E, K, rows_per_expert, P;
  int I;                     // GEMM-1: the gate/up split; GEMM-2: unused
  int H;                     // y row length (GEMM-2)
  int b_box[5];              // rows of each B box (clamped to 2P)
  // GEMM-1 outputs
  uint16_t *h;               // [P, I] bf16
  uint8_t *hq;               // [2P, I] E4M3 terms
  uint8_t *hs;               // [2P, I/32] scale bytes
  // GEMM-2 output
  float *y;                  // [P, H]
};

template <int BN>
struct TcCfg {
  static constexpr int kStages = BN <= 32 ? 10 : BN <= 64 ? 8 : BN <= 128 ? 6 : 4;
  static constexpr int kSfbChunks = (BN + 127) / 128;
  static constexpr int kA = 128 * 128;                 // bytes of one A stage
  static constexpr int kB = BN * 128;
  static constexpr int kSfa = 512;
  static constexpr int kSfb = 512 * kSfbChunks;
  static constexpr int kSfCols = 4 + 4 * kSfbChunks;   // TMEM columns per stage
  static constexpr int kAcc = BN <= 128 ? 2 : 1;        // accumulator buffers
  static constexpr int kUsed = kAcc * BN + kStages * kSfCols;
  static constexpr int kTmemCols = kUsed <= 128 ? 128 : kUsed <= 256 ? 256 : 512;
  static_assert(kUsed <= 512, "TMEM budget");
  static constexpr int kOffB = kStages * kA;
  static constexpr int kOffSfa = kOffB + kStages * kB;
  static constexpr int kOffSfb = kOffSfa + kStages * kSfa;
  static constexpr int kOffBar = kOffSfb + kStages * kSfb;
  static constexpr int kOffXchg = kOffBar + 1024;                // 64 x 8 floats
  static constexpr int kOffTab = kOffXchg + 2048;                 // active list + prefix
  static constexpr int kSmem = kOffTab + 2 * 1025 * 4 + 1024;     // + 1 KB alignment slack
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

constexpr int TC_THREADS = 256;

template <int MODE, int BN>
__global__ void __launch_bounds__(TC_THREADS, 1)
tc_gemm_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *empty = full + C::kStages;
  uint64_t *acc_full = empty + C::kStages;     // [kAcc]
  uint64_t *acc_empty = acc_full + 2;          // [kAcc]
  volatile int *abort = reinterpret_cast<volatile int *>(acc_empty + 2);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 3);
  float *xchg = reinterpret_cast<float *>(smem + C::kOffXchg);
  int *s_act = reinterpret_cast<int *>(smem + C::kOffTab);
  int *s_pre = s_act + 1025;       // tile prefix over active experts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mtiles = MODE == 1 ? a.I / 64 : a.rows_per_expert / 128;
  const int ksteps = a.K / 128;

  // tile table: active experts and the prefix of their tile counts
  if (warp == 0) {
    int n = 0, acc = 0;
    for (int e0 = 0; e0 < a.E; e0 += 32) {
      const int e = e0 + lane;
      const int cnt = e < a.E ? __ldg(a.off + e + 1) - __ldg(a.off + e) : 0;
      const int nt = cnt > 0 ? (2 * cnt + BN - 1) / BN : 0;
      const unsigned b = __ballot_sync(FULL, nt > 0);
      // inclusive scan of tiles among lanes
      int sc = nt * mtiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, sc, o);
        if (lane >= o) sc += y;
      }
      if (nt > 0) {
        const int pos = n + __popc(b & lanemask_lt());
        s_act[pos] = e;
        s_pre[pos] = acc + sc - nt * mtiles;   // exclusive
      }
      n += __popc(b);
      acc += __shfl_sync(FULL, sc, 31);
    }
    if (lane == 0) {
      s_act[1024] = n;
      s_pre[n] = acc;
    }
  } else if (warp == 1 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1 + 32);     // producer expect_tx + 32 scale-loader lanes
      mbar_init(&empty[s], 1);         // MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);     // one arrival per epilogue warp
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  } else if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_act = s_act[1024];
  const int n_tiles = s_pre[n_act];

  // tile index -> (expert, m-block, first B row, B rows in the tile)
  auto decode = [&](int t, int &e, int &mt, int &rowB, int &nB, int &r0, int &ne) {
    int lo = 0, hi = n_act - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    e = s_act[lo];
    r0 = __ldg(a.off + e);
    ne = __ldg(a.off + e + 1) - r0;
    const int nt_cnt = (2 * ne + BN - 1) / BN;
    const int local = t - s_pre[lo];
    mt = local / nt_cnt;
    const int nt = local % nt_cnt;
    rowB = 2 * r0 + nt * BN;
    nB = min(BN, 2 * ne - nt * BN);
  };

  if (warp == 0) {
    // ---------------------------------------------------- TMA producer --
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = blockIdx.x; t < n_tiles && !*abort; t += gridDim.x) {
        int e, mt, rowB, nB, r0, ne;
        decode(t, e, mt, rowB, nB, r0, ne);
        const int ncol = (nB + 15) & ~15;
        const int bsel = ncol <= 16 ? 0 : ncol <= 32 ? 1 : ncol <= 64 ? 2 : ncol <= 128 ? 3 : 4;
        const uint32_t bbytes = (uint32_t)a.b_box[bsel] * 128u;
        const int arow = e * a.rows_per_expert + (MODE == 1 ? mt * 64 : mt * 128);
        for (int kt = 0; kt < ksteps; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort)) break;
          mbar_expect_tx(&full[stage], 128 * 128 / 2 + bbytes);
          uint8_t *sa = smem + stage * C::kA;
          // rows 0-63 of the tile, then rows 64-127 (GEMM-1: gate, then up)
          tma_load_2d(sa, &maps.a, kt * 128, arow, &full[stage], pol_w);
          tma_load_2d(sa + 64 * 128, &maps.a, kt * 128, arow + (MODE == 1 ? a.I : 64),
                      &full[stage], pol_w);
          tma_load_2d(smem + C::kOffB + stage * C::kB, &maps.b[bsel], kt * 128, rowB,
                      &full[stage], pol_x);
          ++issued;
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
      }
      // drain: wait (bounded) until the last issued stages have landed
      if (*abort) {
        for (int s = 0; s < C::kStages && s < issued; ++s) {
          if (--stage < 0) { stage = C::kStages - 1; phase ^= 1; }
          volatile int never = 0;
          mbar_wait(&full[stage], phase, (volatile int *)&never);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------- scale loader --
    const uint32_t kb = a.K / 32;            // scale bytes per row
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < n_tiles && !*abort; t += gridDim.x) {
      int e, mt, rowB, nB, r0, ne;
      decode(t, e, mt, rowB, nB, r0, ne);
      const int ebase = e * a.rows_per_expert;
      for (int kt = 0; kt < ksteps; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort)) break;
        uint8_t *sfa = smem + C::kOffSfa + stage * C::kSfa;
        uint8_t *sfb = smem + C::kOffSfb + stage * C::kSfb;
#pragma unroll
        for (int g = 0; g < 4; ++g) {       // A rows lane + 32g
          const int i = lane + 32 * g;
          int row;
          if (MODE == 1) row = ebase + (i < 64 ? mt * 64 + i : a.I + mt * 64 + i - 64);
          else row = ebase + mt * 128 + i;
          cp_async4(sfa + 16 * lane + 4 * g, a.a_scales + (size_t)row * kb + kt * 4);
        }
#pragma unroll
        for (int g = 0; g < 4 * C::kSfbChunks; ++g) {
          const int i = lane + 32 * g;
          if (i < nB)
            cp_async4(sfb + 512 * (g >> 2) + 16 * lane + 4 * (g & 3),
                      a.b_scales + (size_t)(rowB + i) * kb + kt * 4);
        }
        cp_async_arrive_noinc(&full[stage]);
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == 2) {
    // ----------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t sf_col0 = (uint32_t)(C::kAcc * BN);
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles && !*abort; t += gridDim.x, ++it) {
        int e, mt, rowB, nB, r0, ne;
        decode(t, e, mt, rowB, nB, r0, ne);
        const int ncol = (nB + 15) & ~15;
        const int buf = it % C::kAcc;
        const uint32_t use = (uint32_t)(it / C::kAcc);
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t acc_t = tmem + (uint32_t)(buf * BN);
        bool ok = true;
        for (int kt = 0; kt < ksteps; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
          fence_proxy_async();
          tc_fence_after();
          const uint32_t sfa_t = tmem + sf_col0 + stage * C::kSfCols;
          const uint32_t sfb_t = sfa_t + 4;
          const uint32_t sa = smem_u32(smem + C::kOffSfa + stage * C::kSfa);
          const uint32_t sb = smem_u32(smem + C::kOffSfb + stage * C::kSfb);
          tc_cp_32x128b(sfa_t, smem_desc(sa, 0, 128, kSwizzleNone));
#pragma unroll
          for (int c = 0; c < C::kSfbChunks; ++c)
            tc_cp_32x128b(sfb_t + 4 * c, smem_desc(sb + 512 * c, 0, 128, kSwizzleNone));
          const uint32_t a_addr = smem_u32(smem + stage * C::kA);
          const uint32_t b_addr = smem_u32(smem + C::kOffB + stage * C::kB);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(a_addr + 32 * kk, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(b_addr + 32 * kk, 16, 1024, kSwizzle128B);
            mma_mxf8f6f4(acc_t, ad, bd, idesc_mxf8f6f4(ncol, kk), sfa_t | ((uint32_t)kk << 30),
                         sfb_t | ((uint32_t)kk << 30), (kt > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------- epilogue --
    const int q = warp - 4;                     // TMEM lane quarter
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles && !*abort; t += gridDim.x, ++it) {
      int e, mt, rowB, nB, r0, ne;
      decode(t, e, mt, rowB, nB, r0, ne);
      const int buf = it % C::kAcc;
      const uint32_t use = (uint32_t)(it / C::kAcc);
      if (!mbar_wait(&acc_full[buf], use & 1, abort)) break;
      tc_fence_after();
      const uint32_t acc_t = tmem + (uint32_t)(buf * BN);
      const int ntok = nB >> 1;                 // tokens in this tile (B rows come in pairs)
      const int rtok0 = rowB >> 1;              // sorted row of the tile's first token
      for (int c0 = 0; c0 < nB; c0 += 16) {
        float v[16];
        tc_ld16(acc_t + lane_base + (uint32_t)c0, v);
        if (MODE == 2) {
          const int m = mt * 128 + 32 * q + lane;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int tok = (c0 >> 1) + j;
            if (tok < ntok) a.y[(size_t)(rtok0 + tok) * a.H + m] = v[2 * j] + v[2 * j + 1];
          }
        } else {
          // rows 0-63 gate (quarters 0,1), 64-127 up (quarters 2,3)
          if (q >= 2) {
#pragma unroll
            for (int j = 0; j < 8; ++j) xchg[(32 * (q - 2) + lane) * 8 + j] = v[2 * j] + v[2 * j + 1];
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (q < 2) {
            const int n = mt * 64 + 32 * q + lane;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int tok = (c0 >> 1) + j;
              const float g = v[2 * j] + v[2 * j + 1];
              const float u = xchg[(32 * q + lane) * 8 + j];
              const uint16_t hb = f32_to_bf16_bits(g / (1.f + expf(-g)) * u);
              const float hv = __uint_as_float((uint32_t)hb << 16);
              uint8_t q1, q2, s1, s2;
              split2(hv, q1, q2, s1, s2);     // warp-uniform control flow
              if (tok < ntok) {
                const size_t r = (size_t)(rtok0 + tok);
                a.h[r * a.I + n] = hb;
                a.hq[(2 * r) * a.I + n] = q1;
                a.hq[(2 * r + 1) * a.I + n] = q2;
                if (lane == 0) {
                  a.hs[(2 * r) * (a.I / 32) + n / 32] = s1;
                  a.hs[(2 * r + 1) * (a.I / 32) + n / 32] = s2;
                }
              }
            }
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols));
  }
}

// ----------------------------------------------------------------- host --

inline size_t align256_tc(size_t n) { return (n + 255) & ~size_t(255); }

inline size_t tc_workspace_bytes(size_t P, int H, int I) {
  return align256_tc(2 * P * H) + align256_tc(2 * P * H / 32) + align256_tc(2 * P * I) +
         align256_tc(2 * P * I / 32);
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

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D K-major tensor map: inner dimension `inner` elements, `rows` rows,
// row pitch `pitch` bytes, box 128 x box_rows, 128-byte swizzle.
inline bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner,
                     uint64_t rows, uint64_t pitch, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
int tc_run(const FfnArgs &f, uint8_t *ws, int sms, cudaStream_t s) {
  using C = TcCfg<BN>;
  const size_t P = (size_t)f.T * f.k;
  const int H = f.H, I = f.I, E = f.E;
  uint8_t *xq = ws;
  uint8_t *xs = xq + align256_tc(2 * P * H);
  uint8_t *hq = xs + align256_tc(2 * P * H / 32);
  uint8_t *hs = hq + align256_tc(2 * P * I);

  static bool attr = false;
  if (!attr) {
    attr = true;
    cudaFuncSetAttribute(tc_gemm_kernel<1, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         C::kSmem);
    cudaFuncSetAttribute(tc_gemm_kernel<2, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         C::kSmem);
  }
  {
    const long blocks = (long)P * (H / 32);
    const int grid = (int)std::min<long>((blocks * 32 + 255) / 256, (long)sms * 16);
    split_x_kernel<<<grid, 256, 0, s>>>(f.x, f.sp, (int)P, f.k, H, xq, xs);
  }
  TcMaps maps;
  TcArgs a{};
  a.off = f.off;
  a.E = E;
  a.P = (int)P;
  a.I = I;
  a.H = H;
  a.h = f.h;
  a.hq = hq;
  a.hs = hs;
  a.y = f.y;
  for (int i = 0; i < 5; ++i) a.b_box[i] = (int)std::min<size_t>(16u << i, 2 * P);

  // GEMM-1: W13 [E*2I, H] x x-terms [2P, H]
  if (!make_map(&maps.a, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, f.w13c, H, (uint64_t)E * 2 * I,
                H / 2, 64))
    return MOE_ERR_CUDA;
  for (int i = 0; i < 5; ++i)
    if (!make_map(&maps.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, H, 2 * P, H, a.b_box[i]))
      return MOE_ERR_CUDA;
  a.a_scales = f.w13s;
  a.b_scales = xs;
  a.K = H;
  a.rows_per_expert = 2 * I;
  tc_gemm_kernel<1, BN><<<sms, TC_THREADS, C::kSmem, s>>>(maps, a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;

  // GEMM-2: W2 [E*H, I] x h-terms [2P, I]
  if (!make_map(&maps.a, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, f.w2c, I, (uint64_t)E * H, I / 2,
                64))
    return MOE_ERR_CUDA;
  for (int i = 0; i < 5; ++i)
    if (!make_map(&maps.b[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, hq, I, 2 * P, I, a.b_box[i]))
      return MOE_ERR_CUDA;
  a.a_scales = f.w2s;
  a.b_scales = hs;
  a.K = I;
  a.rows_per_expert = H;
  tc_gemm_kernel<2, BN><<<sms, TC_THREADS, C::kSmem, s>>>(maps, a);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

inline int tc_ffn(const FfnArgs &f, uint8_t *ws, int sms, cudaStream_t s) {
  if (f.H < 512 || f.I < 128) return MOE_ERR_UNSUPPORTED;   // scale rows of >= 16 bytes
  const size_t P = (size_t)f.T * f.k;
  const size_t used = P < (size_t)f.E ? P : (size_t)f.E;
  const size_t rows = (2 * P + used - 1) / used;            // average B rows per expert
  const size_t want = rows + rows / 2;
  if (want <= 16) return tc_run<16>(f, ws, sms, s);
  if (want <= 32) return tc_run<32>(f, ws, sms, s);
  if (want <= 64) return tc_run<64>(f, ws, sms, s);
  if (want <= 128) return tc_run<128>(f, ws, sms, s);
  return tc_run<256>(f, ws, sms, s);
}

}  // namespace moe
