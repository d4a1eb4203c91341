// accept.cuh -- acceptance of drafted blocks.
//
// Greedy: the target keeps the confirmed draft tokens and takes over at the
// first wrong one ("如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？",
// section "二、投机解码").  One thread-block cluster per block row (s, i):
// CTA r of the cluster scans slice r of the row with coalesced 16-byte
// loads, the partial argmaxes meet in CTA 0 through distributed shared
// memory, and CTA 0 reports a mismatching row as the 32-bit key
// (i << 26 | argmax) to an atomicMin on the sequence's slot; the last of the
// K rows to report turns the minimum into (accept_len, next_token).  The
// slots are accept_len / next_token themselves, set up by a one-CTA kernel
// launched just before.  With a bonus row (K+1 target rows per sequence, the
// last one scoring the position after the block) that row has no draft and
// always reports its argmax, so a sequence whose K drafts all match emits the
// target's own next token (the target takes over after the last confirmed
// token, "如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？", section
// "二、投机解码").
//
// Rejection sampling ("MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section
// "数据流概览"): exact test u*q(x) < p(x) in double, first rejection by
// ballot, then an exact integer inverse-CDF draw from max(0, p - q): every
// residual weight is an integer floor(r * 2^40), so the prefix sums are
// independent of summation order and equal on every device.  With a bonus
// row, a sequence whose K drafts are all accepted draws its next token from
// the target row K by the same integer rule on floor(p * 2^40).
#pragma once
#include <cooperative_groups.h>
#include "common.cuh"

namespace moe {
namespace cg = cooperative_groups;

constexpr int GREEDY_THREADS = 256;
constexpr int GREEDY_UNROLL = 10;        // 16-byte loads in flight per thread (a 152K-entry row
                                         // slice of 1/16 in one round)
constexpr int GREEDY_MAX_CLUSTER = 16;   // CTAs per row (non-portable cluster size)
constexpr int GREEDY_TOKEN_BITS = 26;    // key = row << 26 | token; V <= 2^26
constexpr unsigned GREEDY_NO_MISS = 0xffffffffu;

// One 16-byte unit of a row (elements b..b+3), visited in increasing index
// order by this thread: the running (bv, bi) keeps the first occurrence of
// the largest value.  The max of the four is one comparison away from the
// running best, and the index search runs only when the best improves.
__device__ __forceinline__ void scan_unit(const float4 q, int b, float &bv, int &bi) {
  const float m = fmaxf(fmaxf(q.x, q.y), fmaxf(q.z, q.w));
  if (m > bv) {
    bv = m;
    bi = q.x == m ? b : q.y == m ? b + 1 : q.z == m ? b + 2 : b + 3;
  }
}

// Per sequence: accept_len[s] becomes the minimum-key slot (no mismatch
// yet), next_token[s] the count of rows reported.
__global__ void __launch_bounds__(256)
greedy_init_kernel(int S, int32_t *__restrict__ accept_len, int32_t *__restrict__ next_token) {
  pdl_wait();
  pdl_trigger();
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < S; s += gridDim.x * blockDim.x) {
    accept_len[s] = (int32_t)GREEDY_NO_MISS;
    next_token[s] = 0;
  }
}

// grid (cluster_size, R, S), cluster (cluster_size, 1, 1), GREEDY_THREADS;
// R = K rows per sequence, or K + 1 with a bonus row.  Rows hold finite
// values (a row of -inf reports token 0).
__global__ void __launch_bounds__(GREEDY_THREADS)
greedy_kernel(const float *__restrict__ logits, const int32_t *__restrict__ draft,
              int S, int K, int V, int R, int32_t *__restrict__ accept_len,
              int32_t *__restrict__ next_token) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int ncta = (int)cluster.num_blocks();
  const int i = blockIdx.y, s = blockIdx.z;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int bd = blockDim.x;
  __shared__ float red_v[GREEDY_THREADS / 32];
  __shared__ int red_i[GREEDY_THREADS / 32];
  __shared__ float part_v;
  __shared__ int part_i;

  // The logits were complete before the setup kernel passed its own wait,
  // so the scan needs no wait; only the slots do.
  const float *row = logits + ((size_t)s * R + i) * V;
  float bv = -INFINITY;
  int bi = -1;
  if ((V & 3) == 0) {                  // rows 16-byte aligned: float4 units
    const int units = V / 4;
    const int per = (units + ncta - 1) / ncta;
    const int u0 = min(units, rank * per), u1 = min(units, u0 + per);
    const float4 *row4 = reinterpret_cast<const float4 *>(row);
    for (int u = u0 + threadIdx.x; u < u1; u += GREEDY_UNROLL * bd) {
      float4 q[GREEDY_UNROLL];
#pragma unroll
      for (int j = 0; j < GREEDY_UNROLL; ++j)
        if (u + j * bd < u1) q[j] = __ldcs(row4 + u + j * bd);
#pragma unroll
      for (int j = 0; j < GREEDY_UNROLL; ++j)
        if (u + j * bd < u1) scan_unit(q[j], 4 * (u + j * bd), bv, bi);
    }
  } else {
    const int per = (V + ncta - 1) / ncta;
    const int v0 = min(V, rank * per), v1 = min(V, v0 + per);
    for (int v = v0 + threadIdx.x; v < v1; v += GREEDY_UNROLL * bd) {
      float q[GREEDY_UNROLL];
#pragma unroll
      for (int j = 0; j < GREEDY_UNROLL; ++j)
        if (v + j * bd < v1) q[j] = __ldcs(row + v + j * bd);
#pragma unroll
      for (int j = 0; j < GREEDY_UNROLL; ++j)
        if (v + j * bd < v1 && q[j] > bv) { bv = q[j]; bi = v + j * bd; }
    }
  }
  warp_argmax(bv, bi);
  if (lane == 0) { red_v[w] = bv; red_i[w] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = -INFINITY;
    int idx = -1;
    for (int ww = 0; ww < nw; ++ww)
      if (better(red_v[ww], red_i[ww], v, idx)) { v = red_v[ww]; idx = red_i[ww]; }
    part_v = v;
    part_i = idx;
  }
  cluster.sync();
  if (rank == 0 && threadIdx.x == 0) {
    float v = -INFINITY;
    int m = -1;
    for (int r = 0; r < ncta; ++r) {
      const float pv = *cluster.map_shared_rank(&part_v, r);
      const int pi = *cluster.map_shared_rank(&part_i, r);
      if (better(pv, pi, v, m)) { v = pv; m = pi; }
    }
    m = max(m, 0);
    // the bonus row (i == K) has no draft: it always reports its argmax
    const int d = i < K ? __ldg(draft + (size_t)s * K + i) : -1;
    if (i < K && (d < 0 || d >= V)) raise_status(MOE_DEV_BAD_TOKEN);
    pdl_wait();                      // the slots were set up by greedy_init_kernel
    pdl_trigger();
    unsigned *key = reinterpret_cast<unsigned *>(accept_len + s);
    unsigned *cnt = reinterpret_cast<unsigned *>(next_token + s);
    if (d != m) atomicMin(key, ((unsigned)i << GREEDY_TOKEN_BITS) | (unsigned)m);
    __threadfence();
    if (atomicAdd(cnt, 1u) == (unsigned)(R - 1)) {      // the last row of the sequence
      __threadfence();
      const unsigned k = atomicOr(key, 0u);
      const bool miss = k != GREEDY_NO_MISS;
      accept_len[s] = miss ? (int32_t)(k >> GREEDY_TOKEN_BITS) : K;
      next_token[s] = miss ? (int32_t)(k & ((1u << GREEDY_TOKEN_BITS) - 1)) : -1;
    }
  }
  cluster.sync();   // keep every CTA's shared memory alive until CTA 0 is done
}

// One CTA per sequence.  blockDim.x is a multiple of 32, <= 1024.  p holds
// R = K (+1 with a bonus row) rows per sequence, q holds K.
__global__ void __launch_bounds__(1024)
rejection_kernel(const float *__restrict__ p, const float *__restrict__ q,
                 const int32_t *__restrict__ draft, const float *__restrict__ u_accept,
                 const float *__restrict__ u_resample, int S, int K, int V, int R,
                 int32_t *__restrict__ accept_len, int32_t *__restrict__ next_token) {
  pdl_wait();
  pdl_trigger();
  const int s = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nw = blockDim.x >> 5;
  __shared__ int s_a;
  __shared__ unsigned long long s_red[32];

  if (w == 0) {
    bool acc = true;
    if (lane < K) {
      const size_t row = (size_t)s * K + lane;
      const int x = __ldg(draft + row);
      if (x < 0 || x >= V) {
        raise_status(MOE_DEV_BAD_TOKEN);
        acc = false;
      } else {
        const double u = (double)__ldg(u_accept + row);
        const size_t prow = (size_t)s * R + lane;
        acc = u * (double)__ldg(q + row * V + x) < (double)__ldg(p + prow * V + x);
      }
    }
    const unsigned rej = __ballot_sync(FULL, lane < K && !acc);
    if (lane == 0) s_a = rej ? __ffs(rej) - 1 : K;
  }
  __syncthreads();
  const int a = s_a;
  if (tid == 0) accept_len[s] = a;
  const bool bonus = R > K;
  if (a == K && !bonus) {
    if (tid == 0) next_token[s] = -1;
    return;
  }
  // row a of p (the bonus row K when every draft was accepted); q only
  // below K
  const float *pr = p + ((size_t)s * R + a) * V;
  const float *qr = q + ((size_t)s * K + min(a, K - 1)) * V;
  const unsigned long long U = (unsigned long long)((double)__ldg(u_resample + s) * 16777216.0);

  // weight of token v: floor(max(0, p-q) * 2^40), or floor(p * 2^40) (mode 1)
  auto weight_of = [](float pv, float qv, int mode) -> unsigned long long {
    const float r = mode ? pv : fmaxf(__fsub_rn(pv, qv), 0.f);
    return (unsigned long long)((double)r * 1099511627776.0);
  };
  auto weight = [&](int v, int mode) -> unsigned long long {
    return weight_of(__ldg(pr + v), mode ? 0.f : __ldg(qr + v), mode);
  };
  // rows of whole 16-byte groups (the chunk below is then a multiple of 128)
  const bool vec4 = (V & 3) == 0 && ((reinterpret_cast<uintptr_t>(pr) | reinterpret_cast<uintptr_t>(qr)) & 15) == 0;

  // Warp w owns the contiguous range [w*chunk, (w+1)*chunk) of the row: its
  // lanes sum the weights there (consecutive lanes, consecutive tokens), the
  // block adds the warp sums, and only the warp whose range holds the target
  // mass scans it.  The weights are integers, so every order of adding them
  // gives the same sums and the same token.
  const int chunk = (((V + nw - 1) / nw) + 127) & ~127;
  const int c0 = min(V, w * chunk), c1 = min(V, c0 + chunk);
  // the bonus draw takes p itself (mode 1) at once
  for (int mode = a == K ? 1 : 0; mode < 2; ++mode) {
    unsigned long long mine = 0;
    if (vec4) {
      // 16-byte loads: lane l takes tokens c0 + 4(l + 32i) .. +3 (chunk is a
      // multiple of 128 here, so every group of four lies in one warp's range)
      for (int v = c0 + 4 * lane; v < c1; v += 4 * 128) {
        float4 pv[4], qv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int vj = v + 128 * j;
          pv[j] = vj < c1 ? __ldg(reinterpret_cast<const float4 *>(pr + vj)) : make_float4(0, 0, 0, 0);
          qv[j] = (vj < c1 && !mode) ? __ldg(reinterpret_cast<const float4 *>(qr + vj))
                                     : make_float4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mine += weight_of(pv[j].x, qv[j].x, mode) + weight_of(pv[j].y, qv[j].y, mode) +
                  weight_of(pv[j].z, qv[j].z, mode) + weight_of(pv[j].w, qv[j].w, mode);
        }
      }
    } else {
      for (int v = c0 + lane; v < c1; v += 4 * 32) {
        unsigned long long x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x[j] = v + 32 * j < c1 ? weight(v + 32 * j, mode) : 0ull;
        mine += (x[0] + x[1]) + (x[2] + x[3]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(FULL, mine, o);
    __syncthreads();                         // s_red is free (a previous mode read it)
    if (lane == 0) s_red[w] = mine;
    __syncthreads();
    unsigned long long total = 0;
    for (int j = 0; j < nw; ++j) total += s_red[j];
    if (total == 0) continue;
    // target mass m = floor(total * U / 2^24), total < 2^58, U < 2^24
    const unsigned long long lo = total * U, hi = __umul64hi(total, U);
    const unsigned long long m = (hi << 40) | (lo >> 24);
    // the warp whose range holds mass m: its prefix is <= m < prefix + sum
    unsigned long long before = 0;
    for (int j = 0; j < w; ++j) before += s_red[j];
    // every other warp is done (no barrier follows: the owner scans alone)
    if (!(before <= m && m < before + s_red[w])) return;
    unsigned long long run = before;
    for (int b0 = c0; b0 < c1; b0 += 4 * 32) {
      unsigned long long wq[4];              // four steps' weights, loaded together
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = b0 + 32 * j + lane;
        wq[j] = v < c1 ? weight(v, mode) : 0ull;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = b0 + 32 * j + lane;
        const unsigned long long wv = wq[j];
        unsigned long long x = wv;           // inclusive scan over the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long y = __shfl_up_sync(FULL, x, o);
          if (lane >= o) x += y;
        }
        const unsigned long long incl = run + x;
        // the token: the first v whose inclusive prefix exceeds m
        const bool hit = wv > 0 && incl > m && incl - wv <= m;
        if (hit) next_token[s] = v;
        if (__any_sync(FULL, hit)) return;
        run += __shfl_sync(FULL, x, 31);
      }
    }
    if (lane == 0) raise_status(MOE_DEV_NO_MASS);   // not reached: the warp holds mass m
    return;
  }
  // no mode had any mass (total is the same in every thread, so all reach here)
  if (tid == 0) {
    raise_status(MOE_DEV_NO_MASS);
    next_token[s] = -1;
  }
}

}  // namespace moe
