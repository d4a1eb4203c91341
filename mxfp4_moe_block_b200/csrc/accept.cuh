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
  __shared__ int s_found;

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
    if (lane == 0) {
      s_a = rej ? __ffs(rej) - 1 : K;
      s_found = 0;
    }
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
  auto weight = [&](int v, int mode) -> unsigned long long {
    const float pv = __ldg(pr + v);
    const float r = mode ? pv : fmaxf(__fsub_rn(pv, __ldg(qr + v)), 0.f);
    return (unsigned long long)((double)r * 1099511627776.0);
  };
  auto block_sum = [&](unsigned long long x) -> unsigned long long {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    __syncthreads();
    if (lane == 0) s_red[w] = x;
    __syncthreads();
    unsigned long long t = 0;
    for (int j = 0; j < nw; ++j) t += s_red[j];
    return t;
  };

  const int tile = blockDim.x;   // one element per thread per tile, coalesced
  // the bonus draw takes p itself (mode 1) at once
  for (int mode = a == K ? 1 : 0; mode < 2; ++mode) {
    unsigned long long mine = 0;
    for (int v = tid; v < V; v += tile) mine += weight(v, mode);
    const unsigned long long total = block_sum(mine);
    if (total == 0) continue;
    // target mass m = floor(total * U / 2^24), total < 2^58, U < 2^24
    const unsigned long long lo = total * U, hi = __umul64hi(total, U);
    const unsigned long long m = (hi << 40) | (lo >> 24);
    unsigned long long run = 0;   // mass of all tiles before this one
    for (int base = 0; base < V; base += tile) {
      const int v = base + tid;
      const unsigned long long wv = v < V ? weight(v, mode) : 0ull;
      // inclusive scan of wv over the block
      unsigned long long x = wv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
      }
      __syncthreads();
      if (lane == 31) s_red[w] = x;
      __syncthreads();
      unsigned long long before_w = 0, tile_sum = 0;
      for (int j = 0; j < nw; ++j) {
        if (j < w) before_w += s_red[j];
        tile_sum += s_red[j];
      }
      const unsigned long long incl = run + before_w + x;
      // the token: first v whose inclusive prefix exceeds m
      if (wv > 0 && incl > m && incl - wv <= m) {
        next_token[s] = v;
        s_found = 1;
      }
      __syncthreads();
      if (s_found) return;
      run += tile_sum;
    }
    raise_status(MOE_DEV_NO_MASS);   // not reached: m < total always finds a token
    return;
  }
  if (tid == 0) {
    raise_status(MOE_DEV_NO_MASS);
    next_token[s] = -1;
  }
}

}  // namespace moe
