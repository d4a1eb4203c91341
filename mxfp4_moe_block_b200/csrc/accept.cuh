// accept.cuh -- acceptance of drafted blocks.
//
// Greedy: the target keeps the confirmed draft tokens and takes over at the
// first wrong one ("如何评价小米6月9日发布的MiMo-V2.5-Pro-UltraSpeed模式？",
// section "二、投机解码").  One thread-block cluster per sequence: CTA r of the
// cluster scans slice r of every row of the block (coalesced 16-byte loads),
// the per-row partial argmaxes meet in CTA 0 through distributed shared
// memory, and CTA 0 finds the first mismatch with a warp ballot.
//
// Rejection sampling ("MiMo-v2.5-Pro-UltraSpeed - infra 架构解读", section
// "数据流概览"): exact test u*q(x) < p(x) in double, first rejection by
// ballot, then an exact integer inverse-CDF draw from max(0, p - q): every
// residual weight is an integer floor(r * 2^40), so the prefix sums are
// independent of summation order and equal on every device.
#pragma once
#include <cooperative_groups.h>
#include "common.cuh"

namespace moe {
namespace cg = cooperative_groups;

constexpr int GREEDY_MAX_THREADS = 1024;
constexpr int GREEDY_ROWS = 4;       // rows scanned together
constexpr int GREEDY_CLUSTER = 16;   // CTAs per sequence (non-portable cluster size)

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

// grid (cluster_size, S), cluster (cluster_size, 1, 1), blockDim a multiple
// of 32 up to 1024.  CTA r of a sequence's cluster owns slice r of [0, V) of
// every row; a thread walks its units of that slice for up to 8 rows at once
// in increasing index order, keeping one (value, index) candidate per row;
// warps, then the CTA, then the cluster (through distributed shared memory)
// reduce the candidates with the lowest-index tie rule.  Rows hold finite
// values (a row of -inf has no candidate and never matches a draft).
__global__ void __launch_bounds__(GREEDY_MAX_THREADS, 1)
greedy_kernel(const float *__restrict__ logits, const int32_t *__restrict__ draft,
              int S, int K, int V, int32_t *__restrict__ accept_len,
              int32_t *__restrict__ next_token) {
  pdl_wait();
  pdl_trigger();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int ncta = (int)cluster.num_blocks();
  const int s = blockIdx.y;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __shared__ float part_v[32];
  __shared__ int part_i[32];
  __shared__ float red_v[GREEDY_MAX_THREADS / 32][32];
  __shared__ int red_i[GREEDY_MAX_THREADS / 32][32];

  const bool vec = (V & 3) == 0;       // rows 16-byte aligned: float4 units
  const int units = vec ? V / 4 : V;
  const int per = (units + ncta - 1) / ncta;
  const int u0 = min(units, rank * per), u1 = min(units, u0 + per);

  for (int i0 = 0; i0 < K; i0 += GREEDY_ROWS) {
    const int nr = min(GREEDY_ROWS, K - i0);
    const float *rows = logits + ((size_t)s * K + i0) * V;
    float bv[GREEDY_ROWS];
    int bi[GREEDY_ROWS];
#pragma unroll
    for (int r = 0; r < GREEDY_ROWS; ++r) { bv[r] = -INFINITY; bi[r] = -1; }
    if (vec) {
      // two strided units per iteration: 2 x GREEDY_ROWS independent
      // 16-byte loads in flight per thread, consumed in index order
      const float4 *rows4 = reinterpret_cast<const float4 *>(rows);
      const int step = blockDim.x;
      for (int u = u0 + threadIdx.x; u < u1; u += 2 * step) {
        const int u2 = u + step;
        float4 q[2][GREEDY_ROWS];
#pragma unroll
        for (int r = 0; r < GREEDY_ROWS; ++r) {
          const float4 *p = rows4 + (size_t)r * units;
          if (r < nr) q[0][r] = __ldcs(p + u);
          if (r < nr && u2 < u1) q[1][r] = __ldcs(p + u2);
        }
#pragma unroll
        for (int r = 0; r < GREEDY_ROWS; ++r)
          if (r < nr) scan_unit(q[0][r], 4 * u, bv[r], bi[r]);
        if (u2 < u1) {
#pragma unroll
          for (int r = 0; r < GREEDY_ROWS; ++r)
            if (r < nr) scan_unit(q[1][r], 4 * u2, bv[r], bi[r]);
        }
      }
    } else {
      for (int u = u0 + threadIdx.x; u < u1; u += blockDim.x) {
        float q[GREEDY_ROWS];
#pragma unroll
        for (int r = 0; r < GREEDY_ROWS; ++r)
          if (r < nr) q[r] = __ldcs(rows + (size_t)r * V + u);
#pragma unroll
        for (int r = 0; r < GREEDY_ROWS; ++r)
          if (r < nr && q[r] > bv[r]) { bv[r] = q[r]; bi[r] = u; }
      }
    }
#pragma unroll
    for (int r = 0; r < GREEDY_ROWS; ++r) {
      warp_argmax(bv[r], bi[r]);
      if (lane == 0 && r < nr) { red_v[w][i0 + r] = bv[r]; red_i[w][i0 + r] = bi[r]; }
    }
  }
  __syncthreads();
  if (threadIdx.x < K) {
    const int i = threadIdx.x;
    float v = 0.f;
    int idx = -1;
    for (int ww = 0; ww < nw; ++ww)
      if (better(red_v[ww][i], red_i[ww][i], v, idx)) { v = red_v[ww][i]; idx = red_i[ww][i]; }
    part_v[i] = v;
    part_i[i] = idx;
  }
  cluster.sync();
  if (rank == 0 && threadIdx.x < 32) {
    const int i = threadIdx.x;
    float bv = 0.f;
    int bi = -1;
    if (i < K) {
      for (int r = 0; r < ncta; ++r) {
        const float *pv = cluster.map_shared_rank(part_v, r);
        const int *pi = cluster.map_shared_rank(part_i, r);
        if (better(pv[i], pi[i], bv, bi)) { bv = pv[i]; bi = pi[i]; }
      }
    }
    int d = -1;
    if (i < K) {
      d = __ldg(draft + (size_t)s * K + i);
      if (d < 0 || d >= V) raise_status(MOE_DEV_BAD_TOKEN);
    }
    const unsigned miss = __ballot_sync(FULL, i < K && d != bi);
    const int a = miss ? __ffs(miss) - 1 : K;
    const int nt = __shfl_sync(FULL, bi, a < K ? a : 0);
    if (i == 0) {
      accept_len[s] = a;
      next_token[s] = a < K ? nt : -1;
    }
  }
  cluster.sync();   // keep every CTA's shared memory alive until CTA 0 is done
}

// One CTA per sequence.  blockDim.x is a multiple of 32, <= 1024.
__global__ void __launch_bounds__(1024)
rejection_kernel(const float *__restrict__ p, const float *__restrict__ q,
                 const int32_t *__restrict__ draft, const float *__restrict__ u_accept,
                 const float *__restrict__ u_resample, int S, int K, int V,
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
        acc = u * (double)__ldg(q + row * V + x) < (double)__ldg(p + row * V + x);
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
  if (a == K) {
    if (tid == 0) next_token[s] = -1;
    return;
  }
  const float *pr = p + ((size_t)s * K + a) * V;
  const float *qr = q + ((size_t)s * K + a) * V;
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
  for (int mode = 0; mode < 2; ++mode) {
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
