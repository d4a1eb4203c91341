// route_permute.cuh -- top-k routing and the stable grouping of
// (token, slot) pairs by expert.
//
// Routing: each token activates a few experts ("mimo-tilert-1000tps-trillion-
// parameter-inference", section "万亿参数推理为什么特别难"); the selection
// rule (descending logit, ties to the lowest index) and the softmax over the
// selected logits are the library's stated reading, the pages being silent.
#pragma once
#include "common.cuh"

namespace moe {

// One warp per token.  Lane l holds logits l, l+32, ... (PER per lane).
// k rounds of a warp argmax pick the experts in rank order; the winner's
// owner lane marks it taken.  Weights: softmax of the selected logits in
// double, summed in slot order, rounded once to float.
template <int PER>
__device__ __forceinline__ void route_one_token(const float *__restrict__ logits, int t, int E,
                                                int k, int lane, int32_t *topk_idx,
                                                float *topk_w) {
  const float *row = logits + (size_t)t * E;
  float v[PER];
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(row + e) : 0.f;
    if (e >= E) taken |= 1u << i;
  }
  float my_v = 0.f;
  int my_i = -1;
  for (int r = 0; r < k; ++r) {
    float bv = 0.f;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (!((taken >> i) & 1u) && better(v[i], lane + 32 * i, bv, bi)) {
        bv = v[i];
        bi = lane + 32 * i;
      }
    }
    warp_argmax(bv, bi);
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == r) { my_v = bv; my_i = bi; }
  }
  const float vmax = __shfl_sync(FULL, my_v, 0);
  const double ex = (lane < k) ? exp((double)my_v - (double)vmax) : 0.0;
  double sum = 0.0;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(FULL, ex, j);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = my_i;
    topk_w[(size_t)t * k + lane] = (float)(ex / sum);
  }
}

template <int PER>
__global__ void __launch_bounds__(128)
route_topk_kernel(const float *__restrict__ logits, int T, int E, int k,
                  int32_t *__restrict__ topk_idx, float *__restrict__ topk_w) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  route_one_token<PER>(logits, t, E, k, lane, topk_idx, topk_w);
}

// Stable counting sort of P = T*k pairs by expert in one CTA of 1024 threads.
// Warp w owns the contiguous pair range [w*seg, (w+1)*seg).
//   pass A: per-warp, per-expert running counts; each pair's rank inside its
//           warp's range (lanes with equal experts found by __match_any_sync)
//           is parked in pair_row[p];
//   pass B: per expert, exclusive prefix over warps; block scan of the
//           per-expert totals gives expert_offsets;
//   pass C: pos = offset[e] + warp_base[w][e] + local rank.
// Dynamic shared memory: 32*E counters + E offsets (ints).
// topk_idx is read with plain loads: the fused kernel below writes it in
// the same launch.
constexpr int PERM_BATCH = 8;   // steps of 32 pairs whose ids a lane loads at once

__device__ __forceinline__ void permute_block(const int32_t *topk_idx, int P, int E,
                                              int32_t *__restrict__ expert_offsets,
                                              int32_t *__restrict__ sorted_pair,
                                              int32_t *__restrict__ pair_row, int *smem) {
  int *cnt = smem;             // [32][E]
  int *offs = smem + 32 * E;   // [E]
  __shared__ int warp_tot[32];
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int seg = (P + 31) / 32;
  const int p0 = min(P, w * seg), p1 = min(P, p0 + seg);

  for (int e = lane; e < E; e += 32) cnt[w * E + e] = 0;
  __syncwarp();
  // bits of an expert id or of the no-expert key E
  const int kbits = 32 - __clz(E);
  // pass A.  The lane's expert ids for PERM_BATCH steps of 32 pairs are
  // loaded first (independent loads in flight), then ranked step by step.
  for (int b0 = p0; b0 < p1; b0 += 32 * PERM_BATCH) {
    int ev[PERM_BATCH];
#pragma unroll
    for (int j = 0; j < PERM_BATCH; ++j) {
      const int p = b0 + 32 * j + lane;
      ev[j] = p < p1 ? topk_idx[p] : -1;
    }
#pragma unroll
    for (int j = 0; j < PERM_BATCH; ++j) {
      if (b0 + 32 * j >= p1) break;          // warp-uniform: the range has ended
      const int p = b0 + 32 * j + lane;
      int e = ev[j];
      if (p < p1 && (e < 0 || e >= E)) { raise_status(MOE_DEV_BAD_EXPERT); e = -1; }
      if (p >= p1) e = -1;
      // lanes holding the same expert: the bits of e (-1 taken as E) by
      // ballots -- cheaper than __match_any_sync here
      const unsigned key = e < 0 ? (unsigned)E : (unsigned)e;
      unsigned same = FULL;
      for (int bit = 0; bit < kbits; ++bit) {
        const unsigned bb = __ballot_sync(FULL, (key >> bit) & 1u);
        same &= ((key >> bit) & 1u) ? bb : ~bb;
      }
      int before = 0;
      if (e >= 0) before = cnt[w * E + e];
      __syncwarp();
      if (e >= 0) {
        pair_row[p] = before + __popc(same & lanemask_lt());
        if ((same & lanemask_lt()) == 0) cnt[w * E + e] = before + __popc(same);
      }
      __syncwarp();
    }
  }
  __syncthreads();
  // pass B: per expert, exclusive prefix over warps (E <= 1024, checked on
  // the host, so thread e owns expert e); then a block scan of the totals.
  const int e = threadIdx.x;
  int tot = 0;
  if (e < E) {
    for (int ww = 0; ww < 32; ++ww) {
      const int c = cnt[ww * E + e];
      cnt[ww * E + e] = tot;
      tot += c;
    }
  }
  int x = tot;  // inclusive scan of tot over the block
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(FULL, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(FULL, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int incl = x + (w > 0 ? warp_tot[w - 1] : 0);
  if (e < E) {
    offs[e] = incl - tot;
    expert_offsets[e] = incl - tot;
    if (e == E - 1) expert_offsets[E] = incl;
  }
  __syncthreads();
  // pass C (the same batching)
  for (int b0 = p0; b0 < p1; b0 += 32 * PERM_BATCH) {
    int ev[PERM_BATCH], rk[PERM_BATCH];
#pragma unroll
    for (int j = 0; j < PERM_BATCH; ++j) {
      const int p = b0 + 32 * j + lane;
      ev[j] = p < p1 ? topk_idx[p] : -1;
      rk[j] = p < p1 ? pair_row[p] : 0;
    }
#pragma unroll
    for (int j = 0; j < PERM_BATCH; ++j) {
      if (b0 + 32 * j >= p1) break;
      const int p = b0 + 32 * j + lane;
      const int e = ev[j];
      if (p < p1 && e >= 0 && e < E) {
        const int pos = offs[e] + cnt[w * E + e] + rk[j];
        sorted_pair[pos] = p;
        pair_row[p] = pos;
      }
    }
  }
}

__global__ void __launch_bounds__(1024)
permute_kernel(const int32_t *__restrict__ topk_idx, int P, int E,
               int32_t *__restrict__ expert_offsets,
               int32_t *__restrict__ sorted_pair, int32_t *__restrict__ pair_row) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int smem[];
  permute_block(topk_idx, P, E, expert_offsets, sorted_pair, pair_row, smem);
}

// Routing and permutation of a small batch in one CTA: warp w routes tokens
// w, w + 32, ...; after the barrier the block's own global writes of
// topk_idx are visible to it and the permutation runs as above.  One launch
// instead of two on the verify step's critical path.
constexpr int ROUTE_PERMUTE_MAX_T = 128;
template <int PER>
__global__ void __launch_bounds__(1024, 1)
route_permute_kernel(const float *__restrict__ logits, int T, int E, int k,
                     int32_t *topk_idx, float *__restrict__ topk_w,
                     int32_t *__restrict__ expert_offsets, int32_t *__restrict__ sorted_pair,
                     int32_t *__restrict__ pair_row) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int smem[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int t = w; t < T; t += 32) route_one_token<PER>(logits, t, E, k, lane, topk_idx, topk_w);
  __syncthreads();
  permute_block(topk_idx, T * k, E, expert_offsets, sorted_pair, pair_row, smem);
}

}  // namespace moe
