// moe.cuh -- MoE routing and permutation for the grouped GEMM ("FP8 推理提速 83.6%:
// DeepSeek-V3 在 AMD MI250 上的完整落地指南", 官方配置中最关键的四个参数: 256 routed experts,
// 8 active per token; "ROCm 7 ... AITER", section 2.3: block-scale fused MoE).
//
//  k_moe_topk   one warp per token: the k largest of E scores (ties to the lower
//               expert index), then gate weights = selected scores over their fp32 sum
//               in selection order (1/k if the sum is 0).
//  k_moe_sort   one CTA: a stable counting sort of the T*k (token, j) pairs by expert.
//               Per-warp histograms in shared memory give each warp's first slot per
//               expert; each warp then places its pairs 32 at a time in order, ranking
//               equal experts inside a round with __match_any_sync.  Outputs the expert
//               offsets, each sorted row's token and weight, and each pair's row.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace fp8lin {

constexpr int kMoeMaxE = 1024;     // experts (scores per token kept in registers: 32 per lane)
constexpr int kMoeMaxK = 32;       // experts per token

template <int EPL>
__global__ void __launch_bounds__(256) k_moe_topk(const float* __restrict__ scores, int T, int E, int k,
                                                  int32_t* __restrict__ ids, float* __restrict__ w) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float v[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    const float sc = e < E ? __ldg(scores + int64_t(t) * E + e) : -INFINITY;
    v[i] = sc != sc ? -INFINITY : sc;          // a NaN score never wins; every round still picks an expert
  }
  uint32_t taken = 0;                 // bit i: v[i] already selected
  float sel_v = 0.0f;                 // lane j keeps the j-th selected score
  int sel_e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken >> i & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, d);
      const int oe = __shfl_xor_sync(0xffffffffu, be, d);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      sel_v = bv;
      sel_e = be;
    }
  }
  // fp32 sum in selection order, then one division per weight
  float sum = 0.0f;
  for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(0xffffffffu, sel_v, j));
  if (lane < k) {
    ids[int64_t(t) * k + lane] = sel_e;
    w[int64_t(t) * k + lane] = sum == 0.0f ? __fdiv_rn(1.0f, float(k)) : __fdiv_rn(sel_v, sum);
  }
}

// One CTA of 1024 threads; dynamic shared memory = 32 warps x E int32 counters.
__global__ void __launch_bounds__(1024) k_moe_sort(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                                   int T, int E, int k, int32_t* __restrict__ offsets,
                                                   int32_t* __restrict__ row_token, float* __restrict__ row_weight,
                                                   int32_t* __restrict__ token_row) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t cnt[];    // [32][E]: per-warp counts, then per-warp first slots
  __shared__ int32_t tot[kMoeMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t P = int64_t(T) * k;
  const int64_t chunk = (P + 31) / 32;
  const int64_t p0 = warp * chunk, p1 = min(P, p0 + chunk);
  for (int i = threadIdx.x; i < 32 * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  // expert ids come from k_moe_topk (always in [0, E)); clamped so a bad table stays in bounds
  for (int64_t p = p0 + lane; p < p1; p += 32) atomicAdd(&cnt[warp * E + min(max(__ldg(ids + p), 0), E - 1)], 1);
  __syncthreads();
  // per expert: total, then (after the scan over experts) each warp's first slot
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int q = 0; q < 32; ++q) s += cnt[q * E + e];
    tot[e] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      offsets[e] = run;
      const int c = tot[e];
      tot[e] = run;
      run += c;
    }
    offsets[E] = run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = tot[e];
    for (int q = 0; q < 32; ++q) {
      const int c = cnt[q * E + e];
      cnt[q * E + e] = s;
      s += c;
    }
  }
  __syncthreads();
  // place the warp's pairs in order, 32 per round
  for (int64_t base = p0; base < p1; base += 32) {
    const int64_t p = base + lane;
    const bool act = p < p1;
    const unsigned amask = __ballot_sync(0xffffffffu, act);
    if (act) {
      const int e = min(max(__ldg(ids + p), 0), E - 1);
      const unsigned peers = __match_any_sync(amask, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = cnt[warp * E + e] + rank;
      row_token[pos] = int32_t(p / k);
      row_weight[pos] = __ldg(w + p);
      token_row[p] = pos;
      __syncwarp(amask);
      if (rank == 0) cnt[warp * E + e] += __popc(peers);
    }
    __syncwarp();
  }
}

}  // namespace fp8lin
