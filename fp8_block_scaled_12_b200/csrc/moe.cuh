// moe.cuh -- MoE routing and permutation for the grouped GEMM ("FP8 推理提速 83.6%:
// DeepSeek-V3 在 AMD MI250 上的完整落地指南", 官方配置中最关键的四个参数: 256 routed experts,
// 8 active per token; "ROCm 7 ... AITER", section 2.3: block-scale fused MoE).
//
//  k_moe_topk   one warp per token: the k largest of E scores (ties to the lower
//               expert index), then gate weights = selected scores over their fp32 sum
//               in selection order (1/k if the sum is 0).
//  k_moe_count / k_moe_scan / k_moe_place
//               a stable counting sort of the T*k (token, j) pairs by expert over
//               chunks of pairs, one CTA each (below).  Outputs the expert offsets,
//               each sorted row's token and weight, and each pair's row.
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

// ----------------------------------------------------------- stable expert sort
// The T*k (token, j) pairs are cut into chunks of kMoeChunk consecutive pairs, one CTA
// each, so the scattered writes of the sorted rows come from many SMs at once.  The
// caller's workspace ws, int32 [G + 1][E] with G = ceil(T*k / kMoeChunk), carries the
// counts between the three passes:
//   k_moe_count  ws[c][e] <- number of pairs of chunk c routed to expert e
//   k_moe_scan   ws[c][e] <- pairs routed to e in chunks before c; ws[G][e] <- total of e
//   k_moe_place  expert offsets = exclusive scan of ws[G]; chunk c places its pairs at
//                offsets[e] + ws[c][e] + (pairs of e in the chunk's earlier warps and
//                rounds) + (rank among the round's lanes with the same expert), i.e. in
//                pair order within each expert.
constexpr int kMoeChunk = 512;
constexpr int kMoeSortThreads = 256;

__global__ void __launch_bounds__(kMoeSortThreads) k_moe_count(const int32_t* __restrict__ ids, int64_t P, int E,
                                                               int32_t* __restrict__ ws) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t hist[];   // [E]
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int64_t p0 = int64_t(blockIdx.x) * kMoeChunk, p1 = min(P, p0 + kMoeChunk);
  // expert ids come from k_moe_topk (always in [0, E)); clamped so a bad table stays in bounds
  for (int64_t p = p0 + threadIdx.x; p < p1; p += blockDim.x) atomicAdd(&hist[min(max(__ldg(ids + p), 0), E - 1)], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) ws[int64_t(blockIdx.x) * E + e] = hist[e];
}

// One warp per expert: exclusive prefix over the chunks, 32 chunks per step.
__global__ void __launch_bounds__(kMoeSortThreads) k_moe_scan(int G, int E, int32_t* __restrict__ ws) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x * (kMoeSortThreads / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (e >= E) return;
  int carry = 0;
  for (int c0 = 0; c0 < G; c0 += 32) {
    const int c = c0 + lane;
    const int v = c < G ? ws[int64_t(c) * E + e] : 0;
    int incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += u;
    }
    if (c < G) ws[int64_t(c) * E + e] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) ws[int64_t(G) * E + e] = carry;
}

// Chunk c = blockIdx.x (a grid of at least one CTA: CTA 0 also writes the offsets).
// Dynamic shared memory: int32 [E] offsets + [8][E] per-warp counts.  SINGLE: all pairs
// fit in one chunk (T*k <= kMoeChunk); the one CTA takes the totals from its own
// histograms and needs no workspace, so the count and scan passes are not launched.
template <bool SINGLE>
__global__ void __launch_bounds__(kMoeSortThreads) k_moe_place(const int32_t* __restrict__ ids,
                                                               const float* __restrict__ w, int64_t P, int k, int E,
                                                               int G, const int32_t* __restrict__ ws,
                                                               int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ row_token,
                                                               float* __restrict__ row_weight,
                                                               int32_t* __restrict__ token_row) {
  pdl_wait();
  pdl_trigger();
  constexpr int NW = kMoeSortThreads / 32;
  extern __shared__ int32_t sm[];
  int32_t* off = sm;                  // [E]
  int32_t* cnt = sm + E;              // [NW][E]
  __shared__ int32_t wsum[NW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NW * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  // per-warp histograms of the chunk: warp q takes pairs [c0 + q * PW, c0 + (q + 1) * PW)
  constexpr int PW = kMoeChunk / NW;
  const int64_t p0 = int64_t(blockIdx.x) * kMoeChunk + warp * PW, p1 = min(P, p0 + PW);
  int eb[PW / 32];
  float wb[PW / 32];
#pragma unroll
  for (int r = 0; r < PW / 32; ++r) {
    const int64_t p = p0 + r * 32 + lane;
    const bool act = p < p1;
    eb[r] = act ? min(max(__ldg(ids + p), 0), E - 1) : -1;
    wb[r] = act ? __ldg(w + p) : 0.0f;
  }
#pragma unroll
  for (int r = 0; r < PW / 32; ++r)
    if (eb[r] >= 0) atomicAdd(&cnt[warp * E + eb[r]], 1);
  __syncthreads();
  // expert offsets: exclusive scan of the totals (the workspace's last row, or this
  // CTA's own histograms when it holds every pair); thread t holds experts 4t .. 4t+3
  // (E <= 1024 = 4 x 256)
  int v[4], sum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 4 * threadIdx.x + i;
    int t = 0;
    if (e < E) {
      if constexpr (SINGLE) {
        for (int q = 0; q < NW; ++q) t += cnt[q * E + e];
      } else {
        t = ws[int64_t(G) * E + e];
      }
    }
    v[i] = t;
    sum += t;
  }
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int run = incl - sum;
  for (int q = 0; q < warp; ++q) run += wsum[q];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 4 * threadIdx.x + i;
    if (e < E) {
      off[e] = run;
      if (blockIdx.x == 0) offsets[e] = run;
    }
    run += v[i];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) offsets[E] = int32_t(P);
  __syncthreads();
  // first slot of each warp per expert
  const bool have = !SINGLE && int64_t(blockIdx.x) < G;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int r = off[e] + (have ? ws[int64_t(blockIdx.x) * E + e] : 0);
    for (int q = 0; q < NW; ++q) {
      const int c = cnt[q * E + e];
      cnt[q * E + e] = r;
      r += c;
    }
  }
  __syncthreads();
  // place the warp's pairs in order, 32 per round
#pragma unroll
  for (int r = 0; r < PW / 32; ++r) {
    const int64_t p = p0 + r * 32 + lane;
    const bool act = eb[r] >= 0;
    const unsigned amask = __ballot_sync(0xffffffffu, act);
    if (act) {
      const unsigned peers = __match_any_sync(amask, eb[r]);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int pos = cnt[warp * E + eb[r]] + rank;
      row_token[pos] = int32_t(p / k);
      row_weight[pos] = wb[r];
      token_row[p] = pos;
      __syncwarp(amask);
      if (rank == 0) cnt[warp * E + eb[r]] += __popc(peers);
    }
    __syncwarp();
  }
}

}  // namespace fp8lin
