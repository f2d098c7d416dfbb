// gemm.cuh -- block-scaled FP8 GEMMs on the 5th-generation tensor cores (sm_100a).
//
// Operation ("FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250 上的完整落地指南", 运行时:
// fp8_gemm(x, scale, weight, weight.scale); "LLM 推理的 FP8 混合精度工程 2026",
// section 3: FP8 products, FP32 accumulation):
//
//   y[m][n] = sum_kb sa[m][kb] * sw[n/128][kb] * P_kb[m][n],
//   P_kb[m][n] = sum_{k in K-block kb} qa[m][k] * qw[n][k]   (E4M3 x E4M3 -> fp32)
//
// Both kernels share one pipeline, warp-specialised inside a 384-thread CTA:
//   warp 0        TMA producer: one lane streams 128-deep K-blocks of both operands
//                 into a ring of shared-memory stages (128-byte swizzle, K-major).
//   warp 1        MMA issuer: one lane issues 4 x tcgen05.mma (K = 32 each) per
//                 K-block into one of two tensor-memory partial buffers, then
//                 commits to the stage's "empty" barrier and the buffer's "full" one.
//   warps 2-3     idle (their registers are handed to the epilogue).
//   warps 4-11    promotion / epilogue, two warpgroups: per K-block each thread loads
//                 its lane's partials from tensor memory (tcgen05.ld), frees the
//                 buffer and folds them into fp32 register accumulators scaled by
//                 sa * sw; after the last K-block it converts and stores the tile.
// Because the running sum lives in registers, the MMA of K-block kb+1 overlaps the
// promotion of K-block kb, and a CTA can start its next tile while it stores one.
//
//   k_gemm_wide   M-side = 128 activation rows, N-side = 256 weight rows per tile;
//                 persistent over tiles, M fastest so concurrent CTAs share weights.
//   (gemm_swap.cuh holds the weight-stationary variant used for few tokens and for
//   the grouped MoE GEMM.)
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8lin {

constexpr int kBK = 128;                  // K-block = scale block = one 128-byte row
constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;
constexpr uint32_t kTileBytesPerRow = 128;
// Register split between the producer/MMA warpgroup and the two epilogue
// warpgroups.  The kernels are compiled for kLaunchRegs registers per thread
// (launch bounds 384 x 1); the split must not exceed that pool:
// 128 * kProducerRegs + 256 * kConsumerRegs == 384 * kLaunchRegs.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kProducerRegs = 48;
constexpr uint32_t kConsumerRegs = 224;
static_assert(128 * kProducerRegs + 256 * kConsumerRegs <= 384 * kLaunchRegs, "register split exceeds pool");

struct GemmArgs {
  const float* sa;        // [rows][nkb]
  const float* sw;        // [E][nbn][nkb]
  void* y;                // [rows][N]; may be nullptr when the output is quantised (qy)
  const int32_t* offsets; // grouped: device [E+1]; nullptr = one group [0, M)
  int M;                  // activation rows (total rows for grouped)
  int N;                  // weight rows per expert
  int K;
  int E;
  int out_fp32;
  uint8_t* qy = nullptr;  // fused act_quant of the bf16 output: codes [M][N]
  float* sy = nullptr;    //   scales [M][N/128]
  int qmode = 0;          //   kQE4M3Fp32 / kQE4M3Ue8m0 / kQE5M2Fp32 / kQE5M2Ue8m0
  // MoE scatter (grouped GEMM over expert-sorted rows): the output of sorted row r is
  // added, times row_weight[r], into moe_out[row_token[r]] (fp32 [T][N]).
  const int32_t* row_token = nullptr;
  const float* row_weight = nullptr;
  float* moe_out = nullptr;
  int moe_T = 0;
};

// Shared-memory bookkeeping placed after the stage buffers.
template <int STAGES>
struct alignas(8) PipeState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;          // abort path: the issuer's MMAs have finished
  uint32_t tmem_base;
  int abort;
};

// Store 8 consecutive outputs (bf16 or fp32) for one row.
__device__ __forceinline__ void store8(void* y, bool fp32, int64_t idx, const float* v) {
  if (fp32) {
    float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + idx);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 o;
    __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 b2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 b3 = __floats2bfloat162_rn(v[6], v[7]);
    o.x = *reinterpret_cast<uint32_t*>(&b0);
    o.y = *reinterpret_cast<uint32_t*>(&b1);
    o.z = *reinterpret_cast<uint32_t*>(&b2);
    o.w = *reinterpret_cast<uint32_t*>(&b3);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(y) + idx) = o;
  }
}

// =====================================================================
// Wide kernel: tile = 128 activation rows x 256 weight rows.
// =====================================================================
template <int STAGES>
struct WideCfg {
  static constexpr int BM = 128, BN = 256;
  static constexpr uint32_t A_BYTES = BM * kTileBytesPerRow;       // 16 KB
  static constexpr uint32_t B_BYTES = BN * kTileBytesPerRow;       // 32 KB
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;                    // 512
  static constexpr size_t SMEM = 1024 + size_t(STAGES) * STAGE_BYTES + sizeof(PipeState<STAGES>);
};

// QOUT: the epilogue also quantises the bf16 output per (row, 128-column group) for
// the next layer (args.qy / args.sy / args.qmode); y is then optional.
template <int STAGES, bool QOUT = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_wide(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs args) {
  using C = WideCfg<STAGES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  PipeState<STAGES>* ps = reinterpret_cast<PipeState<STAGES>*>(gbase + size_t(STAGES) * C::STAGE_BYTES);
  volatile int* abort = &ps->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (args.M + C::BM - 1) / C::BM;
  const int num_n = (args.N + C::BN - 1) / C::BN;
  const int num_tiles = num_m * num_n;
  const int nkb = args.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ps->full[s]), 1);
      mbar_init(smem_u32(&ps->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ps->tfull[b]), 1);
      mbar_init(smem_u32(&ps->tempty[b]), kEpiThreads / 32);
    }
    mbar_init(smem_u32(&ps->drain), 1);
    ps->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (int(blockIdx.x) < num_tiles)     // first weight tiles of the first tile, to L2
      for (int kb = 0; kb < STAGES && kb < nkb; ++kb)
        tma_prefetch_l2_2d(&tmB, kb * kBK, (int(blockIdx.x) / num_m) * C::BN);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ps->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = ps->tmem_base;

  if (warp < 4) {
    setmaxnreg_dec<kProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ TMA producer
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&ps->empty[s]), ph ^ 1u, abort)) break;
          const uint32_t sa_ = base + s * C::STAGE_BYTES;
          const uint32_t bar = smem_u32(&ps->full[s]);
          mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
          tma_load_2d(sa_, &tmA, bar, kb * kBK, mb * C::BM);
          tma_load_2d(sa_ + C::A_BYTES, &tmB, bar, kb * kBK, nb * C::BN);
        }
      }
      if (*abort) {                      // every load already issued lands before the CTA exits
        for (uint32_t j = it > uint32_t(STAGES) ? it - uint32_t(STAGES) : 0u; j < it; ++j)
          mbar_drain(smem_u32(&ps->full[j % STAGES]), (j / STAGES) & 1u);
      }
      pdl_trigger();                     // every load of this CTA is issued
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_f8_e4m3_f32(C::BM, C::BN);
      uint32_t it = 0, kbc = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*abort; tile += gridDim.x) {
        for (int kb = 0; kb < nkb; ++kb, ++it, ++kbc) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          const uint32_t b = kbc & 1u;
          const uint32_t tph = (kbc >> 1) & 1u;
          if (!mbar_wait(smem_u32(&ps->tempty[b]), tph ^ 1u, abort)) break;
          if (!mbar_wait(smem_u32(&ps->full[s]), ph, abort)) break;
          tc_fence_after();
          const uint32_t a_addr = base + s * C::STAGE_BYTES;
          const uint32_t b_addr = a_addr + C::A_BYTES;
          const uint32_t d = tmem + b * C::BN;
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_f8(d, sw128_kmajor_desc(a_addr + k * 32), sw128_kmajor_desc(b_addr + k * 32), idesc,
                   k > 0 ? 1u : 0u);
          mma_commit(smem_u32(&ps->empty[s]));
          mma_commit(smem_u32(&ps->tfull[b]));
        }
      }
      if (*abort) {                      // the MMAs already issued finish before tensor memory is freed
        mma_commit(smem_u32(&ps->drain));
        mbar_drain(smem_u32(&ps->drain), 0u);
      }
    }
  } else {
    setmaxnreg_inc<kConsumerRegs>();
    // ------------------------------------------------ promotion + epilogue
    const int ew = warp - 4;             // 0..7
    const int wg = ew >> 2;              // column half of the tile
    const int quad = warp & 3;           // tensor-memory lane quadrant of this warp
    const int row_in_tile = quad * 32 + lane;
    const bool out32 = args.out_fp32 != 0;
    uint32_t kbc = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int64_t m = int64_t(mb) * C::BM + row_in_tile;
      const int n0 = nb * C::BN + wg * 128;
      const bool row_ok = m < args.M;
      const bool cols_any = n0 < args.N;
      const float* sa_row = args.sa + (row_ok ? m : 0) * nkb;
      const float* sw_blk = args.sw + int64_t(cols_any ? n0 / 128 : 0) * nkb;
      uint64_t acc[64];                  // 128 fp32 accumulators as packed pairs
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0ull;
      float sa_next = row_ok ? __ldg(sa_row) : 0.0f;
      float sw_next = cols_any ? __ldg(sw_blk) : 0.0f;
      bool aborted = false;
      for (int kb = 0; kb < nkb; ++kb, ++kbc) {
        const float scale = sa_next * sw_next;
        if (kb + 1 < nkb) {
          sa_next = row_ok ? __ldg(sa_row + kb + 1) : 0.0f;
          sw_next = cols_any ? __ldg(sw_blk + kb + 1) : 0.0f;
        }
        const uint32_t b = kbc & 1u;
        if (!mbar_wait(smem_u32(&ps->tfull[b]), (kbc >> 1) & 1u, abort)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t taddr = tmem + (uint32_t(quad * 32) << 16) + b * C::BN + wg * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t p0[32], p1[32];
          tmem_ld32(taddr + h * 64, p0);
          tmem_ld32(taddr + h * 64 + 32, p1);
          tmem_ld_wait();
          tmem_regs_ready(p0);
          tmem_regs_ready(p1);
          if (h == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ps->tempty[b]));
          }
          const uint64_t s2 = pack2(scale, scale);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            ffma2(acc[h * 32 + j], p0[2 * j], p0[2 * j + 1], s2);
            ffma2(acc[h * 32 + 16 + j], p1[2 * j], p1[2 * j + 1], s2);
          }
        }
      }
      if (aborted) break;
      if (row_ok && cols_any) {
        float amax = 0.0f;
        if constexpr (QOUT) {
          // the bf16 output is what the next layer quantises: round in place first
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const float2 f = unpack2(acc[j]);
            const float lo = __bfloat162float(__float2bfloat16_rn(f.x));
            const float hi = __bfloat162float(__float2bfloat16_rn(f.y));
            amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
            acc[j] = pack2(lo, hi);
          }
        }
        if (!QOUT || args.y != nullptr) {
#pragma unroll
          for (int j = 0; j < 128; j += 8) {
            float v[8];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float2 f = unpack2(acc[j / 2 + t]);
              v[2 * t] = f.x;
              v[2 * t + 1] = f.y;
            }
            if (n0 + j < args.N) store8(args.y, out32, m * args.N + n0 + j, v);
          }
        }
        if constexpr (QOUT)
          quant_group128_mode(args.qmode, acc, amax, args.qy + m * args.N + n0, args.sy + m * (args.N / 128) + n0 / 128);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fp8lin
