// gemm_swap.cuh -- weight-stationary block-scaled FP8 GEMM for few tokens per weight
// tile: decode (M <= 160) and the grouped MoE expert GEMM.
//
// Same operation as gemm.cuh ("FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250 上的完整落地
// 指南", 运行时: fp8_gemm; MoE: 256 routed experts, 8 active per token), with the
// operands swapped on the tensor core: the MMA's M side is 128 weight rows and its N
// side is up to NT tokens, so a handful of tokens still fills the 128-row datapath and
// each weight byte is streamed from HBM once.  A work unit is (expert e, weight
// row-block nb); units of one expert are consecutive, so the expert's token rows are
// re-read from L2 while its weights stream from HBM.  Per unit the expert's rows are
// taken in chunks of at most NT tokens and the MMA's N is set per chunk to the token
// count rounded up to 16 (the instruction descriptor is a runtime value).
//
// Roles (384 threads):
//   warp 0       TMA producer: weight tile (128 rows x 128 K) plus the chunk's token
//                rows in 32-row boxes per K-block stage.
//   warps 1-3    MMA issuers, taking K-blocks round robin.  Issuing a K-block keeps
//                its thread busy while the tensor pipe accepts the MMAs one by one, so
//                a single issuer checks its barriers only between K-blocks and the
//                pipe idles meanwhile; with three, one issuer's checks overlap the
//                others' issue.  K-blocks use separate stages and buffers, so their
//                order on the pipe does not matter.
//   warps 4-11   promotion / epilogue: thread = one weight row (tensor-memory lane),
//                warpgroup h = token columns [h*NT/2, (h+1)*NT/2).  Per K-block it loads
//                all its columns in one batch, releases the buffer, then multiplies by
//                the table's sa[token] * sw and accumulates in fp32 registers.
//
// Scales.  The work of a CTA is a sequence of segments (unit, token chunk, up to
// KB_CAP K-blocks).  A segment's scales -- sa[token][kb] for the chunk's tokens and
// sw[e][nb][kb] -- sit in one of two shared-memory tables, row kb holding the tokens
// side by side so the promotion reads four columns per 16-byte load.  The epilogue
// threads fill the table of the NEXT segment with 4-byte cp.async while they promote
// the current one, so only the first segment's load is exposed.  The chunk's sa rows
// are consecutive in memory, so each warp's copies read 128 contiguous bytes.  Once a
// segment has landed, its entries are multiplied by that K-block's sw in place.
#pragma once

#include "gemm.cuh"

namespace fp8lin {

template <int NT_, int NBUF_, int STAGES_, int KB_CAP_>
struct SwapCfg {
  static constexpr int NT = NT_, NBUF = NBUF_, STAGES = STAGES_;
  static constexpr int KB_CAP = KB_CAP_;                            // K-blocks per segment
  static constexpr int CW = NT / 2;                                 // token columns per warpgroup
  static constexpr int TROW = NT + 4;                               // table row: sa[0..NT), sw at [NT]
  static constexpr uint32_t TBUF_BYTES = uint32_t(KB_CAP) * TROW * 4;
  static constexpr uint32_t W_BYTES = 128 * kTileBytesPerRow;      // 16 KB
  static constexpr uint32_t X_BYTES = NT * kTileBytesPerRow;
  static constexpr uint32_t STAGE_BYTES = W_BYTES + X_BYTES;
  static constexpr uint32_t TMEM_COLS = (NBUF * NT <= 32) ? 32 : (NBUF * NT <= 64) ? 64
                                        : (NBUF * NT <= 128) ? 128 : (NBUF * NT <= 256) ? 256 : 512;
  static_assert(NT % 32 == 0 && NT <= 256, "token tile");
  static_assert(NBUF * NT <= 512, "tensor memory holds 512 columns");
  static_assert(CW % 16 == 0 && CW <= 96, "one-batch promotion needs CW staging registers");
  static_assert(X_BYTES % 1024 == 0, "stages stay 1024-byte aligned");
  static_assert(TBUF_BYTES % 16 == 0, "table rows keep 16-byte alignment");
};

constexpr int kSwapIssuersMax = 3;

// Register split of this kernel (same 384 x kLaunchRegs pool as gemm.cuh): its
// producer and issuer threads walk the segment sequence and need more than 48
// registers, its epilogue holds at most 96 token columns per thread.
constexpr uint32_t kSwapProducerRegs = 64;
constexpr uint32_t kSwapConsumerRegs = 216;
static_assert(128 * kSwapProducerRegs + 256 * kSwapConsumerRegs <= 384 * kLaunchRegs, "register split exceeds pool");

template <int STAGES, int NBUF>
struct alignas(8) SwapState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[NBUF];
  uint64_t tempty[NBUF];
  uint64_t seg;            // epilogue warps: segment's table loaded, previous one retired
  uint64_t red[2];         // fused output quantisation: per warpgroup, group maxima exchanged
  uint64_t drain[kSwapIssuersMax];   // abort path: each issuer's MMAs have finished
  uint32_t tmem_base;
  int abort;
};

// Fused output quantisation: group maxima per warpgroup, [2][4 warps][CW columns].
template <class C>
__host__ __device__ constexpr size_t swap_red_bytes() {
  return size_t(2) * 4 * C::CW * sizeof(float);
}

template <class C, bool QOUT = false>
constexpr size_t swap_smem_bytes() {
  return 1024 + size_t(C::STAGES) * C::STAGE_BYTES + 2 * size_t(C::TBUF_BYTES) + (QOUT ? swap_red_bytes<C>() : 0) +
         sizeof(SwapState<C::STAGES, C::NBUF>);
}

// Rows of expert e: [r0, r1).  offsets == nullptr means one group [0, M).
__device__ __forceinline__ void group_range(const GemmArgs& a, int e, int& r0, int& r1) {
  if (a.offsets == nullptr) {
    r0 = 0;
    r1 = a.M;
  } else {
    // clamp into [0, M] so a malformed offsets table can only shrink the work,
    // never address rows outside qa / sa / y
    r0 = __ldg(a.offsets + e);
    r1 = __ldg(a.offsets + e + 1);
    r1 = min(max(r1, 0), a.M);
    r0 = min(max(r0, 0), r1);
  }
}

constexpr int kSwapIssuers = kSwapIssuersMax;

// One segment of a CTA's work: unit u (expert e = u / nbn, weight row-block
// nb = u % nbn), token rows [c0, min(c0 + NT, r1)), K-blocks [seg0, seg0 + KB_CAP).
struct SwapSeg {
  int u, c0, r1, seg0;
};

// First segment of the first unit at or after u (in steps of gridDim.x) that has rows.
__device__ __forceinline__ bool swap_seg_find(const GemmArgs& a, int nbn, int num_units, int u, SwapSeg& s) {
  for (; u < num_units; u += gridDim.x) {
    int r0, r1;
    group_range(a, u / nbn, r0, r1);
    if (r0 < r1) {
      s = SwapSeg{u, r0, r1, 0};
      return true;
    }
  }
  return false;
}

// Advance to the next segment in the order the producer and the issuers walk
// (K-blocks, then token chunks, then units).
template <int NT, int KB_CAP>
__device__ __forceinline__ bool swap_seg_next(const GemmArgs& a, int nbn, int num_units, int nkb, SwapSeg& s) {
  s.seg0 += KB_CAP;
  if (s.seg0 < nkb) return true;
  s.seg0 = 0;
  s.c0 += NT;
  if (s.c0 < s.r1) return true;
  return swap_seg_find(a, nbn, num_units, s.u + gridDim.x, s);
}

// All 256 epilogue threads: start the copies of segment s's scales into the table at
// shared address `tbl`: row kk holds sa[c0 + j][seg0 + kk] at column j, sw at NT.
// Token of sorted row r (MoE scatter), clamped into [0, T) so a malformed routing
// table can never address outside the output.
__device__ __forceinline__ int moe_token(const GemmArgs& a, int r) {
  return min(max(__ldg(a.row_token + r), 0), a.moe_T - 1);
}

template <class C>
__device__ __forceinline__ void swap_seg_load(const GemmArgs& a, const SwapSeg& s, int nbn, int nkb, uint32_t tbl,
                                              int ewarp, int lane) {
  const int cnt = min(C::NT, s.r1 - s.c0);
  const int seglen = min(C::KB_CAP, nkb - s.seg0);
  const float* src = a.sa + int64_t(s.c0) * nkb + s.seg0;
  for (int j = ewarp; j < cnt; j += kEpiThreads / 32)
    for (int kk = lane; kk < seglen; kk += 32)
      cp_async4(tbl + 4u * uint32_t(kk * C::TROW + j), src + int64_t(j) * nkb + kk);
  if (ewarp == 0) {
    const float* sws = a.sw + (int64_t(s.u / nbn) * nbn + s.u % nbn) * nkb + s.seg0;
    for (int kk = lane; kk < seglen; kk += 32) cp_async4(tbl + 4u * uint32_t(kk * C::TROW + C::NT), sws + kk);
  }
}

// QOUT: the epilogue also quantises the bf16 output per (token, 128-row weight block)
// for the next layer (dense GEMM only; args.qy / args.sy / args.qmode).  A group's 128
// outputs sit one per thread across a warpgroup, so each warp reduces its 32 and the
// four warps exchange maxima through shared memory under a bounded mbarrier.
// MOE: the grouped GEMM (over expert-sorted rows, as produced by act_quant_permute)
// adds each output row r, weighted by args.row_weight[r], into
// args.moe_out[args.row_token[r]] (fp32 reductions) instead of storing y.
template <int NT, int NBUF, int STAGES, int KB_CAP, bool QOUT = false, bool MOE = false>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_swap(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const GemmArgs args) {
  using C = SwapCfg<NT, NBUF, STAGES, KB_CAP>;
  constexpr int CW = C::CW;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  float* table = reinterpret_cast<float*>(gbase + size_t(STAGES) * C::STAGE_BYTES);
  float* red = reinterpret_cast<float*>(gbase + size_t(STAGES) * C::STAGE_BYTES + 2 * size_t(C::TBUF_BYTES));
  auto* ps = reinterpret_cast<SwapState<STAGES, NBUF>*>(reinterpret_cast<uint8_t*>(red) +
                                                         (QOUT ? swap_red_bytes<C>() : 0));
  volatile int* abort = &ps->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbn = (args.N + 127) / 128;
  const int num_units = args.E * nbn;
  const int nkb = args.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ps->full[s]), 1);
      mbar_init(smem_u32(&ps->empty[s]), 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(smem_u32(&ps->tfull[b]), 1);
      mbar_init(smem_u32(&ps->tempty[b]), kEpiThreads / 32);
    }
    mbar_init(smem_u32(&ps->seg), kEpiThreads / 32);
    mbar_init(smem_u32(&ps->red[0]), 4);
    mbar_init(smem_u32(&ps->red[1]), 4);
    for (int i = 0; i < kSwapIssuers; ++i) mbar_init(smem_u32(&ps->drain[i]), 1);
    ps->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    // the first weight tiles of this CTA's first unit go to L2 while the previous
    // kernel finishes (an empty expert's prefetch is only a wasted hint)
    if (int(blockIdx.x) < num_units) {
      const int e0 = blockIdx.x / nbn, nb0 = blockIdx.x % nbn;
      for (int kb = 0; kb < STAGES && kb < nkb; ++kb) tma_prefetch_l2_2d(&tmW, kb * kBK, e0 * args.N + nb0 * 128);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ps->tmem_base), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ps->tmem_base;
  pdl_wait();

  if (warp < 4) {
    setmaxnreg_dec<kSwapProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ TMA producer
      uint32_t it = 0;
      for (int u = blockIdx.x; u < num_units && !*abort; u += gridDim.x) {
        const int e = u / nbn, nb = u % nbn;
        int r0, r1;
        group_range(args, e, r0, r1);
        for (int c0 = r0; c0 < r1 && !*abort; c0 += NT) {
          const int cnt = min(NT, r1 - c0);
          const int nbox = (cnt + 31) / 32;
          const uint32_t box_rows = 32u;
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!mbar_wait(smem_u32(&ps->empty[s]), ph ^ 1u, abort)) break;
            const uint32_t w_addr = base + s * C::STAGE_BYTES;
            const uint32_t bar = smem_u32(&ps->full[s]);
            mbar_arrive_expect_tx(bar, C::W_BYTES + uint32_t(nbox) * box_rows * kTileBytesPerRow);
            tma_load_2d(w_addr, &tmW, bar, kb * kBK, e * args.N + nb * 128);
            for (int i = 0; i < nbox; ++i)
              tma_load_2d(w_addr + C::W_BYTES + i * 32 * kTileBytesPerRow, &tmX, bar, kb * kBK, c0 + 32 * i);
          }
        }
      }
      if (*abort) {                      // every load already issued lands before the CTA exits
        for (uint32_t j = it > uint32_t(STAGES) ? it - uint32_t(STAGES) : 0u; j < it; ++j)
          mbar_drain(smem_u32(&ps->full[j % STAGES]), (j / STAGES) & 1u);
      }
      pdl_trigger();                     // every load of this CTA is issued
    } else if (warp >= 1 && warp <= kSwapIssuers && lane == 0) {
      // ------------------------------------------------ MMA issuers (round robin over K-blocks)
      const uint32_t mine = uint32_t(warp - 1);
      uint32_t it = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < num_units && !stop; u += gridDim.x) {
        const int e = u / nbn;
        int r0, r1;
        group_range(args, e, r0, r1);
        for (int c0 = r0; c0 < r1 && !stop; c0 += NT) {
          const int cnt = min(NT, r1 - c0);
          const uint32_t idesc = idesc_f8_e4m3_f32(128, uint32_t((cnt + 15) / 16 * 16));
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            if (it % kSwapIssuers != mine) continue;
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            const uint32_t b = it % NBUF;
            if (!mbar_wait(smem_u32(&ps->tempty[b]), ((it / NBUF) & 1u) ^ 1u, abort)) { stop = true; break; }
            if (!mbar_wait(smem_u32(&ps->full[s]), ph, abort)) { stop = true; break; }
            tc_fence_after();
            const uint32_t w_addr = base + s * C::STAGE_BYTES;
            const uint32_t x_addr = w_addr + C::W_BYTES;
            const uint32_t d = tmem + b * NT;
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_f8(d, sw128_kmajor_desc(w_addr + k * 32), sw128_kmajor_desc(x_addr + k * 32), idesc,
                     k > 0 ? 1u : 0u);
            mma_commit(smem_u32(&ps->empty[s]));
            mma_commit(smem_u32(&ps->tfull[b]));
          }
        }
      }
      if (*abort) {                      // the MMAs already issued finish before tensor memory is freed
        mma_commit(smem_u32(&ps->drain[mine]));
        mbar_drain(smem_u32(&ps->drain[mine]), 0u);
      }
    }
  } else {
    setmaxnreg_inc<kSwapConsumerRegs>();
    // ------------------------------------------------ promotion + epilogue
    const int ew = threadIdx.x - 128;    // 0..255
    const int ewarp = ew >> 5;           // 0..7
    const int wg = ew >> 7;              // token-column half
    const int quad = warp & 3;
    const bool out32 = args.out_fp32 != 0;
    const int col0 = wg * CW;            // first token column of this warpgroup
    const uint32_t table_s = smem_u32(table);
    const uint32_t segbar = smem_u32(&ps->seg);
    uint32_t rph = 0;                    // phases of this warpgroup's exchange barrier
    SwapSeg cur;
    bool have = swap_seg_find(args, nbn, num_units, blockIdx.x, cur);
    if (have) swap_seg_load<C>(args, cur, nbn, nkb, table_s, ewarp, lane);
    uint32_t sidx = 0, sph = 0, kbc = 0;
    bool aborted = false;
    uint64_t acc[CW / 2];                                // CW fp32 accumulators as packed pairs
    while (have) {
      const int seglen = min(KB_CAP, nkb - cur.seg0);
      if (cur.seg0 == 0) {
#pragma unroll
        for (int j = 0; j < CW / 2; ++j) acc[j] = 0ull;
      }
      // This segment's table is complete once every warp has seen its own copies
      // land; the same arrival says the warp is done with the previous segment, whose
      // buffer the next prefetch overwrites.
      cp_async_wait_all();
      __syncwarp();
      if (lane == 0) mbar_arrive(segbar);
      bool ok = mbar_wait(segbar, sph & 1u, abort);
      ++sph;
      if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
      {
        SwapSeg nxt = cur;
        if (swap_seg_next<NT, KB_CAP>(args, nbn, num_units, nkb, nxt))
          swap_seg_load<C>(args, nxt, nbn, nkb, table_s + ((sidx + 1) & 1u) * C::TBUF_BYTES, ewarp, lane);
      }
      float* tb = table + (sidx & 1u) * (C::TBUF_BYTES / 4);
      // Fold sw[kb] into the segment's rows once, so the promotion multiplies by one
      // table entry per column: entry (kk, j) becomes fl32(sa * sw), the same product
      // the promotion would form.
      {
        const int cnt = min(NT, cur.r1 - cur.c0);
        for (int i = ew; i < seglen * NT; i += kEpiThreads) {
          const int kk = i / NT, j = i - kk * NT;
          if (j < cnt) tb[kk * C::TROW + j] = __fmul_rn(tb[kk * C::TROW + j], tb[kk * C::TROW + NT]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(segbar);
      ok = mbar_wait(segbar, sph & 1u, abort);
      ++sph;
      if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
      for (int kk = 0; kk < seglen; ++kk, ++kbc) {
        const uint32_t b = kbc % NBUF;
        ok = mbar_wait(smem_u32(&ps->tfull[b]), (kbc / NBUF) & 1u, abort);
        if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t taddr = tmem + (uint32_t(quad * 32) << 16) + b * NT + col0;
        uint32_t p[CW];
#pragma unroll
        for (int c = 0; c + 32 <= CW; c += 32) tmem_ld32(taddr + c, *reinterpret_cast<uint32_t(*)[32]>(&p[c]));
        if constexpr (CW % 32 == 16)
          tmem_ld16(taddr + (CW - 16), *reinterpret_cast<uint32_t(*)[16]>(&p[CW - 16]));
        tmem_ld_wait();
        tmem_regs_ready(p);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ps->tempty[b]));
        const float* row = tb + kk * C::TROW + col0;
        // column scales in batches of 32: the loads of a batch issue back to back
#pragma unroll
        for (int j0 = 0; j0 < CW; j0 += 32) {
          constexpr int kMaxQ = 8;
          ulonglong2 sc[kMaxQ];
#pragma unroll
          for (int q = 0; q < kMaxQ; ++q)
            if (j0 + 4 * q < CW) sc[q] = *reinterpret_cast<const ulonglong2*>(row + j0 + 4 * q);
#pragma unroll
          for (int q = 0; q < kMaxQ; ++q)
            if (j0 + 4 * q < CW) {
              const int j = j0 + 4 * q;
              ffma2(acc[j / 2], p[j], p[j + 1], sc[q].x);
              ffma2(acc[j / 2 + 1], p[j + 2], p[j + 3], sc[q].y);
            }
        }
      }
      if (aborted) break;
      const int n = (cur.u % nbn) * 128 + quad * 32 + lane;   // weight row of this thread
      if constexpr (QOUT) {
        if (cur.seg0 + seglen >= nkb) {
          // the dense fused GEMM has N % 128 == 0, so every thread's row n is valid
          const int ncols = max(0, min(CW, min(NT, cur.r1 - cur.c0) - col0));
          float* rw = red + (wg * 4 + quad) * CW;
#pragma unroll
          for (int j0 = 0; j0 < CW; j0 += 8) {
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int j = j0 + i;
              const float2 f = unpack2(acc[j / 2]);
              const float v = __bfloat162float(__float2bfloat16_rn((j & 1) ? f.y : f.x));
              acc[j / 2] = (j & 1) ? pack2(f.x, v) : pack2(v, f.y);
              mx[i] = (j < ncols) ? fabsf(v) : 0.0f;
            }
#pragma unroll
            for (int d = 16; d > 0; d >>= 1)
#pragma unroll
              for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], d));
            if (lane == 0)
#pragma unroll
              for (int i = 0; i < 8; ++i) rw[j0 + i] = mx[i];
          }
          __syncwarp();
          const uint32_t rbar = smem_u32(&ps->red[wg]);
          if (lane == 0) mbar_arrive(rbar);
          bool rok = mbar_wait(rbar, rph & 1u, abort);
          ++rph;
          if (__any_sync(0xffffffffu, !rok)) { aborted = true; break; }
          const float* rg = red + wg * 4 * CW;
#pragma unroll
          for (int j = 0; j < CW; ++j) {       // unrolled: acc stays in registers
            if (j < ncols) {
              const float amax = fmaxf(fmaxf(rg[j], rg[CW + j]), fmaxf(rg[2 * CW + j], rg[3 * CW + j]));
              const float2 f = unpack2(acc[j / 2]);
              const float v = (j & 1) ? f.y : f.x;
              float sc;
              const uint8_t code = quant_one_mode(args.qmode, v, amax, sc);
              const int64_t tok = cur.c0 + col0 + j;
              args.qy[tok * args.N + n] = code;
              if (quad == 0 && lane == 0) args.sy[tok * (args.N / 128) + n / 128] = sc;
              if (args.y != nullptr)
                reinterpret_cast<__nv_bfloat16*>(args.y)[tok * args.N + n] = __float2bfloat16_rn(v);
            }
          }
          // the next group's maxima may overwrite the table once all four warps read it
          __syncwarp();
          if (lane == 0) mbar_arrive(rbar);
          rok = mbar_wait(rbar, rph & 1u, abort);
          ++rph;
          if (__any_sync(0xffffffffu, !rok)) { aborted = true; break; }
        }
      } else if (MOE && cur.seg0 + seglen >= nkb) {
        // weighted scatter-add of the expert outputs into the token-major result: the
        // warp's columns' tokens and gate weights are loaded once (one per lane) and
        // broadcast; each add is a fire-and-forget reduction
        const int ncols = max(0, min(CW, min(NT, cur.r1 - cur.c0) - col0));
        constexpr int CQ = (CW + 31) / 32;
        int tkn[CQ];
        float gwt[CQ];
#pragma unroll
        for (int q = 0; q < CQ; ++q) {
          const int jj = q * 32 + lane;
          const int r = cur.c0 + col0 + jj;
          tkn[q] = jj < ncols ? moe_token(args, r) : 0;
          gwt[q] = jj < ncols ? __ldg(args.row_weight + r) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          if (j < ncols) {                   // uniform across the warp
            const int t = __shfl_sync(0xffffffffu, tkn[j / 32], j % 32);
            const float g = __shfl_sync(0xffffffffu, gwt[j / 32], j % 32);
            const float2 f = unpack2(acc[j / 2]);
            const float v = (j & 1) ? f.y : f.x;
            if (n < args.N) red_add_f32(args.moe_out + int64_t(t) * args.N + n, __fmul_rn(g, v));
          }
        }
      } else if (cur.seg0 + seglen >= nkb && n < args.N) {
        const int ncols = max(0, min(CW, min(NT, cur.r1 - cur.c0) - col0));   // valid token columns
        const int64_t idx0 = int64_t(cur.c0 + col0) * args.N + n;
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          if (j < ncols) {
            const int64_t idx = idx0 + int64_t(j) * args.N;
            const float2 f = unpack2(acc[j / 2]);
            const float v = (j & 1) ? f.y : f.x;
            if (out32)
              reinterpret_cast<float*>(args.y)[idx] = v;
            else
              reinterpret_cast<__nv_bfloat16*>(args.y)[idx] = __float2bfloat16_rn(v);
          }
        }
      }
      have = swap_seg_next<NT, KB_CAP>(args, nbn, num_units, nkb, cur);
      ++sidx;
    }
    cp_async_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fp8lin
