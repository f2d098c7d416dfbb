// gemm_mx.cuh -- FP8 GEMM with power-of-two block scales applied by the tensor core
// (tcgen05.mma kind::mxf8f6f4.block_scale), accumulating all of K in tensor memory.
//
// Operation.  The microscaling variant of the block-scaled GEMM ("ROCm 7 ... AITER",
// section 1.2: blocks of 32 elements with their own scale; section 1.1: MXFP8 = 8 bits
// plus a shared exponent):
//
//   y[m][n] = sum_k dec(qa[m][k]) 2^(ea(m, k/32) - 127) * dec(qw[n][k]) 2^(ew(n, k/32) - 127)
//
// with E8M0 exponent bytes ea / ew.  Because every scale is a power of two the tensor
// core applies it exactly to each product, so no per-K-block promotion is needed: the
// partial sums of all K-blocks accumulate in one fp32 tensor-memory accumulator and the
// epilogue runs once per tile.  The ue8m0 scales of the block GEMM (128-element groups,
// 128x128 weight blocks: "FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250 上的完整落地指南",
// 关键配置参数 scale_fmt ue8m0) are the same operation once each scale is replicated
// onto its four 32-element blocks (k_mx_pack_pow2).
//
// Scale layout in global memory ("tiled", the tensor core's own order): an operand of
// R rows and K columns has ceil(R/128) x ceil(K/128) atoms of 512 bytes, atom (rb, kb)
// at byte (rb * ceil(K/128) + kb) * 512; inside it row r (0..127 of the row block) and
// 32-element block j (0..3 of the K-block) sit at byte (r % 32) * 16 + (r / 32) * 4 + j.
// One atom is one bulk copy into shared memory and one tcgen05.cp (32 rows x 128 bits,
// broadcast to the four 32-lane sub-partitions) into tensor memory, where row r lands in
// lane r % 32 of every sub-partition, column base + r / 32, byte j -- the layout the
// block-scaled MMA reads, picking byte j with the sf_id fields of its descriptor.
//
// Roles (384 threads):
//   warp 0       TMA producer: per 128-deep K-block, the P tile (128 rows) and the Q tile
//                (NQ rows) with their scale atoms into a ring of stages.
//   warp 1       MMA issuer: per K-block, tcgen05.cp of the atoms into one of two
//                tensor-memory scale slots, then 4 block-scaled MMAs (K = 32 each).
//   warp 2       SWAP tiles only: a second issuer.  Issuing a K-block's copies and MMAs
//                keeps one thread busy ~440 clk, about the whole K-block period of a
//                weight stream, so the two issuers take alternate K-blocks, each into
//                its own accumulator and scale slots; the epilogue adds the two
//                accumulators (a fixed order, so the result is deterministic).
//   warps 4-11   epilogue: after a tile's last K-block, tensor memory -> registers,
//                release the accumulator, then convert and store while the next tile's
//                MMAs run.
// Orientation: WIDE tiles put 128 activation rows on the MMA's M side (P) and 256 weight
// rows on its N side (Q); SWAP tiles (few tokens) put 128 weight rows on P and up to NQ
// tokens on Q, so the weights stream from HBM once.  A Q tile may start 32, 64 or 96 rows
// into an atom: the MMA's Q scale address is then moved by that many 32-row columns.
#pragma once

#include "gemm.cuh"
#include "quant.cuh"

namespace fp8lin {

enum : int { kSfE8m0x32 = 0, kSfPow2x128 = 1 };

// Register split of this kernel: its epilogue holds one tile's accumulator slice (at
// most 128 values) rather than 128 running sums plus staged partials, so the
// producer warpgroup (TMA and MMA issue) gets more registers than in
// the promotion kernels.  128 * 104 + 256 * 200 == 384 * kLaunchRegs.
constexpr uint32_t kMxProducerRegs = 104;
constexpr uint32_t kMxConsumerRegs = 200;
static_assert(128 * kMxProducerRegs + 256 * kMxConsumerRegs <= 384 * kLaunchRegs, "register split exceeds pool");

// Device error word, bit 1: a scale given to the power-of-two layout was not a
// positive normal power of two (its mantissa would be dropped); reported by
// fp8_device_error() as FP8_ERR_INVALID_SCALE.
constexpr unsigned int kErrBadScale = 2u;

// ---------------------------------------------------------------- PTX pieces
// Block-scaled MMA, E4M3 x E4M3 -> fp32, scale factors read from tensor memory.
__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared memory -> tensor memory: 32 rows x 128 bits, written to lanes 0-31 of all
// four sub-partitions (4 consecutive 32-bit columns from taddr).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy
// reads of them (tcgen05.cp), once the consumer has synchronised with the writer.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Descriptor of a 512-byte scale atom (32 rows of 16 bytes, contiguous, no swizzle):
// start >> 4 in [0,14), leading offset 16 B (one 16-byte column) in [16,30), stride
// between 8-row core matrices 128 B in [32,46), version 1 in [46,48), layout 0.
__device__ __forceinline__ uint64_t sf_atom_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)(16 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}

// Instruction descriptor for kind::mxf8f6f4 with E8M0 scales: B scale byte id in
// [4,6), A and B E4M3 (0 in [7,10), [10,13)), K-major, N >> 3 in [17,23), scale
// format E8M0 (bit 23), M >> 4 in [24,29), A scale byte id in [29,31), K = 32.
__device__ __forceinline__ uint32_t idesc_mx_e4m3(uint32_t m, uint32_t n, uint32_t sf_id) {
  return (sf_id << 4) | ((n >> 3) << 17) | (1u << 23) | ((m >> 4) << 24) | (sf_id << 29);
}

// ------------------------------------------------------------- configuration
constexpr int gcd_c(int a, int b) { return b == 0 ? a : gcd_c(b, a % b); }

template <bool SWAP_, int NQ_, int STAGES_>
struct MxCfg {
  static constexpr bool SWAP = SWAP_;
  static constexpr int NQ = NQ_;                                  // Q-side rows per tile (MMA N)
  static constexpr int STAGES = STAGES_;                          // operand ring
  // Q atoms a tile can touch: tiles start at multiples of NQ, so at most
  // 128 - gcd(NQ, 128) rows into an atom
  static constexpr int QOFF_MAX = 128 - gcd_c(NQ, 128);
  static constexpr int QATOMS = (QOFF_MAX + NQ + 127) / 128;
  static constexpr uint32_t P_BYTES = 128 * kTileBytesPerRow;
  static constexpr uint32_t Q_BYTES = NQ * kTileBytesPerRow;
  static constexpr uint32_t STAGE_BYTES = P_BYTES + Q_BYTES;
  static constexpr uint32_t SF_BYTES = 512u * (1 + QATOMS);       // scale atoms of one stage
  static constexpr int ISSUERS = SWAP ? 2 : 1;                    // MMA issuers, one accumulator each
  static constexpr uint32_t SF_SLOT_COLS = 16;                    // tensor-memory columns per slot
  static constexpr uint32_t SF_COL0 = ISSUERS * NQ;               // after the accumulators
  static constexpr uint32_t TMEM_NEED = ISSUERS * NQ + 2 * ISSUERS * SF_SLOT_COLS;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                        : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(NQ % 32 == 0 && NQ >= 32 && NQ <= 256, "MMA N");
  static_assert(SWAP || NQ % 128 == 0, "wide Q tiles start on atom boundaries");
  static_assert(QATOMS <= 2, "a Q tile spans at most two atoms (one 16-column scale slot)");
  static_assert(QOFF_MAX % 32 == 0, "Q tiles start on 32-row columns of an atom");
  static_assert(TMEM_NEED <= 512, "tensor memory");
  static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-byte aligned");
};

template <int STAGES>
struct alignas(8) MxState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull;
  uint64_t tempty;
  uint64_t drain[2];       // abort path: each issuer's MMAs and scale copies have finished
  uint32_t tmem_base;
  int abort;
};

template <class C>
constexpr size_t mx_smem_bytes() {
  return 1024 + size_t(C::STAGES) * (C::STAGE_BYTES + C::SF_BYTES) + sizeof(MxState<C::STAGES>);
}

struct MxArgs {
  const uint8_t* sfa;   // tiled E8M0 scales of qa (M rows)
  const uint8_t* sfw;   // tiled E8M0 scales of qw (N rows)
  void* y;              // [M][N] bf16 or fp32
  int M, N, K;
  int out_fp32;
};

// Bulk copy of `bytes` contiguous bytes global -> shared, counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

template <class C>
__device__ __forceinline__ void mx_tile(const MxArgs& a, int t, int& p0, int& q0, int& qn) {
  if (!C::SWAP) {
    const int num_m = (a.M + 127) / 128;
    p0 = (t % num_m) * 128;              // activation rows, M fastest: concurrent CTAs share W tiles
    q0 = (t / num_m) * C::NQ;            // weight rows
    qn = min(C::NQ, a.N - q0);
  } else {
    const int nch = (a.M + C::NQ - 1) / C::NQ;
    p0 = (t / nch) * 128;                // weight rows
    q0 = (t % nch) * C::NQ;              // tokens
    qn = min(C::NQ, a.M - q0);
  }
}

template <class C>
__device__ __forceinline__ int mx_num_tiles(const MxArgs& a) {
  if (!C::SWAP) return ((a.M + 127) / 128) * ((a.N + C::NQ - 1) / C::NQ);
  return ((a.N + 127) / 128) * ((a.M + C::NQ - 1) / C::NQ);
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_mx(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmQ, const MxArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sf_base = base + C::STAGES * C::STAGE_BYTES;   // [STAGES][1 + QATOMS][512]
  auto* ps = reinterpret_cast<MxState<C::STAGES>*>(gbase + size_t(C::STAGES) * (C::STAGE_BYTES + C::SF_BYTES));
  volatile int* abort = &ps->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = mx_num_tiles<C>(args);
  const int nkb = args.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&ps->full[s]), 1);
      mbar_init(smem_u32(&ps->empty[s]), 1);
    }
    mbar_init(smem_u32(&ps->tfull), C::ISSUERS);
    mbar_init(smem_u32(&ps->tempty), kEpiThreads / 32);
    mbar_init(smem_u32(&ps->drain[0]), 1);
    mbar_init(smem_u32(&ps->drain[1]), 1);
    ps->abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmQ);
    if (int(blockIdx.x) < num_tiles) {   // first weight tiles of the first tile, to L2
      int p0, q0, qn;
      mx_tile<C>(args, blockIdx.x, p0, q0, qn);
      for (int kb = 0; kb < C::STAGES && kb < nkb; ++kb) {
        if (C::SWAP)
          tma_prefetch_l2_2d(&tmP, kb * kBK, p0);
        else
          tma_prefetch_l2_2d(&tmQ, kb * kBK, q0);
      }
    }
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
    setmaxnreg_dec<kMxProducerRegs>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ TMA producer
      const uint8_t* sfp = C::SWAP ? args.sfw : args.sfa;            // P-side scales
      const uint8_t* sfq = C::SWAP ? args.sfa : args.sfw;            // Q-side scales
      const int qrows = C::SWAP ? args.M : args.N;
      const int q_atoms_total = (qrows + 127) / 128;
      uint32_t it = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort; t += gridDim.x) {
        int p0, q0, qn;
        mx_tile<C>(args, t, p0, q0, qn);
        // SWAP: only the boxes of 32 tokens that hold valid rows (the MMA's N covers them)
        const int qbox = C::SWAP ? 32 : C::NQ;
        const int nqbox = C::SWAP ? (qn + 31) / 32 : 1;
        const int qa0 = q0 / 128;                                      // first Q atom row block
        const int nqa = min(C::QATOMS, min(q_atoms_total, (q0 + qn + 127) / 128) - qa0);
        const uint32_t bytes = C::P_BYTES + uint32_t(nqbox * qbox) * kTileBytesPerRow + 512u * uint32_t(1 + nqa);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(smem_u32(&ps->empty[s]), ph ^ 1u, abort)) break;
          const uint32_t pa = base + s * C::STAGE_BYTES;
          const uint32_t sfs = sf_base + s * C::SF_BYTES;
          const uint32_t bar = smem_u32(&ps->full[s]);
          mbar_arrive_expect_tx(bar, bytes);
          tma_load_2d(pa, &tmP, bar, kb * kBK, p0);
          for (int i = 0; i < nqbox; ++i)
            tma_load_2d(pa + C::P_BYTES + i * qbox * kTileBytesPerRow, &tmQ, bar, kb * kBK, q0 + i * qbox);
          bulk_load(sfs, sfp + (size_t(p0 / 128) * nkb + kb) * 512, 512u, bar);
          for (int a = 0; a < nqa; ++a)
            bulk_load(sfs + 512u * (1 + a), sfq + (size_t(qa0 + a) * nkb + kb) * 512, 512u, bar);
        }
      }
      if (*abort) {                      // every load already issued lands before the CTA exits
        for (uint32_t j = it > uint32_t(C::STAGES) ? it - uint32_t(C::STAGES) : 0u; j < it; ++j)
          mbar_drain(smem_u32(&ps->full[j % C::STAGES]), (j / C::STAGES) & 1u);
      }
      pdl_trigger();                     // every load of this CTA is issued
    } else if (warp >= 1 && warp <= C::ISSUERS && lane == 0) {
      // ------------------------------------------------ MMA issuer(s): issuer i takes the
      // K-blocks kb % ISSUERS == i of every tile into accumulator i
      const int mine = warp - 1;
      const uint32_t dacc = tmem + uint32_t(mine) * C::NQ;
      uint32_t it = 0, tc = 0, own = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < num_tiles && !stop; t += gridDim.x, ++tc) {
        int p0, q0, qn;
        mx_tile<C>(args, t, p0, q0, qn);
        const uint32_t n_mma = C::SWAP ? uint32_t((qn + 15) / 16 * 16) : uint32_t(C::NQ);
        const uint32_t qcol = uint32_t(q0 % 128) / 32;                 // Q tile's first 32-row column
        // the accumulator is free once the epilogue has drained the previous tile
        if (!mbar_wait(smem_u32(&ps->tempty), (tc & 1u) ^ 1u, abort)) break;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          if (kb % C::ISSUERS != mine) continue;
          const int s = it % C::STAGES;
          if (!mbar_wait(smem_u32(&ps->full[s]), (it / C::STAGES) & 1u, abort)) { stop = true; break; }
          tc_fence_after();
          const uint32_t slot = C::SF_COL0 + (uint32_t(mine) * 2 + (own++ & 1u)) * C::SF_SLOT_COLS;
          const uint32_t sfs = sf_base + s * C::SF_BYTES;
          tmem_cp_32x128b_x4(tmem + slot, sf_atom_desc(sfs));                          // P scales
#pragma unroll
          for (int a = 0; a < C::QATOMS; ++a)                                           // Q scales
            tmem_cp_32x128b_x4(tmem + slot + 8 + 4 * a, sf_atom_desc(sfs + 512u * (1 + a)));
          const uint32_t pa = base + s * C::STAGE_BYTES;
          const uint32_t qa = pa + C::P_BYTES;
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            const uint32_t sfid = uint32_t(k) << 30;
            mma_mx(dacc, sw128_kmajor_desc(pa + k * 32), sw128_kmajor_desc(qa + k * 32),
                   idesc_mx_e4m3(128, n_mma, uint32_t(k)), (tmem + slot) | sfid, (tmem + slot + 8 + qcol) | sfid,
                   (kb >= C::ISSUERS || k > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&ps->empty[s]));
        }
        if (stop) break;
        mma_commit(smem_u32(&ps->tfull));      // also when this issuer had no K-block (nkb == 1)
      }
      if (*abort) {                      // the MMAs already issued finish before tensor memory is freed
        mma_commit(smem_u32(&ps->drain[mine]));
        mbar_drain(smem_u32(&ps->drain[mine]), 0u);
      }
    }
  } else {
    setmaxnreg_inc<kMxConsumerRegs>();
    // ------------------------------------------------ epilogue
    const int ew = warp - 4;             // 0..7
    const int wg = ew >> 2;              // column half of the tile
    const int quad = warp & 3;           // tensor-memory lane quadrant of this warp
    constexpr int CW = C::NQ / 2;        // accumulator columns per thread
    const bool out32 = args.out_fp32 != 0;
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tc) {
      int p0, q0, qn;
      mx_tile<C>(args, t, p0, q0, qn);
      const bool ok = mbar_wait(smem_u32(&ps->tfull), tc & 1u, abort);
      if (__any_sync(0xffffffffu, !ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (uint32_t(quad * 32) << 16) + wg * CW;
      uint32_t v[CW];
#pragma unroll
      for (int c = 0; c + 32 <= CW; c += 32) tmem_ld32(taddr + c, *reinterpret_cast<uint32_t(*)[32]>(&v[c]));
      if constexpr (CW % 32 == 16) tmem_ld16(taddr + (CW - 16), *reinterpret_cast<uint32_t(*)[16]>(&v[CW - 16]));
      tmem_ld_wait();
      tmem_regs_ready(v);
      if (C::ISSUERS == 2 && nkb > 1) {
        // y = fl32(acc0 + acc1): the second issuer's accumulator, 16 columns at a time
#pragma unroll
        for (int c = 0; c < CW; c += 16) {
          uint32_t u[16];
          tmem_ld16(taddr + C::NQ + c, u);
          tmem_ld_wait();
          tmem_regs_ready(u);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[c + i] = __float_as_uint(__fadd_rn(__uint_as_float(v[c + i]), __uint_as_float(u[i])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ps->tempty));
      const int prow = p0 + quad * 32 + lane;          // P row of this thread
      const int qc0 = wg * CW;                         // first Q column of this thread
      if (!C::SWAP) {
        // y[m = prow][n = q0 + qc0 + j]
        if (prow < args.M) {
#pragma unroll
          for (int j = 0; j < CW; j += 8) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(v[j + i]);
            if (qc0 + j < qn) store8(args.y, out32, int64_t(prow) * args.N + q0 + qc0 + j, f);
          }
        }
      } else {
        // y[token = q0 + qc0 + j][n = prow]: a warp writes 32 consecutive outputs per token
        if (prow < args.N) {
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            if (qc0 + j < qn) {
              const int64_t idx = int64_t(q0 + qc0 + j) * args.N + prow;
              const float f = __uint_as_float(v[j]);
              if (out32)
                reinterpret_cast<float*>(args.y)[idx] = f;
              else
                reinterpret_cast<__nv_bfloat16*>(args.y)[idx] = __float2bfloat16_rn(f);
            }
          }
        }
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

// ---------------------------------------------------------------- scale packing
// fp32 power-of-two scales (the block GEMM's ue8m0 layouts) -> tiled E8M0 bytes.  One
// thread per (row, K-block): s[row / row_block][kb] is replicated onto the row's four
// 32-element blocks of that K-block as the E8M0 byte (the fp32 exponent field).  A
// scale that is not a positive normal power of two raises kErrBadScale.
__global__ void __launch_bounds__(256) k_mx_pack_pow2(const float* __restrict__ s, int64_t rows, int64_t nkb,
                                                      int row_block, uint8_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * nkb) return;
  const int64_t r = i / nkb, kb = i - r * nkb;
  const uint32_t b = __float_as_uint(__ldg(s + (r / row_block) * nkb + kb));
  if ((b & 0x807FFFFFu) != 0u || (b >> 23) == 0u || (b >> 23) == 255u) atomicOr(&g_device_error, kErrBadScale);
  const int64_t o = mx_tiled_offset(r, kb * 4, nkb);
  *reinterpret_cast<uint32_t*>(out + o) = (b >> 23) * 0x01010101u;   // bytes j = 0..3 of the K-block
}

}  // namespace fp8lin
