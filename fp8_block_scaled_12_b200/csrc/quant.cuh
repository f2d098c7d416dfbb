// quant.cuh -- memory-bound FP8 quantisers for sm_100a.
//
//  k_act_quant      per token, per 128-channel group ("FP8 推理提速 83.6%: DeepSeek-V3
//                   在 AMD MI250 上的完整落地指南", 运行时: act_quant); four lanes own
//                   one (row, group): 4 x 16-byte loads each, two shuffle-xor steps for
//                   the amax, scale, cast, 16-byte stores.
//  k_block_quant    one CTA per 128x128 weight block (same page, FP8 权重转换: e4m3
//                   weights with a 128x128 block scale_inv).
//  k_tensor_amax / k_tensor_cast / k_tensor_scale
//                   per-tensor scaling ("ROCm 7 ... AITER", section 1.2: one scale per
//                   tensor; "FP8 推理", Dynamic Scaling: scale = max|x| / 448): pass 1
//                   folds the tensor's amax into the caller's scale slot with an
//                   integer atomicMax, pass 2 casts (walking the tensor backwards so the
//                   tail that pass 1 left in L2 is read from L2), pass 3 stores the scale.
//
// Arithmetic shared by all three (the pages' Q(x) with the scale as a divisor,
// "量化：FP8 与混合精度推理", FP8 也需要 scale):
//   s = max(fl32(amax / Fmax), 2^-126), or for ue8m0 the power of two 2^ceil(log2 .)
//   q = cvt.rn.satfinite(fl32(x / s))  -- round to nearest even, clamp to +-Fmax.
// (GroupScale below says how the division is carried out.)
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace fp8lin {

enum : int { kE4M3 = 0, kE5M2 = 1 };
enum : int { kScaleFp32 = 0, kScaleUe8m0 = 1 };

template <int FMT>
struct FmtTraits;
template <>
struct FmtTraits<kE4M3> {
  static constexpr float kMax = 448.0f;
};
template <>
struct FmtTraits<kE5M2> {
  static constexpr float kMax = 57344.0f;
};

// bf16 pair (little-endian: element 2i in the low half) -> two fp32, exactly.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Scale of a group and what the cast needs to divide by it.  amax is finite, >= 0.
//
// fp32 scales: x / s by a correctly rounded reciprocal r = 1/s' and one residual
// correction (Markstein's division: q0 = x' r, e = x' - q0 s' exactly by FMA,
// q = q0 + e r, then the sign of x), 4 FP operations and a sign merge instead of an
// IEEE division per element.  Groups
// with s < 2^-64 first scale x and s by 2^64 (exact) so every residual that can
// decide a code stays a normal number.  For every bf16 amax and every bf16 x with
// |x| <= amax this gives the same FP8 code as fl32(x / s) rounded to nearest even:
// tests/division_identity.c restates this arithmetic on the host and compares codes.
// Its exhaustive run (every bf16 amax, 2 x 1,065,402,238 (amax, x) pairs, E4M3 and
// E5M2, 0 mismatches) is recorded in tests/golden/division_identity_exhaustive.txt;
// tests/test_division_identity.py reruns it stratified by default and exhaustively
// with FP8LIN_EXHAUSTIVE=1.  The fp32 quotients themselves may differ only where
// they are far below the smallest FP8 subnormal.
// ue8m0 scales: a multiplication by the exact power of two 2^-e, which rounds
// identically to the IEEE quotient (same exact value, one rounding).
template <int FMT, int SF>
struct GroupScale {
  float s;     // stored dequantisation multiplier
  float rinv;  // fp32: RN(1 / (s * pre)); ue8m0: 2^-e (exact)
  float pre;   // fp32: 1 or 2^64; ue8m0: unused
  float ss;    // fp32: s * pre (exact)
  __device__ __forceinline__ explicit GroupScale(float amax) {
    const float v = __fdiv_rn(amax, FmtTraits<FMT>::kMax);
    if (SF == kScaleFp32) {
      s = fmaxf(v, 1.17549435082228750797e-38f);  // 2^-126
      pre = (s < 5.42101086242752217004e-20f) ? 18446744073709551616.0f : 1.0f;   // 2^-64 : 2^64
      ss = __fmul_rn(s, pre);
      rinv = __frcp_rn(ss);
    } else {
      // e = ceil(log2 v) from the bits of v; v == 0 or subnormal -> e <= -126 -> -126
      const uint32_t b = __float_as_uint(v);
      const int ex = int(b >> 23);
      int e = (ex == 0) ? -126 : ex - 127 + ((b & 0x7FFFFFu) != 0u ? 1 : 0);
      e = max(e, -126);
      s = __uint_as_float(uint32_t(e + 127) << 23);
      rinv = __uint_as_float(uint32_t(127 - e) << 23);
      pre = 1.0f;
      ss = s;
    }
  }
  __device__ __forceinline__ float apply(float x) const {
    if (SF == kScaleFp32) {
      const float xs = __fmul_rn(x, pre);
      const float q0 = __fmul_rn(xs, rinv);
      const float e = __fmaf_rn(-q0, ss, xs);
      // the sign of the quotient is the sign of x (s > 0); the correction step would
      // turn a -0 quotient into +0
      return copysignf(__fmaf_rn(e, rinv, q0), x);
    }
    return __fmul_rn(x, rinv);
  }
};

// Two fp32 -> two FP8 codes in one 16-bit word; `lo` lands in the low byte.
template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
  uint16_t r;
  if (FMT == kE4M3)
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  else
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 8 bf16 (one uint4) -> 8 codes (one uint2) under scale sc.
template <int FMT, int SF>
__device__ __forceinline__ uint2 quant8(const uint4 v, const GroupScale<FMT, SF>& sc) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = cvt2<FMT>(sc.apply(bf16_lo(w[i])), sc.apply(bf16_hi(w[i])));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ float amax8(const uint4 v, float a) {
  a = fmaxf(a, fabsf(bf16_lo(v.x)));
  a = fmaxf(a, fabsf(bf16_hi(v.x)));
  a = fmaxf(a, fabsf(bf16_lo(v.y)));
  a = fmaxf(a, fabsf(bf16_hi(v.y)));
  a = fmaxf(a, fabsf(bf16_lo(v.z)));
  a = fmaxf(a, fabsf(bf16_hi(v.z)));
  a = fmaxf(a, fabsf(bf16_lo(v.w)));
  a = fmaxf(a, fabsf(bf16_hi(v.w)));
  return a;
}

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Byte offset of the E8M0 exponent of (row r, 32-element block g) in the tiled scale
// layout the block-scaled MMA reads (gemm_mx.cuh): 512-byte atoms of 128 rows x 4
// blocks, atom (r / 128, g / 4) at (r / 128 * nkb + g / 4) * 512, nkb = ceil(K / 128);
// inside it (r % 32) * 16 + (r % 128 / 32) * 4 + g % 4.
__host__ __device__ __forceinline__ int64_t mx_tiled_offset(int64_t r, int64_t g, int64_t nkb) {
  const int64_t rb = r >> 7, rr = r & 127, kb = g >> 2, j = g & 3;
  return (rb * nkb + kb) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + j;
}

// ---------------------------------------------------------------- act_quant
// Work item = (row m, group g) of 128 channels, owned by 4 consecutive lanes: lane
// quarter t holds channels [32t, 32t+32) of the group (four 16-byte loads), so the
// group amax needs two shuffles and each lane casts 32 values with one scale.  A
// warp takes 8 consecutive items per step (consecutive groups of a row are adjacent
// in memory: a 2 KB contiguous span), and UNROLL steps per loop iteration.
//
// MX = true is the MXFP8 variant ("ROCm 7 ... AITER", section 1.2: blocks of 32
// elements, each with its own scale; section 1.1: a shared exponent): each lane's 32
// channels are one block, so the block amax needs no shuffle; the scale follows the
// ue8m0 rule and is stored as its E8M0 byte (the fp32 exponent field of the power of
// two) in s_out, in the tiled layout of mx_tiled_offset.  Otherwise s_out = fp32
// [M][ceil(K/128)].
//
// PERMUTE = true writes each row's codes and scales to perm_k rows of the output, row
// m going to rows perm[m * perm_k + j] (MoE: a token's k expert-sorted rows), so the
// grouped GEMM reads contiguous rows and the permutation costs no separate pass.
template <int FMT, int SF, int UNROLL, bool MX = false, bool PERMUTE = false>
__global__ void __launch_bounds__(256) k_act_quant(const uint16_t* __restrict__ x, int64_t M,
                                                   int64_t K, int64_t ldx, uint8_t* __restrict__ q,
                                                   void* __restrict__ s_out, const int32_t* __restrict__ perm = nullptr,
                                                   int perm_k = 1, int64_t perm_rows = 0) {
  pdl_wait();
  pdl_trigger();
  static_assert(!MX || SF == kScaleUe8m0, "MXFP8 exponents follow the ue8m0 rule");
  const int64_t ng = (K + 127) / 128;
  const int64_t total = M * ng;
  const int lane = threadIdx.x & 31;
  const int slot = lane >> 2, qt = lane & 3;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarp = (int64_t(gridDim.x) * blockDim.x) >> 5;

  for (int64_t base = warp * (8 * UNROLL); base < total; base += nwarp * (8 * UNROLL)) {
    uint4 v[UNROLL][4];
    int64_t row[UNROLL], col[UNROLL];
    bool item_ok[UNROLL];
    // one division per warp step; the items that follow are stepped to
    const int64_t m0 = base / ng;
    const int64_t g0 = base - m0 * ng;
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t item = base + 8 * u + slot;
      int64_t m = m0, g = g0 + 8 * u + slot;
      while (g >= ng) { g -= ng; ++m; }   // at most 8*UNROLL steps
      row[u] = m;
      col[u] = g * 128 + qt * 32;
      item_ok[u] = item < total;
      const uint16_t* src = x + m * ldx + col[u];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool ok = item_ok[u] && (col[u] + 8 * j < K);
        v[u][j] = ok ? __ldg(reinterpret_cast<const uint4*>(src + 8 * j)) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) a = amax8(v[u][j], a);
      if (!MX) {
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
      }
      const GroupScale<FMT, SF> sc(a);
      if (PERMUTE && item_ok[u]) {
        uint4 c[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint2 lo = quant8<FMT, SF>(v[u][2 * h], sc);
          const uint2 hi = quant8<FMT, SF>(v[u][2 * h + 1], sc);
          c[h] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        for (int j = 0; j < perm_k; ++j) {
          // destination rows are clamped so a malformed permutation stays in bounds
          const int64_t dr = min(max(int64_t(__ldg(perm + row[u] * perm_k + j)), int64_t(0)), perm_rows - 1);
          uint8_t* dst = q + dr * K + col[u];
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (col[u] + 16 * h < K) *reinterpret_cast<uint4*>(dst + 16 * h) = c[h];
          if (qt == 0) static_cast<float*>(s_out)[dr * ng + (col[u] >> 7)] = sc.s;
        }
      } else if (item_ok[u]) {
        uint8_t* dst = q + row[u] * K + col[u];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (col[u] + 16 * h < K) {
            const uint2 lo = quant8<FMT, SF>(v[u][2 * h], sc);
            const uint2 hi = quant8<FMT, SF>(v[u][2 * h + 1], sc);
            *reinterpret_cast<uint4*>(dst + 16 * h) = make_uint4(lo.x, lo.y, hi.x, hi.y);
          }
        }
        if (MX) {
          if (col[u] < K)
            static_cast<uint8_t*>(s_out)[mx_tiled_offset(row[u], col[u] >> 5, ng)] =
                uint8_t(__float_as_uint(sc.s) >> 23);
        } else if (qt == 0) {
          static_cast<float*>(s_out)[row[u] * ng + (col[u] >> 7)] = sc.s;
        }
      }
    }
  }
}

// ------------------------------------------------------- 128x128 block quant
// One CTA (256 threads) per block: thread t covers columns (t & 15) * 8 .. +8 of
// rows (t >> 4) + 16 i, i = 0..7, so each warp reads two full 256-byte row
// segments per load instruction.
template <int FMT, int SF>
__global__ void __launch_bounds__(256) k_block_quant(const uint16_t* __restrict__ w, int64_t N,
                                                     int64_t K, uint8_t* __restrict__ q,
                                                     float* __restrict__ s_inv) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  const int64_t nbk = (K + 127) / 128;
  const int64_t bn = blockIdx.y, bk = blockIdx.x;
  const int t = threadIdx.x;
  const int64_t c = bk * 128 + (t & 15) * 8;
  const bool col_ok = c < K;
  uint4 v[8];
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = bn * 128 + (t >> 4) + 16 * i;
    const bool ok = col_ok && r < N;
    v[i] = ok ? ldg_stream(reinterpret_cast<const uint4*>(w + r * K + c)) : make_uint4(0u, 0u, 0u, 0u);
    a = amax8(v[i], a);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((t & 31) == 0) red[t >> 5] = a;
  __syncthreads();
  a = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
  const GroupScale<FMT, SF> sc(a);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = bn * 128 + (t >> 4) + 16 * i;
    if (col_ok && r < N) *reinterpret_cast<uint2*>(q + r * K + c) = quant8<FMT, SF>(v[i], sc);
  }
  if (t == 0) s_inv[bn * nbk + bk] = sc.s;
}

// ------------------------------------------------------------ per-tensor
// Pass 1: amax of n8*8 elements folded into *amax_bits (non-negative floats order
// like their bit patterns, so an unsigned atomicMax is an exact float max).
__global__ void __launch_bounds__(256) k_tensor_amax(const uint16_t* __restrict__ x, int64_t n8,
                                                     unsigned int* amax_bits) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  float a = 0.0f;
  const uint4* p = reinterpret_cast<const uint4*>(x);
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  // four independent 16-byte loads in flight per thread per step
  for (; i + 3 * stride < n8; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ldg_stream(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) a = amax8(v[u], a);
  }
  for (; i < n8; i += stride) a = amax8(ldg_stream(p + i), a);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
    atomicMax(amax_bits, __float_as_uint(a));
  }
}

// Pass 2: cast with the scale derived from the finished amax; indices run from the
// end of the tensor backwards.
template <int FMT, int SF>
__global__ void __launch_bounds__(256) k_tensor_cast(const uint16_t* __restrict__ x, int64_t n8,
                                                     const unsigned int* amax_bits,
                                                     uint8_t* __restrict__ q) {
  pdl_wait();
  pdl_trigger();
  const GroupScale<FMT, SF> sc(__uint_as_float(*amax_bits));
  const uint4* p = reinterpret_cast<const uint4*>(x);
  uint2* o = reinterpret_cast<uint2*>(q);
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n8; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ldg_stream(p + (n8 - 1 - (i + u * stride)));
#pragma unroll
    for (int u = 0; u < 4; ++u) o[n8 - 1 - (i + u * stride)] = quant8<FMT, SF>(v[u], sc);
  }
  for (; i < n8; i += stride) {
    const int64_t j = n8 - 1 - i;
    o[j] = quant8<FMT, SF>(ldg_stream(p + j), sc);
  }
}

// Pass 3: replace the amax bits with the scale.
template <int FMT, int SF>
__global__ void k_tensor_scale(unsigned int* slot) {
  pdl_wait();
  pdl_trigger();
  const GroupScale<FMT, SF> sc(__uint_as_float(*slot));
  *reinterpret_cast<float*>(slot) = sc.s;
}

// ------------------------------------------------------- delayed scaling
// One step of delayed per-tensor scaling ("ROCm 7 ... AITER", section 4.3: divide by the
// previous step's scale, clamp to +-Fmax, cast; the next scale comes from this step's
// amax; section 6: an amax history whose max sets the scale; the checklist's count of
// clipped elements).  One pass over x: k_delayed_cast casts with the stored scale,
// folds the tensor's amax into the history slot of this step (integer atomicMax on
// the bits of non-negative floats) and counts the elements whose quotient lies beyond
// +-Fmax; k_delayed_finalize turns the history into the next step's scale.

// x / s for an arbitrary positive normal fp32 scale s (the previous step's scale):
// Markstein's correction on a correctly rounded reciprocal as in GroupScale, with s
// brought into [2^-64, 2^64) by an exact power of two so the reciprocal stays normal,
// and quotients already beyond 2^100 (which saturate whatever their last bits) taken
// as they are, so an overflowing quotient never turns into NaN.  tests/
// division_delayed.c checks, for every bf16 x and scales of every binary exponent, that
// the FP8 code and the clipped flag |q| > Fmax equal those of the IEEE quotient.
struct DelayedDiv {
  float pre, ss, r;
  __device__ __forceinline__ explicit DelayedDiv(float s) {
    pre = (s < 5.42101086242752217004e-20f) ? 18446744073709551616.0f
          : (s >= 18446744073709551616.0f ? 5.42101086242752217004e-20f : 1.0f);   // 2^64 / 2^-64 / 1
    ss = __fmul_rn(s, pre);
    r = __frcp_rn(ss);
  }
  __device__ __forceinline__ float apply(float x) const {
    const float xs = __fmul_rn(x, pre);
    const float q0 = __fmul_rn(xs, r);
    if (fabsf(q0) >= 1.2676506002282294e30f) return q0;                              // 2^100
    return copysignf(__fmaf_rn(__fmaf_rn(-q0, ss, xs), r, q0), x);
  }
};

template <int FMT>
__device__ __forceinline__ uint2 delayed8(const uint4 v, const DelayedDiv& dv, uint32_t& clipped) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = dv.apply(bf16_lo(w[i])), hi = dv.apply(bf16_hi(w[i]));
    clipped += (fabsf(lo) > FmtTraits<FMT>::kMax ? 1u : 0u) + (fabsf(hi) > FmtTraits<FMT>::kMax ? 1u : 0u);
    c[i] = cvt2<FMT>(lo, hi);
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// The caller owns the slot index; it is taken modulo the history length so a corrupted
// state can never address outside the history.
__device__ __forceinline__ int delayed_slot(const int32_t* pos, int hist_len) {
  return ((*pos % hist_len) + hist_len) % hist_len;
}

template <int FMT>
__global__ void __launch_bounds__(256) k_delayed_cast(const uint16_t* __restrict__ x, int64_t n8,
                                                      const float* __restrict__ scale,
                                                      const int32_t* __restrict__ pos, int hist_len, float* history,
                                                      uint8_t* __restrict__ q, unsigned long long* n_clipped,
                                                      float* s_used) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red_a[8];
  __shared__ uint32_t red_c[8];
  const float s = *scale;
  const DelayedDiv dv(s);
  const uint4* p = reinterpret_cast<const uint4*>(x);
  uint2* o = reinterpret_cast<uint2*>(q);
  float a = 0.0f;
  uint32_t clipped = 0;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n8; i += 4 * stride) {        // four 16-byte loads in flight
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = ldg_stream(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a = amax8(v[u], a);
      o[i + u * stride] = delayed8<FMT>(v[u], dv, clipped);
    }
  }
  for (; i < n8; i += stride) {
    const uint4 v = ldg_stream(p + i);
    a = amax8(v, a);
    o[i] = delayed8<FMT>(v, dv, clipped);
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, d));
    clipped += __shfl_xor_sync(0xffffffffu, clipped, d);
  }
  if ((threadIdx.x & 31) == 0) {
    red_a[threadIdx.x >> 5] = a;
    red_c[threadIdx.x >> 5] = clipped;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t c = 0;
    for (int w = 0; w < 8; ++w) {
      a = fmaxf(a, red_a[w]);
      c += red_c[w];
    }
    atomicMax(reinterpret_cast<unsigned int*>(history + delayed_slot(pos, hist_len)), __float_as_uint(a));
    if (c) atomicAdd(n_clipped, (unsigned long long)c);
    if (blockIdx.x == 0) *s_used = s;
  }
}

// One warp: next scale = (max over the history, or this step's amax) / target, at
// least 2^-126; then clear the next slot and advance the slot index.
__global__ void k_delayed_finalize(float target, int hist_len, int algo, float* scale, int32_t* pos,
                                   float* history) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x;
  const int p = delayed_slot(pos, hist_len);
  float a = 0.0f;
  if (algo == 1) {
    for (int h = lane; h < hist_len; h += 32) a = fmaxf(a, history[h]);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, d));
  } else {
    a = history[p];
  }
  __syncwarp();
  if (lane == 0) {
    *scale = fmaxf(__fdiv_rn(a, target), 1.17549435082228750797e-38f);   // 2^-126
    const int np = (p + 1) % hist_len;
    history[np] = 0.0f;
    *pos = np;
  }
}

// ------------------------------------------------------ weight dequantisation
// The BF16 path of the DeepSeek-V3 page (运行时: weight_dequant(weight, weight.scale);
// FP8 权重转换: fp8_cast_bf16.py): w = bf16(fl32(dec(q) * scale_inv)).  FP8 codes widen
// exactly to f16 (both E4M3 and E5M2 values are f16 values), then to fp32; one fp32
// product, one round to nearest even to bf16.  A thread converts 16 codes (one 16-byte
// load, two 16-byte stores); K % 16 == 0 keeps 16 codes inside one 128-column block.
template <int FMT>
__device__ __forceinline__ float2 fp8x2_to_f32(uint16_t two) {
  uint32_t h2;
  if (FMT == kE4M3)
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
  else
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(two));
  const __half2 h = *reinterpret_cast<const __half2*>(&h2);
  return __half22float2(h);
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

template <int FMT>
__global__ void __launch_bounds__(256) k_weight_dequant(const uint8_t* __restrict__ q, const float* __restrict__ s_inv,
                                                        int64_t N, int64_t K, int block,
                                                        uint16_t* __restrict__ w) {
  pdl_wait();
  pdl_trigger();
  const int64_t k16 = K / 16, total = N * k16;
  const int64_t nbk = block > 0 ? (K + block - 1) / block : 1;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  // four 16-code chunks per thread and step, all loads issued before any conversion, so
  // each thread keeps 64 bytes of codes in flight behind the (twice larger) store stream
  constexpr int U = 4;
  for (int64_t i0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i0 < total; i0 += U * stride) {
    uint4 c[U];
    float s[U];
    int64_t off[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      off[u] = -1;
      if (i < total) {
        const int64_t n = i / k16, k = (i - n * k16) * 16;
        off[u] = n * K + k;
        s[u] = block > 0 ? __ldg(s_inv + (n / block) * nbk + k / block) : __ldg(s_inv);
        c[u] = ldg_stream(reinterpret_cast<const uint4*>(q + off[u]));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (off[u] < 0) continue;
      const uint32_t cw[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 a = fp8x2_to_f32<FMT>(uint16_t(cw[j] & 0xFFFFu));
        const float2 b = fp8x2_to_f32<FMT>(uint16_t(cw[j] >> 16));
        o[2 * j] = bf16x2_rn(__fmul_rn(a.x, s[u]), __fmul_rn(a.y, s[u]));
        o[2 * j + 1] = bf16x2_rn(__fmul_rn(b.x, s[u]), __fmul_rn(b.y, s[u]));
      }
      uint4* dst = reinterpret_cast<uint4*>(w + off[u]);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

// ------------------------------------------ act_quant of a GEMM output in registers
// The next layer's activation quantisation fused into a GEMM epilogue: 128 consecutive
// outputs of one row (one 128-channel group), already rounded to bf16 and held as fp32
// pairs, are quantised exactly as k_act_quant would quantise that bf16 row: amax,
// GroupScale, cast.  16-byte code stores; the scale goes to *s.
template <int FMT, int SF>
__device__ __forceinline__ void quant_group128(const uint64_t (&v)[64], float amax, uint8_t* q, float* s) {
  const GroupScale<FMT, SF> sc(amax);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v[c * 8 + 2 * i]));
      uint32_t lo2, hi2;
      asm("mov.b64 {%0, %1}, %2;" : "=r"(lo2), "=r"(hi2) : "l"(v[c * 8 + 2 * i + 1]));
      w[i] = cvt2<FMT>(sc.apply(__uint_as_float(lo)), sc.apply(__uint_as_float(hi))) |
             (cvt2<FMT>(sc.apply(__uint_as_float(lo2)), sc.apply(__uint_as_float(hi2))) << 16);
    }
    *reinterpret_cast<uint4*>(q + 16 * c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  *s = sc.s;
}

// Quantisation mode of a fused epilogue: code format and scale format.
enum : int { kQE4M3Fp32 = 0, kQE4M3Ue8m0 = 1, kQE5M2Fp32 = 2, kQE5M2Ue8m0 = 3 };

__device__ __forceinline__ void quant_group128_mode(int mode, const uint64_t (&v)[64], float amax, uint8_t* q,
                                                    float* s) {
  switch (mode) {
    case kQE4M3Fp32: quant_group128<kE4M3, kScaleFp32>(v, amax, q, s); break;
    case kQE4M3Ue8m0: quant_group128<kE4M3, kScaleUe8m0>(v, amax, q, s); break;
    case kQE5M2Fp32: quant_group128<kE5M2, kScaleFp32>(v, amax, q, s); break;
    default: quant_group128<kE5M2, kScaleUe8m0>(v, amax, q, s); break;
  }
}

// One value: scale of its group (computed from the group amax) and its code.
template <int FMT, int SF>
__device__ __forceinline__ uint8_t quant_one(float v, float amax, float& s) {
  const GroupScale<FMT, SF> sc(amax);
  s = sc.s;
  return uint8_t(cvt2<FMT>(sc.apply(v), 0.0f) & 0xFFu);
}

__device__ __forceinline__ uint8_t quant_one_mode(int mode, float v, float amax, float& s) {
  switch (mode) {
    case kQE4M3Fp32: return quant_one<kE4M3, kScaleFp32>(v, amax, s);
    case kQE4M3Ue8m0: return quant_one<kE4M3, kScaleUe8m0>(v, amax, s);
    case kQE5M2Fp32: return quant_one<kE5M2, kScaleFp32>(v, amax, s);
    default: return quant_one<kE5M2, kScaleUe8m0>(v, amax, s);
  }
}

}  // namespace fp8lin
