// fp8lin.cu -- the C ABI (include/fp8lin.h): argument checks, TMA descriptors and
// kernel launches.  The whole library is this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/fp8lin.h"
#include "gemm.cuh"
#include "gemm_mx.cuh"
#include "gemm_swap.cuh"
#include "moe.cuh"
#include "ptx.cuh"
#include "quant.cuh"

using namespace fp8lin;

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FP8_OK;
  return FP8_ERR_CUDA;
}

// Streaming multiprocessors of the current device (cached per device).
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Blocks of `kern` (`threads` threads, no dynamic shared memory) that one SM holds at
// once -- its register count decides it -- from the occupancy calculator, once per
// device; `cache` belongs to the calling launch function.
template <typename K>
int resident_blocks(std::atomic<int> (&cache)[64], K kern, int threads) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = -1;
  if (dev >= 0) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, 0) != cudaSuccess || n <= 0) n = 1;
  if (dev >= 0) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major byte matrix [rows][cols] (row stride = cols bytes),
// box = box_rows x 128 bytes, 128-byte swizzle, out-of-range reads give zeros.
bool make_map_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------- GEMM launches
constexpr int kWideStages = 4;

// Every kernel is launched with programmatic stream serialisation: the runtime may
// schedule it while the previous kernel on the stream is finishing (its prologue --
// barrier set-up, tensor-memory allocation, descriptor and weight prefetch -- then
// overlaps that kernel's tail), and the kernel waits for the previous one (pdl_wait)
// before it touches operand data.  Preceding work that is not a kernel (a memset, a
// copy) orders the launch as usual.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// The warpgroup register split inside the GEMM kernels (setmaxnreg) draws on the
// registers the CTA was launched with; refuse to launch a build whose register
// count differs from the one the split was sized for (it could never satisfy
// the increase).
template <typename K>
bool launch_regs_ok(K kern) {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
  return fa.numRegs == int(kLaunchRegs);
}

// The register check and the dynamic shared-memory limit of a warp-specialised kernel
// persist in the device's context, so they run on its first launch per device only
// (`ready`: one bit per device, owned by the calling launch function; devices past 63
// are set up on every launch).
template <typename K>
int kernel_setup(std::atomic<uint64_t>& ready, K kern, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8_ERR_CUDA;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0u;
  if (bit != 0u && (ready.load(std::memory_order_acquire) & bit) != 0u) return FP8_OK;
  if (!launch_regs_ok(kern)) return FP8_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return FP8_ERR_CUDA;
  ready.fetch_or(bit, std::memory_order_acq_rel);
  return FP8_OK;
}

template <int NT, int NBUF, int STAGES, int KB_CAP, bool QOUT = false, bool MOE = false>
int launch_swap(const void* qa, const void* qw, const GemmArgs& a, int64_t w_rows, cudaStream_t st) {
  using C = SwapCfg<NT, NBUF, STAGES, KB_CAP>;
  constexpr size_t smem = swap_smem_bytes<C, QOUT>();
  static_assert(smem <= 232448, "dynamic shared memory of one CTA (227 KB)");
  CUtensorMap mw, mx;
  if (!make_map_u8(&mw, qw, uint64_t(w_rows), uint64_t(a.K), 128)) return FP8_ERR_CUDA;
  if (!make_map_u8(&mx, qa, uint64_t(a.M > 0 ? a.M : 1), uint64_t(a.K), 32)) return FP8_ERR_CUDA;
  auto kern = k_gemm_swap<NT, NBUF, STAGES, KB_CAP, QOUT, MOE>;
  static std::atomic<uint64_t> ready{0};
  if (const int st_ = kernel_setup(ready, kern, smem)) return st_;
  const int nbn = (a.N + 127) / 128;
  const int64_t units = int64_t(a.E) * nbn;
  const int grid = int(units < num_sms() ? units : num_sms());
  return cuda_status(launch(kern, grid, kThreads, smem, st, mw, mx, a));
}

// Block-scaled (power-of-two) GEMM on the tensor core's scale path.  WIDE: P = 128
// activation rows, Q = 256 weight rows; SWAP (few tokens): P = 128 weight rows, Q =
// up to NQ tokens in 32-row boxes.
template <bool SWAP, int NQ, int STAGES>
int launch_mx(const void* qa, const void* qw, const MxArgs& a, cudaStream_t st) {
  using C = MxCfg<SWAP, NQ, STAGES>;
  constexpr size_t smem = mx_smem_bytes<C>();
  static_assert(smem <= 232448, "dynamic shared memory of one CTA (227 KB)");
  CUtensorMap mp, mq;
  const void* pp = SWAP ? qw : qa;
  const void* qp = SWAP ? qa : qw;
  const uint64_t prow = uint64_t(SWAP ? a.N : a.M), qrow = uint64_t(SWAP ? a.M : a.N);
  if (!make_map_u8(&mp, pp, prow, uint64_t(a.K), 128)) return FP8_ERR_CUDA;
  if (!make_map_u8(&mq, qp, qrow, uint64_t(a.K), SWAP ? 32u : uint32_t(NQ))) return FP8_ERR_CUDA;
  auto kern = k_gemm_mx<C>;
  static std::atomic<uint64_t> ready{0};
  if (const int st_ = kernel_setup(ready, kern, smem)) return st_;
  const int64_t tiles = SWAP ? int64_t((a.N + 127) / 128) * ((a.M + NQ - 1) / NQ)
                             : int64_t((a.M + 127) / 128) * ((a.N + NQ - 1) / NQ);
  const int grid = int(tiles < num_sms() ? tiles : num_sms());
  return cuda_status(launch(kern, grid, kThreads, smem, st, mp, mq, a));
}

template <bool QOUT = false>
int launch_wide(const void* qa, const void* qw, const GemmArgs& a, cudaStream_t st) {
  using C = WideCfg<kWideStages>;
  CUtensorMap ma, mb;
  if (!make_map_u8(&ma, qa, uint64_t(a.M), uint64_t(a.K), C::BM)) return FP8_ERR_CUDA;
  if (!make_map_u8(&mb, qw, uint64_t(a.N), uint64_t(a.K), C::BN)) return FP8_ERR_CUDA;
  auto kern = k_gemm_wide<kWideStages, QOUT>;
  static std::atomic<uint64_t> ready{0};
  if (const int st_ = kernel_setup(ready, kern, size_t(C::SMEM))) return st_;
  const int64_t tiles = int64_t((a.M + C::BM - 1) / C::BM) * ((a.N + C::BN - 1) / C::BN);
  const int grid = int(tiles < num_sms() ? tiles : num_sms());
  return cuda_status(launch(kern, grid, kThreads, C::SMEM, st, ma, mb, a));
}

// ------------------------------------------------------ MoE routing
int launch_moe_route(const float* scores, int64_t T, int64_t E, int64_t k, int32_t* ids, float* w, int32_t* offsets,
                     int32_t* row_token, float* row_weight, int32_t* token_row, int32_t* ws, cudaStream_t st) {
  const int64_t P = T * k;
  const int G = int((P + kMoeChunk - 1) / kMoeChunk);
  if (T > 0) {
    const unsigned blocks = unsigned((T * 32 + 255) / 256);
    const cudaError_t e = E <= 256 ? launch(k_moe_topk<8>, blocks, 256, 0, st, scores, int(T), int(E), int(k), ids, w)
                                   : launch(k_moe_topk<32>, blocks, 256, 0, st, scores, int(T), int(E), int(k), ids, w);
    if (e != cudaSuccess) return FP8_ERR_CUDA;
  }
  const size_t smem = size_t(1 + kMoeSortThreads / 32) * size_t(E) * sizeof(int32_t);
  if (G <= 1)   // every pair in one chunk: one CTA sorts them all
    return cuda_status(launch(k_moe_place<true>, 1, kMoeSortThreads, smem, st, static_cast<const int32_t*>(ids),
                              static_cast<const float*>(w), P, int(k), int(E), G, static_cast<const int32_t*>(ws),
                              offsets, row_token, row_weight, token_row));
  if (launch(k_moe_count, unsigned(G), kMoeSortThreads, size_t(E) * 4, st, static_cast<const int32_t*>(ids), P,
             int(E), ws) != cudaSuccess)
    return FP8_ERR_CUDA;
  const unsigned sblocks = unsigned((E + kMoeSortThreads / 32 - 1) / (kMoeSortThreads / 32));
  if (launch(k_moe_scan, sblocks, kMoeSortThreads, 0, st, G, int(E), ws) != cudaSuccess) return FP8_ERR_CUDA;
  return cuda_status(launch(k_moe_place<false>, unsigned(G), kMoeSortThreads, smem, st,
                            static_cast<const int32_t*>(ids), static_cast<const float*>(w), P, int(k), int(E), G,
                            static_cast<const int32_t*>(ws), offsets, row_token, row_weight, token_row));
}

// ------------------------------------------------------ quantiser launches
// Grid of the grid-stride quantisers (k_act_quant and its MX / permute variants):
// every warp takes the same number of steps (8 * U groups each).  With `one_wave` the
// grid is the blocks the SMs hold at once (`resident` per SM: 3 at these kernels' 80
// registers), so no block waits for a second wave; otherwise it is sized for 8 blocks
// per SM and runs as two to three such waves.  Measured on B200s (bit-identical outputs): one
// wave makes the MX kernel 8% faster at 16384 x 7168; for act_quant it is 5% slower
// with fp32 scales at 4096 x 7168, 12% slower for the permuted variant and mixed with
// ue8m0 scales (+3% at 4096 rows, -1.4% at 16384), so those keep the waves.
inline int64_t stride_blocks(int64_t steps, int resident, bool one_wave) {
  const int64_t max_warps = int64_t(num_sms()) * (one_wave ? resident : 8) * 8;
  const int64_t per_warp = (steps + max_warps - 1) / max_warps;
  const int64_t warps = (steps + per_warp - 1) / per_warp;
  return (warps + 7) / 8;
}

template <int FMT, int SF>
int launch_act_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, float* s,
                     cudaStream_t st) {
  constexpr int U = 2;
  auto kern = k_act_quant<FMT, SF, U>;
  static std::atomic<int> occ[64];
  const int64_t steps = (M * ((K + 127) / 128) + 8 * U - 1) / (8 * U);
  const int64_t blocks = stride_blocks(steps, resident_blocks(occ, kern, 256), false);
  return cuda_status(launch(kern, unsigned(blocks), 256, 0, st, x, M, K, ldx, q, s,
                            static_cast<const int32_t*>(nullptr), 1, int64_t(0)));
}

template <int FMT, int SF>
int launch_act_quant_permute(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, float* s,
                             const int32_t* perm, int k, cudaStream_t st) {
  constexpr int U = 2;
  auto kern = k_act_quant<FMT, SF, U, false, true>;
  static std::atomic<int> occ[64];
  const int64_t steps = (M * ((K + 127) / 128) + 8 * U - 1) / (8 * U);
  const int64_t blocks = stride_blocks(steps, resident_blocks(occ, kern, 256), false);
  return cuda_status(launch(kern, unsigned(blocks), 256, 0, st, x, M, K, ldx, q, s, perm, k, M * k));
}

template <int FMT>
int launch_mx_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, uint8_t* e8,
                    cudaStream_t st) {
  constexpr int U = 2;
  auto kern = k_act_quant<FMT, kScaleUe8m0, U, true>;
  static std::atomic<int> occ[64];
  const int64_t steps = (M * ((K + 127) / 128) + 8 * U - 1) / (8 * U);
  const int64_t blocks = stride_blocks(steps, resident_blocks(occ, kern, 256), true);
  return cuda_status(launch(kern, unsigned(blocks), 256, 0, st, x, M, K, ldx, q, e8,
                            static_cast<const int32_t*>(nullptr), 1, int64_t(0)));
}

template <int FMT>
int launch_dequant(const uint8_t* q, const float* s, int64_t N, int64_t K, int block, uint16_t* w, cudaStream_t st) {
  const int64_t total = N * (K / 16);
  int64_t blocks = (total + 255) / 256;
  static std::atomic<int> occ[64];
  const int64_t cap = int64_t(num_sms()) * resident_blocks(occ, k_weight_dequant<FMT>, 256);
  if (blocks > cap) blocks = cap;
  return cuda_status(launch(k_weight_dequant<FMT>, unsigned(blocks), 256, 0, st, q, s, N, K, block, w));
}

template <int FMT, int SF>
int launch_block_quant(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s, cudaStream_t st) {
  dim3 grid(unsigned((K + 127) / 128), unsigned((N + 127) / 128));
  return cuda_status(launch(k_block_quant<FMT, SF>, grid, 256, 0, st, w, N, K, q, s));
}

template <int FMT, int SF>
int launch_tensor_quant(const uint16_t* x, int64_t n, uint8_t* q, float* s, cudaStream_t st) {
  const int64_t n8 = n / 8;
  int64_t blocks = (n8 + 255) / 256;
  const int64_t cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  unsigned int* slot = reinterpret_cast<unsigned int*>(s);
  cudaError_t e = cudaMemsetAsync(slot, 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return FP8_ERR_CUDA;
  if (launch(k_tensor_amax, unsigned(blocks), 256, 0, st, x, n8, slot) != cudaSuccess) return FP8_ERR_CUDA;
  if (launch(k_tensor_cast<FMT, SF>, unsigned(blocks), 256, 0, st, x, n8, slot, q) != cudaSuccess) return FP8_ERR_CUDA;
  return cuda_status(launch(k_tensor_scale<FMT, SF>, 1, 1, 0, st, slot));
}

// One warp whose mbarrier never completes: the bounded wait that every pipelined
// wait of the GEMM kernels uses gives up after limit_ns, records the timeout in the
// device error word and the kernel returns normally.
__global__ void k_selftest_wait(uint64_t limit_ns) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0u, &abort_flag, limit_ns);
  __syncwarp();
}

}  // namespace

// =====================================================================
// C ABI
// =====================================================================
extern "C" {

const char* fp8_status_string(int status) {
  switch (status) {
    case FP8_OK: return "ok";
    case FP8_ERR_INVALID_ARG: return "invalid argument";
    case FP8_ERR_SHAPE: return "unsupported shape";
    case FP8_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case FP8_ERR_UNSUPPORTED: return "unsupported option";
    case FP8_ERR_CUDA: return "CUDA error";
    case FP8_ERR_TIMEOUT: return "device wait timed out";
    case FP8_ERR_INVALID_SCALE: return "a scale given as a power of two is not one";
    default: return "unknown status";
  }
}

int fp8_act_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int group, int fmt, int scale_fmt,
                  void* q, float* s, void* stream) {
  if (M < 0 || K <= 0 || ldx < K) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (scale_fmt != FP8_SCALE_FP32 && scale_fmt != FP8_SCALE_UE8M0) return FP8_ERR_INVALID_ARG;
  if (group != 128) return FP8_ERR_UNSUPPORTED;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (M == 0) return FP8_OK;
  if (!x || !q || !s) return FP8_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4)) return FP8_ERR_ALIGNMENT;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  uint8_t* qb = static_cast<uint8_t*>(q);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fmt == FP8_E4M3)
    return scale_fmt == FP8_SCALE_FP32 ? launch_act_quant<kE4M3, kScaleFp32>(xb, M, K, ldx, qb, s, st)
                                       : launch_act_quant<kE4M3, kScaleUe8m0>(xb, M, K, ldx, qb, s, st);
  return scale_fmt == FP8_SCALE_FP32 ? launch_act_quant<kE5M2, kScaleFp32>(xb, M, K, ldx, qb, s, st)
                                     : launch_act_quant<kE5M2, kScaleUe8m0>(xb, M, K, ldx, qb, s, st);
}

int fp8_weight_quant(const void* w, int64_t N, int64_t K, int block, int fmt, int scale_fmt, void* q,
                     float* s_inv, void* stream) {
  if (N < 0 || K <= 0) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (scale_fmt != FP8_SCALE_FP32 && scale_fmt != FP8_SCALE_UE8M0) return FP8_ERR_INVALID_ARG;
  if (block != 128 && block != 0) return FP8_ERR_UNSUPPORTED;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (N == 0) return FP8_OK;
  if (!w || !q || !s_inv) return FP8_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(s_inv, 4)) return FP8_ERR_ALIGNMENT;
  const uint16_t* wb = static_cast<const uint16_t*>(w);
  uint8_t* qb = static_cast<uint8_t*>(q);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (block == 128) {
    if (fmt == FP8_E4M3)
      return scale_fmt == FP8_SCALE_FP32 ? launch_block_quant<kE4M3, kScaleFp32>(wb, N, K, qb, s_inv, st)
                                         : launch_block_quant<kE4M3, kScaleUe8m0>(wb, N, K, qb, s_inv, st);
    return scale_fmt == FP8_SCALE_FP32 ? launch_block_quant<kE5M2, kScaleFp32>(wb, N, K, qb, s_inv, st)
                                       : launch_block_quant<kE5M2, kScaleUe8m0>(wb, N, K, qb, s_inv, st);
  }
  const int64_t n = N * K;
  if (fmt == FP8_E4M3)
    return scale_fmt == FP8_SCALE_FP32 ? launch_tensor_quant<kE4M3, kScaleFp32>(wb, n, qb, s_inv, st)
                                       : launch_tensor_quant<kE4M3, kScaleUe8m0>(wb, n, qb, s_inv, st);
  return scale_fmt == FP8_SCALE_FP32 ? launch_tensor_quant<kE5M2, kScaleFp32>(wb, n, qb, s_inv, st)
                                     : launch_tensor_quant<kE5M2, kScaleUe8m0>(wb, n, qb, s_inv, st);
}

static int check_gemm_common(const void* qa, const float* sa, const void* qw, const float* sw, int64_t M,
                             int64_t N, int64_t K, int out_dtype, void* y) {
  if (M < 0 || N <= 0 || K <= 0) return FP8_ERR_INVALID_ARG;
  if (out_dtype != FP8_OUT_BF16 && out_dtype != FP8_OUT_FP32) return FP8_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 16 != 0) return FP8_ERR_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return FP8_ERR_SHAPE;
  if (!qw || !sw) return FP8_ERR_INVALID_ARG;
  if (M > 0 && (!qa || !sa || !y)) return FP8_ERR_INVALID_ARG;
  if (!aligned(qw, 16) || !aligned(sw, 4)) return FP8_ERR_ALIGNMENT;
  if (M > 0 && (!aligned(qa, 16) || !aligned(sa, 4) || !aligned(y, 16))) return FP8_ERR_ALIGNMENT;
  return FP8_OK;
}

int fp8_block_gemm(const void* qa, const float* sa, const void* qw, const float* sw, int64_t M, int64_t N,
                   int64_t K, int out_dtype, void* y, void* stream) {
  int rc = check_gemm_common(qa, sa, qw, sw, M, N, K, out_dtype, y);
  if (rc != FP8_OK) return rc;
  if (M == 0) return FP8_OK;
  GemmArgs a{sa, sw, y, nullptr, int(M), int(N), int(K), 1, out_dtype == FP8_OUT_FP32 ? 1 : 0};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M <= 64) return launch_swap<64, 4, 8, 56>(qa, qw, a, N, st);
  if (M <= 160) return launch_swap<160, 3, 5, 28>(qa, qw, a, N, st);
  return launch_wide(qa, qw, a, st);
}

int fp8_block_gemm_quant(const void* qa, const float* sa, const void* qw, const float* sw, int64_t M, int64_t N,
                         int64_t K, void* y, int fmt, int scale_fmt, void* qy, float* sy, void* stream) {
  int rc = check_gemm_common(qa, sa, qw, sw, M, N, K, FP8_OUT_BF16, M > 0 ? qy : nullptr);
  if (rc != FP8_OK) return rc;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (scale_fmt != FP8_SCALE_FP32 && scale_fmt != FP8_SCALE_UE8M0) return FP8_ERR_INVALID_ARG;
  if (N % 128 != 0) return FP8_ERR_SHAPE;                    // whole 128-channel groups
  if (M == 0) return FP8_OK;
  if (!qy || !sy) return FP8_ERR_INVALID_ARG;
  if (!aligned(qy, 16) || !aligned(sy, 4) || (y && !aligned(y, 16))) return FP8_ERR_ALIGNMENT;
  GemmArgs a{sa, sw, y, nullptr, int(M), int(N), int(K), 1, 0};
  a.qy = static_cast<uint8_t*>(qy);
  a.sy = sy;
  a.qmode = (fmt == FP8_E4M3 ? 0 : 2) + (scale_fmt == FP8_SCALE_UE8M0 ? 1 : 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M <= 64) return launch_swap<64, 4, 8, 56, true>(qa, qw, a, N, st);
  if (M <= 160) return launch_swap<160, 3, 5, 28, true>(qa, qw, a, N, st);
  return launch_wide<true>(qa, qw, a, st);
}

int fp8_weight_dequant(const void* q, const float* s_inv, int64_t N, int64_t K, int block, int fmt, void* w,
                       void* stream) {
  if (N < 0 || K <= 0) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (block != 128 && block != 0) return FP8_ERR_UNSUPPORTED;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (N == 0) return FP8_OK;
  if (!q || !s_inv || !w) return FP8_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(s_inv, 4) || !aligned(w, 16)) return FP8_ERR_ALIGNMENT;
  const uint8_t* qb = static_cast<const uint8_t*>(q);
  uint16_t* wb = static_cast<uint16_t*>(w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return fmt == FP8_E4M3 ? launch_dequant<kE4M3>(qb, s_inv, N, K, block, wb, st)
                         : launch_dequant<kE5M2>(qb, s_inv, N, K, block, wb, st);
}

int fp8_grouped_gemm(const void* qa, const float* sa, const void* qw, const float* sw,
                     const int32_t* group_offsets, int64_t E, int64_t total_M, int64_t N, int64_t K,
                     int out_dtype, void* y, void* stream) {
  int rc = check_gemm_common(qa, sa, qw, sw, total_M, N, K, out_dtype, y);
  if (rc != FP8_OK) return rc;
  if (E <= 0 || E > INT32_MAX || !group_offsets) return FP8_ERR_INVALID_ARG;
  if (!aligned(group_offsets, 4)) return FP8_ERR_ALIGNMENT;
  if (E * N > INT32_MAX) return FP8_ERR_SHAPE;
  if (total_M == 0) return FP8_OK;
  GemmArgs a{sa, sw, y, group_offsets, int(total_M), int(N), int(K), int(E),
             out_dtype == FP8_OUT_FP32 ? 1 : 0};
  return launch_swap<160, 3, 5, 28>(qa, qw, a, E * N, static_cast<cudaStream_t>(stream));
}

int fp8_delayed_quant(const void* x, int64_t n, int fmt, float target, int64_t hist_len, int algo, float* scale,
                      int32_t* pos, float* history, void* q, uint64_t* n_clipped, float* s_used, void* stream) {
  if (n < 0 || hist_len < 1 || hist_len > 65536) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (algo != FP8_AMAX_MOST_RECENT && algo != FP8_AMAX_MAX) return FP8_ERR_INVALID_ARG;
  if (!(target > 0.0f) || !(target < 3.0e38f)) return FP8_ERR_INVALID_ARG;
  if (!scale || !pos || !history || !n_clipped || !s_used || (n > 0 && (!x || !q))) return FP8_ERR_INVALID_ARG;
  if (n % 8 != 0) return FP8_ERR_SHAPE;
  if ((n > 0 && (!aligned(x, 16) || !aligned(q, 16))) || !aligned(scale, 4) || !aligned(pos, 4) ||
      !aligned(history, 4) || !aligned(n_clipped, 8) || !aligned(s_used, 4))
    return FP8_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(n_clipped, 0, sizeof(uint64_t), st) != cudaSuccess) return FP8_ERR_CUDA;
  const int64_t n8 = n / 8;
  int64_t blocks = (n8 + 255) / 256;
  const int64_t cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  uint8_t* qb = static_cast<uint8_t*>(q);
  unsigned long long* nc = reinterpret_cast<unsigned long long*>(n_clipped);
  const cudaError_t e = fmt == FP8_E4M3
      ? launch(k_delayed_cast<kE4M3>, unsigned(blocks), 256, 0, st, xb, n8, scale, pos, int(hist_len), history, qb, nc, s_used)
      : launch(k_delayed_cast<kE5M2>, unsigned(blocks), 256, 0, st, xb, n8, scale, pos, int(hist_len), history, qb, nc, s_used);
  if (e != cudaSuccess) return FP8_ERR_CUDA;
  return cuda_status(launch(k_delayed_finalize, 1, 32, 0, st, target, int(hist_len), algo, scale, pos, history));
}

int fp8_mx_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int fmt, void* q, void* e8, void* stream) {
  if (M < 0 || K <= 0 || ldx < K) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (M == 0) return FP8_OK;
  if (!x || !q || !e8) return FP8_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(q, 16)) return FP8_ERR_ALIGNMENT;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  uint8_t* qb = static_cast<uint8_t*>(q);
  uint8_t* eb = static_cast<uint8_t*>(e8);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return fmt == FP8_E4M3 ? launch_mx_quant<kE4M3>(xb, M, K, ldx, qb, eb, st)
                         : launch_mx_quant<kE5M2>(xb, M, K, ldx, qb, eb, st);
}

int fp8_mx_gemm(const void* qa, const void* sfa, const void* qw, const void* sfw, int64_t M, int64_t N,
                int64_t K, int out_dtype, void* y, void* stream) {
  if (M < 0 || N <= 0 || K <= 0) return FP8_ERR_INVALID_ARG;
  if (out_dtype != FP8_OUT_BF16 && out_dtype != FP8_OUT_FP32) return FP8_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 16 != 0) return FP8_ERR_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return FP8_ERR_SHAPE;
  if (!qw || !sfw) return FP8_ERR_INVALID_ARG;
  if (M > 0 && (!qa || !sfa || !y)) return FP8_ERR_INVALID_ARG;
  if (!aligned(qw, 16) || !aligned(sfw, 16)) return FP8_ERR_ALIGNMENT;
  if (M > 0 && (!aligned(qa, 16) || !aligned(sfa, 16) || !aligned(y, 16))) return FP8_ERR_ALIGNMENT;
  if (M == 0) return FP8_OK;
  MxArgs a{static_cast<const uint8_t*>(sfa), static_cast<const uint8_t*>(sfw), y, int(M), int(N), int(K),
           out_dtype == FP8_OUT_FP32 ? 1 : 0};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M <= 64) return launch_mx<true, 64, 8>(qa, qw, a, st);
  if (M <= 160) return launch_mx<true, 160, 5>(qa, qw, a, st);
  return launch_mx<false, 256, 4>(qa, qw, a, st);
}

int fp8_mx_pack_pow2(const float* s, int64_t rows, int64_t K, int row_block, void* sf, void* stream) {
  if (rows < 0 || K <= 0) return FP8_ERR_INVALID_ARG;
  if (row_block != 1 && row_block != 128) return FP8_ERR_INVALID_ARG;
  if (K % 128 != 0) return FP8_ERR_SHAPE;
  if (rows == 0) return FP8_OK;
  if (!s || !sf) return FP8_ERR_INVALID_ARG;
  if (!aligned(s, 4) || !aligned(sf, 16)) return FP8_ERR_ALIGNMENT;
  const int64_t nkb = K / 128, n = rows * nkb;
  return cuda_status(launch(k_mx_pack_pow2, unsigned((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream), s, rows,
                            nkb, row_block, static_cast<uint8_t*>(sf)));
}

int fp8_moe_route(const float* scores, int64_t T, int64_t E, int64_t k, int32_t* ids, float* w, int32_t* offsets,
                  int32_t* row_token, float* row_weight, int32_t* token_row, void* workspace, int64_t workspace_bytes,
                  void* stream) {
  if (T < 0 || E < 1 || E > kMoeMaxE || k < 1 || k > kMoeMaxK || k > E) return FP8_ERR_INVALID_ARG;
  if (T * k > INT32_MAX) return FP8_ERR_SHAPE;
  if (!offsets || !workspace) return FP8_ERR_INVALID_ARG;
  if (T > 0 && (!scores || !ids || !w || !row_token || !row_weight || !token_row)) return FP8_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(ids, 4) || !aligned(w, 4) || !aligned(offsets, 4) || !aligned(row_token, 4) ||
      !aligned(row_weight, 4) || !aligned(token_row, 4) || !aligned(workspace, 4))
    return FP8_ERR_ALIGNMENT;
  if (workspace_bytes < FP8_MOE_ROUTE_WS_BYTES(T, k, E)) return FP8_ERR_SHAPE;
  return launch_moe_route(scores, T, E, k, ids, w, offsets, row_token, row_weight, token_row,
                          static_cast<int32_t*>(workspace), static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------ routing without a caller workspace
// The sort's scratch in a file-scope device array of fixed size: 256 KiB, i.e. (G + 1) * E
// <= 65536 int32 for G = ceil(T*k / 512) chunks (e.g. 4096 tokens, top-8 of 256 experts:
// 65 x 256).  One array per device, shared by every call on that device.
constexpr int64_t kRouteScratchInts = 65536;
constexpr int kRouteMaxDevices = 64;
static __device__ __align__(256) int32_t g_route_scratch[kRouteScratchInts];

int fp8_moe_route_noalloc(const float* scores, int64_t T, int64_t E, int64_t k, int32_t* ids, float* w,
                          int32_t* offsets, int32_t* row_token, float* row_weight, int32_t* token_row, void* stream) {
  if (T < 0 || E < 1 || E > kMoeMaxE || k < 1 || k > kMoeMaxK || k > E) return FP8_ERR_INVALID_ARG;
  if (T * k > INT32_MAX) return FP8_ERR_SHAPE;
  if (FP8_MOE_ROUTE_WS_BYTES(T, k, E) > kRouteScratchInts * int64_t(sizeof(int32_t))) return FP8_ERR_SHAPE;
  if (!offsets) return FP8_ERR_INVALID_ARG;
  if (T > 0 && (!scores || !ids || !w || !row_token || !row_weight || !token_row)) return FP8_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(ids, 4) || !aligned(w, 4) || !aligned(offsets, 4) || !aligned(row_token, 4) ||
      !aligned(row_weight, 4) || !aligned(token_row, 4))
    return FP8_ERR_ALIGNMENT;
  // the array's device address, looked up once per device with that device current
  static std::mutex mu;
  static int32_t* scratch[kRouteMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kRouteMaxDevices) return FP8_ERR_CUDA;
  int32_t* ws;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!scratch[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return FP8_ERR_CUDA;
      scratch[dev] = static_cast<int32_t*>(p);
    }
    ws = scratch[dev];
  }
  // every workspace entry the passes read is written earlier in the same call (the count
  // pass writes each chunk's full histogram row, the scan pass the totals row), so
  // nothing has to start at zero and nothing is cleared
  return launch_moe_route(scores, T, E, k, ids, w, offsets, row_token, row_weight, token_row, ws,
                          static_cast<cudaStream_t>(stream));
}

int fp8_act_quant_permute(const void* x, int64_t T, int64_t K, int64_t ldx, int fmt, int scale_fmt,
                          const int32_t* token_row, int64_t k, void* q, float* s, void* stream) {
  if (T < 0 || K <= 0 || ldx < K || k < 1 || k > kMoeMaxK) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (scale_fmt != FP8_SCALE_FP32 && scale_fmt != FP8_SCALE_UE8M0) return FP8_ERR_INVALID_ARG;
  if (K % 16 != 0) return FP8_ERR_SHAPE;
  if (T * k > INT32_MAX) return FP8_ERR_SHAPE;
  if (T == 0) return FP8_OK;
  if (!x || !q || !s || !token_row) return FP8_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4) || !aligned(token_row, 4))
    return FP8_ERR_ALIGNMENT;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  uint8_t* qb = static_cast<uint8_t*>(q);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int kk = int(k);
  if (fmt == FP8_E4M3)
    return scale_fmt == FP8_SCALE_FP32 ? launch_act_quant_permute<kE4M3, kScaleFp32>(xb, T, K, ldx, qb, s, token_row, kk, st)
                                       : launch_act_quant_permute<kE4M3, kScaleUe8m0>(xb, T, K, ldx, qb, s, token_row, kk, st);
  return scale_fmt == FP8_SCALE_FP32 ? launch_act_quant_permute<kE5M2, kScaleFp32>(xb, T, K, ldx, qb, s, token_row, kk, st)
                                     : launch_act_quant_permute<kE5M2, kScaleUe8m0>(xb, T, K, ldx, qb, s, token_row, kk, st);
}

int fp8_moe_gemm(const void* qa, const float* sa, const void* qw, const float* sw, const int32_t* offsets,
                 const int32_t* row_token, const float* row_weight, int64_t T, int64_t E, int64_t k, int64_t N,
                 int64_t K, float* out, void* stream) {
  if (T < 0 || E <= 0 || k <= 0 || N <= 0 || K <= 0) return FP8_ERR_INVALID_ARG;
  if (K % 128 != 0 || N % 16 != 0) return FP8_ERR_SHAPE;
  if (T * k > INT32_MAX || E * N > INT32_MAX || K > INT32_MAX || T * N > (int64_t(1) << 40)) return FP8_ERR_SHAPE;
  if (!qw || !sw || !offsets || !out) return FP8_ERR_INVALID_ARG;
  if (T > 0 && (!qa || !sa || !row_token || !row_weight)) return FP8_ERR_INVALID_ARG;
  if (!aligned(qw, 16) || !aligned(sw, 4) || !aligned(offsets, 4) || !aligned(out, 4)) return FP8_ERR_ALIGNMENT;
  if (T > 0 && (!aligned(qa, 16) || !aligned(sa, 4) || !aligned(row_token, 4) || !aligned(row_weight, 4)))
    return FP8_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T == 0) return FP8_OK;
  if (cudaMemsetAsync(out, 0, size_t(T) * size_t(N) * sizeof(float), st) != cudaSuccess) return FP8_ERR_CUDA;
  GemmArgs a{sa, sw, nullptr, offsets, int(T * k), int(N), int(K), int(E), 1};
  a.row_token = row_token;
  a.row_weight = row_weight;
  a.moe_out = out;
  a.moe_T = int(T);
  return launch_swap<160, 3, 5, 28, false, true>(qa, qw, a, E * N, st);
}

int fp8_selftest_bounded_wait(int64_t limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 10000000000ll) return FP8_ERR_INVALID_ARG;
  return cuda_status(launch(k_selftest_wait, 1, 32, 0, static_cast<cudaStream_t>(stream), uint64_t(limit_ns)));
}

int fp8_set_wait_limit_ns(int64_t limit_ns) {
  if (limit_ns < 0 || limit_ns > 10000000000ll) return FP8_ERR_INVALID_ARG;
  const unsigned long long v = limit_ns == 0 ? FP8LIN_WAIT_NS : (unsigned long long)limit_ns;
  return cuda_status(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
}

int fp8_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP8_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return FP8_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return FP8_ERR_CUDA;
  if (v & 1u) return FP8_ERR_TIMEOUT;
  if (v & kErrBadScale) return FP8_ERR_INVALID_SCALE;
  return FP8_OK;
}

}  // extern "C"
