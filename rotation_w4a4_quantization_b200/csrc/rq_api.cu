// librq: the C ABI declared in include/rq.h.  Host-side argument checks,
// kernel selection and launches.  All kernels live in the headers included
// below (one translation unit, so the device error word is a single symbol).
#include <nvtx3/nvToolsExt.h>
#include "../../include/rq.h"

#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "rq_common.cuh"
#include "rq_rotate.cuh"
#include "rq_gemm.cuh"
#include "rq_attn.cuh"

namespace {

using namespace rq;

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxKBlock = 32768;
constexpr size_t kSmemBudget = 220 * 1024;

int num_sms_of_current_device() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// Raise a kernel's dynamic shared memory limit once per (kernel, device).  The
// default is the whole per-CTA budget; kernels with static shared memory pass
// what they need (static + dynamic must stay within the per-CTA maximum).
bool ensure_smem(const void* kernel, int bytes = (int)kSmemBudget + 7 * 1024) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, uint64_t>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = (dev < 64) ? (1ull << dev) : 0;
  std::lock_guard<std::mutex> lock(mu);
  for (auto& e : done)
    if (e.first == kernel && bit && (e.second & bit)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  for (auto& e : done)
    if (e.first == kernel) {
      e.second |= bit;
      return true;
    }
  done.emplace_back(kernel, bit);
  return true;
}

rq_status last_launch_status() { return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA; }

// Geometry of the rotate kernel: warps per group G, rows per stage RPS,
// groups per CTA GPC and ring depth, for a block-diagonal (full = false) or
// full-width rotation of K channels.
struct RotCfg {
  int G, RPS, GPC, stages, threads;
  size_t smem;
};

RotCfg rotate_config(int64_t K, bool full, int mode) {
  const int nb = (int)(K / 128);
  RotCfg c;
  if (32 % nb == 0) {
    c.G = 1;
    c.RPS = 32 / nb;
  } else {
    c.G = (nb + 31) / 32;
    c.RPS = 1;
  }
  const int warps = full ? RQ_FULL_WIDTH_THREADS / 32 : 12;  // must match the kernel's launch bounds
  c.GPC = warps / c.G > 0 ? warps / c.G : 1;
  for (;;) {
    const size_t sb = RotSmemLayout::stage_bytes(c.RPS, (int)K);
    const size_t fixed = RotSmemLayout::total(c.RPS, (int)K, 0, c.GPC, c.G) + (size_t)c.GPC * 4 * 8;
    const int st = (int)((kSmemBudget - fixed) / (sb * c.GPC));
    c.stages = st > 4 ? 4 : st;
    if (c.stages >= 2 || c.GPC == 1) break;
    --c.GPC;
  }
  c.threads = 32 * c.G * c.GPC;
  c.smem = RotSmemLayout::total(c.RPS, (int)K, c.stages, c.GPC, c.G);
  return c;
}

// pdl = false for a launch that directly follows a non-kernel stream operation
// (a memset), which programmatic launch must not overlap.
template <int MODE, int NBF, int LOGB = 7>
rq_status launch_rotate(RotParams p, cudaStream_t st, bool pdl = true) {
  const RotCfg c = rotate_config(p.K, NBF != 0, MODE);
  if (c.stages < 2) return RQ_ERR_UNSUPPORTED_SHAPE;
  p.G = c.G;
  p.RPS = c.RPS;
  p.GPC = c.GPC;
  p.stages = c.stages;
  p.num_tiles = (p.rows + c.RPS - 1) / c.RPS;
  const int64_t ctas = (p.num_tiles + c.GPC - 1) / c.GPC;
  const int64_t grid = ctas < num_sms_of_current_device() ? ctas : num_sms_of_current_device();
  if (!ensure_smem(reinterpret_cast<const void*>(rotate_kernel<MODE, NBF, LOGB>))) return RQ_ERR_CUDA;
  if (pdl)
    (void)launch_pdl(rotate_kernel<MODE, NBF, LOGB>, dim3((unsigned)grid), dim3(c.threads), c.smem, st, p);
  else
    rotate_kernel<MODE, NBF, LOGB><<<(unsigned)grid, c.threads, c.smem, st>>>(p);
  return last_launch_status();
}

// Block-diagonal rotation: blocks of 128, or of 16 / 32 (p.logb 4 / 5, the
// format-sized blocks), or of one channel (p.logb 0: no rotation, signs only);
// not for KV4, whose block is the head.
template <int MODE>
rq_status launch_block(RotParams p, cudaStream_t st, bool pdl = true) {
  if constexpr (MODE != kModeKv4) {
    if (p.logb == 0) return launch_rotate<MODE, 0, 0>(p, st, pdl);
    if (p.logb == 4) return launch_rotate<MODE, 0, 4>(p, st, pdl);
    if (p.logb == 5) return launch_rotate<MODE, 0, 5>(p, st, pdl);
  }
  return launch_rotate<MODE, 0, 7>(p, st, pdl);
}

// K = 4096: the 64 x 64 two-pass kernel, one CTA of eight row teams per SM,
// each CTA's rows staged through a ring of up to kF4kSlots shared-memory slots.
template <int MODE>
rq_status launch_full4096(RotParams p, cudaStream_t st) {
  const int64_t cap = (int64_t)num_sms_of_current_device();
  const int64_t grid = p.rows < cap ? p.rows : cap;
  const int64_t rpc = (p.rows + grid - 1) / grid;  // the most rows any CTA takes
  const int slots = rpc <= kF4kSlots ? (int)rpc : kF4kSlots;
  if (!ensure_smem(reinterpret_cast<const void*>(rotate_full4096_kernel<MODE>), (int)f4k_smem_bytes(kF4kSlots)))
    return RQ_ERR_CUDA;
  (void)launch_pdl(rotate_full4096_kernel<MODE>, dim3((unsigned)grid), dim3(kR64Threads), f4k_smem_bytes(slots), st,
                   p, slots);
  return last_launch_status();
}

template <int MODE>
rq_status launch_full(RotParams p, cudaStream_t st) {
  switch (p.nb) {
    case 2: return launch_rotate<MODE, 2>(p, st);
    case 4: return launch_rotate<MODE, 4>(p, st);
    case 8: return launch_rotate<MODE, 8>(p, st);
    case 16: return launch_rotate<MODE, 16>(p, st);
    case 32: return launch_full4096<MODE>(p, st);
    default: return RQ_ERR_UNSUPPORTED_SHAPE;
  }
}

// Dynamic NVFP4 in one pass (rotate_nvfp4_resident_kernel): every CTA keeps its
// rows in shared memory; needs all CTAs resident (cooperative launch).  Returns
// RQ_ERR_UNSUPPORTED_SHAPE (nothing launched) when the rows do not fit.
template <int LOGB>
rq_status launch_nvfp4_resident_b(RotParams p, cudaStream_t st) {
  int dev = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
    return RQ_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms_of_current_device();
  const int64_t rpc = (p.rows + sms - 1) / sms;
  const size_t smem = (size_t)rpc * p.K * 2 + (size_t)p.nb * 64 * 4 + (size_t)rpc * 8 + 48;
  if (smem > kSmemBudget) return RQ_ERR_UNSUPPORTED_SHAPE;
  // the rotated values wait in tensor memory between the passes when a CTA's
  // 128-value units fit its 512 columns x 128 lanes
  int stash = rpc * p.nb <= kResStashUnits ? 1 : 0;
  const int grid = (int)((p.rows + rpc - 1) / rpc);
  if (!ensure_smem(reinterpret_cast<const void*>(rotate_nvfp4_resident_kernel<LOGB>))) return RQ_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_nvfp4_resident_kernel<LOGB>, kResThreads, smem) !=
          cudaSuccess ||
      per_sm < 1 || grid > per_sm * sms)
    return RQ_ERR_UNSUPPORTED_SHAPE;
  p.nvfp4_dynamic = 1;
  int rows_per_cta = (int)rpc;
  void* args[] = {&p, &rows_per_cta, &stash};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kResThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(rotate_nvfp4_resident_kernel<LOGB>), args) != cudaSuccess)
    return RQ_ERR_CUDA;
  return RQ_OK;
}

rq_status launch_nvfp4_resident(RotParams p, cudaStream_t st) {
  if (p.logb == 0) return launch_nvfp4_resident_b<0>(p, st);
  if (p.logb == 4) return launch_nvfp4_resident_b<4>(p, st);
  if (p.logb == 5) return launch_nvfp4_resident_b<5>(p, st);
  return launch_nvfp4_resident_b<7>(p, st);
}

// Common checks of the X / K / signs / block arguments.
// Pointers are only required (and checked) when there is work: M = 0 is a no-op.
rq_status check_rotation_args(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* signs, int block) {
  if (M > 0 && (!X || !signs)) return RQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || ldx < K) return RQ_ERR_INVALID_ARG;
  if (K % 128 != 0 || K > kMaxKBlock) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (block != 0 && block != 1 && block != 16 && block != 32 && block != 128) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (block == 0 && !(is_pow2(K) && K >= 256 && K <= 4096)) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(X, 16) || (ldx * 2) % 16 != 0 || !aligned(signs, 16)) return RQ_ERR_ALIGNMENT;
  return RQ_OK;
}

// Block-diagonal rotation size (1, 16, 32 or 128; 0 = full width leaves 128).
void set_block(RotParams& p, int block) {
  const int b = (block == 1 || block == 16 || block == 32) ? block : 128;
  p.logb = b == 1 ? 0 : (b == 16 ? 4 : (b == 32 ? 5 : 7));
  p.cblk = (float)(1.0 / std::sqrt((double)b));
}

RotParams matrix_params(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* signs) {
  RotParams p;
  std::memset(&p, 0, sizeof(p));
  p.x = static_cast<const uint8_t*>(X);
  p.rows = M;
  p.K = (int)K;
  p.nb = (int)(K / 128);
  p.S = M > 0 ? M : 1;
  p.H = 1;
  p.sS = ldx * 2;
  p.sH = 0;
  p.sB = 0;
  p.contiguous = (ldx == K) ? 1 : 0;
  p.signs = signs;
  p.cfull = (float)(1.0 / std::sqrt((double)K));
  set_block(p, 128);
  return p;
}

rq_status rotate_quantize_impl(const void* X, int64_t M, int64_t K, int64_t ldx, const int8_t* signs, int block,
                               rq_format fmt, rq_gscale gmode, uint8_t* codes, void* scales, float* gscale,
                               void* workspace, cudaStream_t st) {
  rq_status s = check_rotation_args(X, M, K, ldx, signs, block);
  if (s != RQ_OK) return s;
  if (fmt != RQ_INT4 && fmt != RQ_NVFP4 && fmt != RQ_MXFP4 && fmt != RQ_INT8 && fmt != RQ_INT6 &&
      fmt != RQ_INT4_ASYM && fmt != RQ_INT4_BYTES)
    return RQ_ERR_INVALID_ARG;
  if (gmode != RQ_SCALE_DYNAMIC && gmode != RQ_SCALE_STATIC) return RQ_ERR_INVALID_ARG;
  const bool int_fmt = fmt == RQ_INT4 || fmt == RQ_INT8 || fmt == RQ_INT6 || fmt == RQ_INT4_BYTES;
  if (!int_fmt && block == 0) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return RQ_OK;
  if (!codes || !scales) return RQ_ERR_INVALID_ARG;
  if (!aligned(codes, 16)) return RQ_ERR_ALIGNMENT;
  if (fmt == RQ_NVFP4) {
    if (!gscale) return RQ_ERR_INVALID_ARG;
    if (gmode == RQ_SCALE_DYNAMIC && !workspace) return RQ_ERR_INVALID_ARG;
    if (!aligned(scales, 8) || !aligned(gscale, 4)) return RQ_ERR_ALIGNMENT;
    if (workspace && !aligned(workspace, 16)) return RQ_ERR_ALIGNMENT;
  } else {
    if (!aligned(scales, 4)) return RQ_ERR_ALIGNMENT;  // INT4 fp32 scales, MXFP4 4 bytes per 128-block
  }
  if (M == 0) return RQ_OK;

  RotParams p = matrix_params(X, M, K, ldx, signs);
  set_block(p, block);
  p.codes = codes;
  if (fmt == RQ_INT4) {
    p.scales_f32 = static_cast<float*>(scales);
    if (block == 0) return launch_full<kModeInt4>(p, st);
    return launch_block<kModeInt4>(p, st);
  }
  if (fmt == RQ_INT4_ASYM) {
    p.kv_scale = static_cast<__half*>(scales);
    return launch_block<kModeAsym4>(p, st);
  }
  if (fmt == RQ_INT8 || fmt == RQ_INT6 || fmt == RQ_INT4_BYTES) {
    // one code per byte; RQ_INT4_BYTES is the INT4 rule (qmax 7, the same
    // reciprocal and rounding as the packed INT4 kernels) in this layout
    p.scales_f32 = static_cast<float*>(scales);
    p.qmax = fmt == RQ_INT8 ? 127.0f : (fmt == RQ_INT6 ? 31.0f : 7.0f);
    if (block == 0) return launch_full<kModeInt8>(p, st);
    return launch_block<kModeInt8>(p, st);
  }
  if (fmt == RQ_MXFP4) {
    p.scales_e4m3 = static_cast<uint8_t*>(scales);
    return launch_block<kModeMxfp4>(p, st);
  }
  p.scales_e4m3 = static_cast<uint8_t*>(scales);
  if (gmode == RQ_SCALE_DYNAMIC) {
    p.amax_word = static_cast<unsigned*>(workspace);
    p.g_out = gscale;
    if (cudaMemsetAsync(workspace, 0, 2 * sizeof(unsigned), st) != cudaSuccess) return RQ_ERR_CUDA;
    // one pass over HBM when the whole tensor fits in the SMs' shared memory
    s = launch_nvfp4_resident(p, st);
    if (s != RQ_ERR_UNSUPPORTED_SHAPE) return s;
    s = launch_block<kModeAmax>(p, st, /*pdl=*/false);  // follows the memset
    if (s != RQ_OK) return s;
    p.nvfp4_dynamic = 1;
    p.g_out = gscale;
  } else {
    p.nvfp4_dynamic = 0;
    p.g_in = gscale;
  }
  return launch_block<kModeNvfp4>(p, st);
}

// ---------------------------------------------------------------------------
// Scratch for rq_rotate_quantize_nvfp4_noalloc.  The dynamic NVFP4 scale needs
// one word of device memory that starts at zero (the max of |X~| is gathered
// there by atomics); this entry point takes it from this static array instead
// of a caller-allocated workspace.  Every GPU that loads the library holds
// these 256 bytes until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[256];

// Device address of g_noalloc_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
rq_status noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RQ_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return RQ_OK;
}

}  // namespace


// An NVTX range around each public call (a no-op unless a profiler such as
// Nsight Systems or Nsight Compute with NVTX filtering is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

extern "C" {

rq_status rq_rotate_quantize_nvfp4_noalloc(const void* X_dev, int64_t M, int64_t K, int64_t ldx,
                                           const int8_t* signs_dev, uint8_t* codes_dev, void* scales_dev,
                                           float* gscale_dev, rq_stream_t stream) {
  NvtxRange nvtx_("rq_rotate_quantize_nvfp4_noalloc");
  // The scratch this path needs does not grow with M or K; the check keeps the
  // static array's stated size honest if that ever changes.
  if (rq_workspace_bytes(RQ_NVFP4) > sizeof(g_noalloc_scratch)) return RQ_ERR_UNSUPPORTED_SHAPE;
  rq_status s = check_rotation_args(X_dev, M, K, ldx, signs_dev, 128);
  if (s != RQ_OK) return s;
  if (M == 0) return RQ_OK;
  void* scratch = nullptr;
  s = noalloc_scratch_address(&scratch);
  if (s != RQ_OK) return s;
  // the max word is cleared by the call itself (cudaMemsetAsync on the stream)
  return rotate_quantize_impl(X_dev, M, K, ldx, signs_dev, 128, RQ_NVFP4, RQ_SCALE_DYNAMIC, codes_dev, scales_dev,
                              gscale_dev, scratch, static_cast<cudaStream_t>(stream));
}

const char* rq_status_string(rq_status status) {
  switch (status) {
    case RQ_OK: return "ok";
    case RQ_ERR_INVALID_ARG: return "invalid argument";
    case RQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case RQ_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case RQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0, sm_100a)";
    case RQ_ERR_CUDA: return "CUDA error";
    case RQ_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

rq_status rq_init(int device) {
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || device < 0 || device >= n) return RQ_ERR_UNSUPPORTED_DEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return RQ_ERR_UNSUPPORTED_DEVICE;
  if (prop.major != 10 || prop.minor != 0) return RQ_ERR_UNSUPPORTED_DEVICE;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return RQ_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return RQ_ERR_CUDA;
  cudaFuncAttributes attr;
  const cudaError_t e = cudaFuncGetAttributes(&attr, rotate_kernel<kModeInt4, 0>);
  (void)cudaSetDevice(prev);
  if (e != cudaSuccess) return RQ_ERR_UNSUPPORTED_DEVICE;
  return RQ_OK;
}

size_t rq_workspace_bytes(rq_format fmt) { return fmt == RQ_NVFP4 ? 16 : 0; }

rq_status rq_rotate_quantize(const void* X_dev, int64_t M, int64_t K, int64_t ldx, const int8_t* signs_dev,
                             int block, rq_format fmt, rq_gscale gmode, uint8_t* codes_dev, void* scales_dev,
                             float* gscale_dev, void* workspace_dev, rq_stream_t stream) {
  NvtxRange nvtx_("rq_rotate_quantize");
  return rotate_quantize_impl(X_dev, M, K, ldx, signs_dev, block, fmt, gmode, codes_dev, scales_dev, gscale_dev,
                              workspace_dev, static_cast<cudaStream_t>(stream));
}

rq_status rq_prepare_weights(const void* W_dev, int64_t N, int64_t K, int64_t ldw, const int8_t* signs_dev,
                             int block, rq_format fmt, uint8_t* codes_dev, void* scales_dev, float* gscale_dev,
                             void* workspace_dev, rq_stream_t stream) {
  NvtxRange nvtx_("rq_prepare_weights");
  return rotate_quantize_impl(W_dev, N, K, ldw, signs_dev, block, fmt, RQ_SCALE_DYNAMIC, codes_dev, scales_dev,
                              gscale_dev, workspace_dev, static_cast<cudaStream_t>(stream));
}

rq_status rq_rotate_f32(const void* X_dev, int64_t M, int64_t K, int64_t ldx, const int8_t* signs_dev, int block,
                        float* out_dev, int64_t ldo, rq_stream_t stream) {
  NvtxRange nvtx_("rq_rotate_f32");
  rq_status s = check_rotation_args(X_dev, M, K, ldx, signs_dev, block);
  if (s != RQ_OK) return s;
  if (ldo < K) return RQ_ERR_INVALID_ARG;
  if (M == 0) return RQ_OK;
  if (!out_dev) return RQ_ERR_INVALID_ARG;
  if (!aligned(out_dev, 16) || ldo % 4 != 0) return RQ_ERR_ALIGNMENT;
  RotParams p = matrix_params(X_dev, M, K, ldx, signs_dev);
  set_block(p, block);
  p.out_f32 = out_dev;
  p.ldo = ldo;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (block == 0) return launch_full<kModeF32>(p, st);
  return launch_block<kModeF32>(p, st);
}

rq_status rq_kv_rotate_quantize(const void* KV_dev, int64_t B, int64_t H, int64_t S, int64_t D,
                                const int64_t* strides_host, const int8_t* signs_dev, uint8_t* codes_dev,
                                void* scale_dev, void* zero_dev, rq_stream_t stream) {
  NvtxRange nvtx_("rq_kv_rotate_quantize");
  if (B < 0 || H < 0 || S < 0) return RQ_ERR_INVALID_ARG;
  if (D != 128) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (B * H * S == 0) return RQ_OK;
  if (!KV_dev || !strides_host || !signs_dev || !codes_dev || !scale_dev || !zero_dev) return RQ_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (strides_host[i] < 0) return RQ_ERR_INVALID_ARG;
  if (!aligned(KV_dev, 16) || !aligned(codes_dev, 16) || !aligned(scale_dev, 2) || !aligned(zero_dev, 2) ||
      !aligned(signs_dev, 16))
    return RQ_ERR_ALIGNMENT;
  for (int i = 0; i < 3; ++i)
    if ((strides_host[i] * 2) % 16 != 0) return RQ_ERR_ALIGNMENT;
  const int64_t rows = B * H * S;
  if (rows == 0) return RQ_OK;
  RotParams p;
  std::memset(&p, 0, sizeof(p));
  p.x = static_cast<const uint8_t*>(KV_dev);
  p.rows = rows;
  p.K = 128;
  p.nb = 1;
  p.S = S;
  p.H = H;
  p.sB = strides_host[0] * 2;
  p.sH = strides_host[1] * 2;
  p.sS = strides_host[2] * 2;
  p.contiguous = (strides_host[2] == 128 && (H == 1 || strides_host[1] == S * 128) &&
                  (B == 1 || strides_host[0] == H * S * 128)) ? 1 : 0;
  p.signs = signs_dev;
  p.codes = codes_dev;
  p.kv_scale = static_cast<__half*>(scale_dev);
  p.kv_zero = static_cast<__half*>(zero_dev);
  set_block(p, 128);
  return launch_block<kModeKv4>(p, static_cast<cudaStream_t>(stream));
}

rq_status rq_w4a4_gemm(const uint8_t* xcodes_dev, const void* xscales_dev, const float* xgscale_dev,
                       const uint8_t* wcodes_dev, const void* wscales_dev, const float* wgscale_dev, int64_t M,
                       int64_t N, int64_t K, rq_format fmt, void* Y_dev, int64_t ldy, rq_out out,
                       rq_stream_t stream) {
  NvtxRange nvtx_("rq_w4a4_gemm");
  return rq::gemm_dispatch(xcodes_dev, xscales_dev, xgscale_dev, wcodes_dev, wscales_dev, wgscale_dev, M, N, K, fmt,
                           Y_dev, ldy, out, static_cast<cudaStream_t>(stream));
}

rq_status rq_int_gemm(const uint8_t* xcodes_dev, const float* xscales_dev, rq_format xfmt, const uint8_t* wcodes_dev,
                      const float* wscales_dev, rq_format wfmt, int64_t M, int64_t N, int64_t K, void* Y_dev,
                      int64_t ldy, rq_out out, rq_stream_t stream) {
  NvtxRange nvtx_("rq_int_gemm");
  return rq::int_gemm_dispatch(xcodes_dev, xscales_dev, xfmt, wcodes_dev, wscales_dev, wfmt, M, N, K, Y_dev, ldy, out,
                               static_cast<cudaStream_t>(stream));
}

rq_status rq_selftest_wait_timeout(int64_t limit_cycles, rq_stream_t stream) {
  if (limit_cycles <= 0 || limit_cycles > (int64_t)kWaitLimitCycles) return RQ_ERR_INVALID_ARG;
  rq::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((long long)limit_cycles);
  return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

rq_status rq_get_device_error(rq_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return RQ_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, rq::g_device_error, sizeof(v)) != cudaSuccess) return RQ_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(rq::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return RQ_ERR_CUDA;
  return v ? RQ_ERR_TIMEOUT : RQ_OK;
}

// ---------------------------------------------------------------------------
// KV4 decode attention
// ---------------------------------------------------------------------------
size_t rq_kv4_attention_workspace_bytes(int64_t B, int64_t H, int64_t S) {
  if (B <= 0 || H <= 0 || S <= 0) return 0;
  const int64_t nchunks = (S + kAttnChunk - 1) / kAttnChunk;
  return (size_t)(B * H * nchunks) * kAttnPart * sizeof(float);
}

rq_status rq_kv4_decode_attention(const void* q_dev, int64_t B, int64_t H, int64_t S, const uint8_t* kcodes_dev,
                                  const void* kscale_dev, const void* kzero_dev, const uint8_t* vcodes_dev,
                                  const void* vscale_dev, const void* vzero_dev, const int8_t* signs_dev,
                                  float softmax_scale, void* out_dev, rq_out out, void* workspace_dev,
                                  rq_stream_t stream) {
  NvtxRange nvtx_("rq_kv4_decode_attention");
  if (B < 0 || H < 0 || S < 0) return RQ_ERR_INVALID_ARG;
  if (out != RQ_OUT_F32 && out != RQ_OUT_BF16) return RQ_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.0f) || !std::isfinite(softmax_scale)) return RQ_ERR_INVALID_ARG;
  if (B == 0 || H == 0) return RQ_OK;
  if (S == 0) return RQ_ERR_INVALID_ARG;  // softmax over no tokens
  if (!q_dev || !kcodes_dev || !kscale_dev || !kzero_dev || !vcodes_dev || !vscale_dev || !vzero_dev || !signs_dev ||
      !out_dev || !workspace_dev)
    return RQ_ERR_INVALID_ARG;
  const int64_t BH = B * H;
  const int64_t nchunks = (S + kAttnChunk - 1) / kAttnChunk;
  if (BH * nchunks > (int64_t)INT32_MAX || S > ((int64_t)1 << 40) / BH) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(q_dev, 16) || !aligned(kcodes_dev, 16) || !aligned(vcodes_dev, 16) || !aligned(signs_dev, 16) ||
      !aligned(workspace_dev, 16) || !aligned(kscale_dev, 2) || !aligned(kzero_dev, 2) || !aligned(vscale_dev, 2) ||
      !aligned(vzero_dev, 2) || !aligned(out_dev, out == RQ_OUT_BF16 ? 2 : 4))
    return RQ_ERR_ALIGNMENT;
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q_dev);
  p.kc = kcodes_dev;
  p.ks = static_cast<const __half*>(kscale_dev);
  p.kz = static_cast<const __half*>(kzero_dev);
  p.vc = vcodes_dev;
  p.vs = static_cast<const __half*>(vscale_dev);
  p.vz = static_cast<const __half*>(vzero_dev);
  p.signs = signs_dev;
  const double sc = softmax_scale > 0.0f ? (double)softmax_scale : 1.0 / std::sqrt(128.0);
  p.qscale = (float)(sc * 1.4426950408889634 / std::sqrt(128.0));
  p.S = S;
  p.nchunks = (int)nchunks;
  p.part = static_cast<float*>(workspace_dev);
  p.out = out_dev;
  p.out_bf16 = out == RQ_OUT_BF16 ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!ensure_smem(reinterpret_cast<const void*>(kv4_attn_partial_kernel), (int)kAttnSmem)) return RQ_ERR_CUDA;
  (void)launch_pdl(kv4_attn_partial_kernel, dim3((unsigned)(BH * nchunks)), dim3(128), kAttnSmem, st, p);
  if (cudaGetLastError() != cudaSuccess) return RQ_ERR_CUDA;
  (void)launch_pdl(kv4_attn_combine_kernel, dim3((unsigned)BH), dim3(128), 0, st, p);
  return last_launch_status();
}

}  // extern "C"

