// Shared device helpers for the rq kernels (sm_100a only): mbarriers, bulk
// copies, the sticky device error word and bit tricks for 4-bit packing.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "rq kernels are written for sm_100a only"
#endif

namespace rq {

// Device error word: a kernel that gives up on a bounded wait ORs a code in
// here and returns; the host reads (and clears) it with rq_get_device_error.
enum DeviceError : unsigned {
  kDevErrNone = 0u,
  kDevErrTimeout = 1u,        // an mbarrier wait exceeded its limit
  kDevErrTmemAlloc = 2u,      // tcgen05.alloc did not return the expected columns
};

__device__ unsigned g_device_error;

// Spin limit for mbarrier waits, in SM clock cycles (about 1 s at 1.9 GHz):
// far above any legitimate wait in these kernels.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Programmatic dependent launch.  Kernels launched with launch_pdl may start
// while the previous kernel in the stream is still finishing; each kernel
// first waits (griddep_wait) until every earlier grid has completed and its
// memory is visible -- before it touches any global memory -- and then lets
// the next kernel launch early (griddep_trigger).  What overlaps is the
// launch, the CTA start-up and the previous kernel's tail; not one memory
// access.  Without the launch attribute both instructions do nothing.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Bounded wait on an mbarrier phase. Returns false (and records a timeout in
// the device error word) if the phase did not complete within `limit` SM
// clock cycles (kWaitLimitCycles, ~1 s, unless given).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity,
                                                  long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) {
      atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
      return false;
    }
  }
  return true;
}

// Self-test of the timeout path: one thread waits on an mbarrier that expects
// an arrival nobody makes, with a short limit, and so records a timeout.
__global__ void selftest_wait_timeout_kernel(long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait_bounded(&bar, 0u, limit);
  }
}

// 1-D bulk copy global -> shared (TMA engine, no tensor map), completion
// signalled on an mbarrier as transaction bytes.  Both addresses 16-B aligned,
// size a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Number-format helpers
// ---------------------------------------------------------------------------

// 1.5 * 2^23: adding it to a float in (-2^22, 2^22) rounds to an integer
// (round-to-nearest-even, the FPU's rounding) and leaves that integer, in
// two's complement, in the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;

// Low bytes of four 32-bit words -> one word (byte i from word i).
__device__ __forceinline__ uint32_t gather_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t ab = __byte_perm(a, b, 0x0040);  // [a.b0, b.b0, a.b0, a.b0]
  const uint32_t cd = __byte_perm(c, d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);               // [a.b0, b.b0, c.b0, d.b0]
}

// Pack eight "magic-rounded" floats (integer in the low nibble of each) into a
// word: element t -> bits [4t, 4t+4).  Even elements go to low nibbles.
__device__ __forceinline__ uint32_t pack8_magic(const float* f) {
  const uint32_t lo = gather_low_bytes(__float_as_uint(f[0]), __float_as_uint(f[2]), __float_as_uint(f[4]),
                                       __float_as_uint(f[6]));
  const uint32_t hi = gather_low_bytes(__float_as_uint(f[1]), __float_as_uint(f[3]), __float_as_uint(f[5]),
                                       __float_as_uint(f[7]));
  return (lo & 0x0F0F0F0Fu) | ((hi << 4) & 0xF0F0F0F0u);
}

// Eight floats -> eight E2M1 codes (round to nearest even, saturating), element
// t in bits [4t, 4t+4).  Codes whose magnitude is zero are written as +0.
__device__ __forceinline__ uint32_t pack8_e2m1(float f0, float f1, float f2, float f3, float f4, float f5, float f6,
                                               float f7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(f0), "f"(f1), "f"(f2), "f"(f3), "f"(f4), "f"(f5), "f"(f6), "f"(f7));
  // Clear the sign of nibbles whose magnitude bits are all zero (-0 -> +0).
  const uint32_t nz = ((out & 0x77777777u) + 0x77777777u) & 0x88888888u;
  return out & (0x77777777u | nz);
}

// fp32 -> E4M3 code (round to nearest even, saturating to 448).  Input >= 0.
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(x));
  return out & 0xFFu;
}

// E4M3 code -> fp32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  const uint16_t c = (uint16_t)code;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

}  // namespace rq
