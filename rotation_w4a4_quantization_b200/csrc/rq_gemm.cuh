// W4A4 GEMM on the 5th-generation tensor cores (tcgen05), sm_100a.
//
// Y[M,N] = deq(X codes) . deq(W codes)^T -- the quantized product of
// "Rotations for 4-Bit Activations: QuaRot, SpinQuant, and Friends", section
// "What it buys in 4 bits, and what it doesn't".  Both operands were rotated
// by the same Q, so this equals the layer output up to quantization error
// (section "A rotation changes nothing, and that is the point").
//
// INT4 path (kind::i8).  Blackwell has no 4-bit x 4-bit integer MMA (the
// SpinQuant and QuaRot pages make the same point about earlier hardware), so
// the packed nibbles are widened to int8: W in shared memory, X (M > 128) in
// tensor memory.  Each nibble q is placed in the HIGH half of its byte (the
// byte is 16*q, exact in int8), which needs only a mask and a byte permute
// per four codes; the MMA then accumulates 256 * sum(qx*qw) exactly in int32
// (|acc| <= 2^14 K < 2^31 for K <= 65536) and the epilogue shifts right by 8.
//
// NVFP4 path (kind::mxf4nvf4, block16).  E2M1 codes go by TMA straight into
// 128B-swizzled shared memory; the E4M3 block scales are written into tensor
// memory with tcgen05.st in the layout the block-scaled MMA reads: for a
// 64-wide K slice, row r's four scales sit in lane (r mod 32) of every lane
// quadrant, column r/32.
//
// All kernels are persistent and warp-specialized: warp 0 is the TMA
// producer, warp 1 allocates TMEM and issues the MMAs, converter / scale-mover
// warps feed the operands, and epilogue warps drain the accumulators
// (TMEM -> registers -> scale -> global, through shared memory and TMA for
// bf16).  For M <= 128 one SM computes a 128 x 256 tile; above that two SMs
// (cta_group::2) share one M = 256 MMA per K step of a 256 x 256 tile: each
// CTA holds its own 128 rows of X and 128 of the tile's rows of W, the
// operand-ready arrivals of both CTAs go to the even CTA, the MMA commits
// multicast to both, and both epilogues arrive on the even CTA's
// accumulator-free barrier.
#pragma once

#include <cuda.h>

#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "rq_common.cuh"
#include "rq_tc.cuh"

namespace rq {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kGemmThreads = 320;

struct GemmParams {
  int M, N, K;
  const void* xscale;   // INT4: float [M]; NVFP4: uint8 [M, K/16]
  const void* wscale;   // INT4: float [N]; NVFP4: uint8 [N, K/16]
  const float* xg;      // NVFP4 per-tensor scales
  const float* wg;
  void* y;
  int64_t ldy;
  int out;              // 0 f32, 1 bf16, 2 i32 accumulators
  int vec_ok;           // 1: Y rows allow 16-byte vector stores
  int tma_store;        // 1: bf16 Y is written by TMA from a shared-memory staging tile
  int tiles_m, tiles_n, num_tiles;
  int acc_shift;        // integer accumulators hold 2^acc_shift * sum qx qw (8: W4A4, 4: A8 x W4, 0: A8 x W8)
};

// Bounded wait used by every role; on timeout the role stops issuing work.
__device__ __forceinline__ bool wait_or_fail(uint64_t* bar, unsigned parity, int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;  // the common case: one shared-memory round trip
  if (*((volatile int*)abort_flag)) return false;
  if (!mbar_wait_bounded(bar, parity)) {
    *((volatile int*)abort_flag) = 1;
    return false;
  }
  return true;
}

// Epilogue for one 32-row x 256-column slab held by this warp's TMEM lanes.
// acc_kind 0: int32 accumulators of 2^p.acc_shift * sum (integer codes), 1: fp32 (FP4).
// Arrives on `acc_empty` once the slab has been read out of tensor memory.
template <int ACC_KIND>
__device__ __forceinline__ void epilogue_store(const GemmParams& p, uint32_t tacc, int m0, int n0, int q, int lane,
                                               float rowscale, const float* colscale, float gscale,
                                               uint64_t* acc_empty, uint32_t acc_empty_cluster = 0) {
  const int row = m0 + 32 * q + lane;
  const bool row_ok = row < p.M;
  const uint32_t tq = tacc + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
  for (int cc = 0; cc < kBN / 32; ++cc) {
    uint32_t r[32];
    __syncwarp();
    tmem_ld32(tq + (uint32_t)(32 * cc), r);
    tmem_wait_ld();
    const int c0 = n0 + 32 * cc;
    if (!row_ok || c0 >= p.N) continue;
    const bool full = (c0 + 32 <= p.N) && p.vec_ok;
    if (p.out == 2) {  // raw int32 accumulators (integer codes only)
      int32_t* dst = reinterpret_cast<int32_t*>(p.y) + (int64_t)row * p.ldy + c0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<int4*>(dst + j) = make_int4((int)r[j] >> p.acc_shift, (int)r[j + 1] >> p.acc_shift,
                                                        (int)r[j + 2] >> p.acc_shift, (int)r[j + 3] >> p.acc_shift);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < p.N) dst[j] = (int)r[j] >> p.acc_shift;
      }
      continue;
    }
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float a = (ACC_KIND == 0) ? (float)((int)r[j] >> p.acc_shift) : __uint_as_float(r[j]);
      v[j] = a * rowscale;
    }
    if (ACC_KIND == 0) {
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 s = *reinterpret_cast<const float4*>(colscale + c0 + j);
          v[j] *= s.x;
          v[j + 1] *= s.y;
          v[j + 2] *= s.z;
          v[j + 3] *= s.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= (c0 + j < p.N) ? colscale[c0 + j] : 0.f;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= gscale;
    }
    if (p.out == 0) {
      float* dst = reinterpret_cast<float*>(p.y) + (int64_t)row * p.ldy + c0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < p.N) dst[j] = v[j];
      }
    } else {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.y) + (int64_t)row * p.ldy + c0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          __nv_bfloat162 b0 = __floats2bfloat162_rn(v[j], v[j + 1]);
          __nv_bfloat162 b1 = __floats2bfloat162_rn(v[j + 2], v[j + 3]);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(v[j + 4], v[j + 5]);
          __nv_bfloat162 b3 = __floats2bfloat162_rn(v[j + 6], v[j + 7]);
          *reinterpret_cast<uint4*>(dst + j) =
              make_uint4(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1),
                         *reinterpret_cast<uint32_t*>(&b2), *reinterpret_cast<uint32_t*>(&b3));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < p.N) dst[j] = __float2bfloat16_rn(v[j]);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) {
    if (acc_empty_cluster)
      mbar_arrive_cluster(acc_empty_cluster);
    else
      mbar_arrive(acc_empty);
  }
}

// bf16 epilogue through shared memory: the slab is read out of TMEM in two
// 128-column halves, scaled, rounded to bf16 and written into two 128B-swizzled
// 64-column boxes; TMEM is released as soon as the last half has been read;
// one thread stores each half with TMA (which also clips rows >= M, columns >= N).
// `stage` is the 32 KB staging buffer, `ytmap` the bf16 Y tensor map with
// 64 x 128 boxes, `epi_tid` 0..127 the thread's index among the epilogue warps.
__device__ __forceinline__ void epilogue_bf16_tma(const GemmParams& p, const CUtensorMap* ytmap, uint32_t tacc,
                                                  int m0, int n0, int q, int lane, int epi_tid, float gscale,
                                                  uint8_t* stage, uint64_t* acc_empty,
                                                  uint32_t acc_empty_cluster = 0) {
  const uint32_t tq = tacc + ((uint32_t)(32 * q) << 16);
  const int row = 32 * q + lane;  // row within the tile
#pragma unroll 1
  for (int hh = 0; hh < 2; ++hh) {
    if (hh == 1 || epi_tid == 0) {
      // the staging buffer must have been read by the previous TMA store
      if (epi_tid == 0) bulk_wait_read0();
    }
    named_sync(1, 128);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
      tmem_ld32(tq + (uint32_t)(128 * hh + 32 * cc), r);
      tmem_wait_ld();
      uint8_t* box = stage + (cc >> 1) * (kBM * 128);
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // 4 x 16 bytes = 32 bf16 of this chunk
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 8 * k + 2 * e;
          __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r[j]) * gscale, __uint_as_float(r[j + 1]) * gscale);
          w[e] = *reinterpret_cast<uint32_t*>(&b);
        }
        const int c16 = 4 * (cc & 1) + k;  // 16-byte chunk within the 128-byte box row
        *reinterpret_cast<uint4*>(box + row * 128 + 16 * (c16 ^ (row & 7))) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    if (hh == 1) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // accumulator free for the next tile's MMAs
        if (acc_empty_cluster)
          mbar_arrive_cluster(acc_empty_cluster);
        else
          mbar_arrive(acc_empty);
      }
    }
    fence_proxy_async_smem();
    named_sync(1, 128);
    if (epi_tid == 0) {
      tma_store_2d(ytmap, stage, n0 + 128 * hh, m0);
      tma_store_2d(ytmap, stage + kBM * 128, n0 + 128 * hh + 64, m0);
      bulk_commit();
    }
  }
}

// ---------------------------------------------------------------------------
// INT4 x INT4 -> int32 (kind::i8)
// ---------------------------------------------------------------------------
constexpr int kI4BK = 128;                 // K elements per k-tile (64 packed bytes per row)
constexpr int kI4Stg = 3;                  // packed staging stages
constexpr int kI4Ops = 3;                  // widened operand stages
constexpr int kI4ConvWarps = 8;            // nibble -> int8 converter warps (warps 2..9)
constexpr int kI4Threads = 32 * (2 + kI4ConvWarps + 4);
constexpr int kI4StgA = kBM * 64, kI4StgB = kBN * 64;
constexpr int kI4OpA = kBM * 128, kI4OpB = kBN * 128;
constexpr size_t kI4Smem = 1024 + (size_t)kI4Stg * (kI4StgA + kI4StgB) + (size_t)kI4Ops * (kI4OpA + kI4OpB) + 256;

// Widen 16 packed bytes (32 INT4 codes, element 2i in the low nibble) to 32
// bytes of int8 holding 16*q.
__device__ __forceinline__ void widen16(const uint4 in, uint4& o0, uint4& o1) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = (w[i] << 4) & 0xF0F0F0F0u;  // elements 0,2,4,6 (x16)
    const uint32_t hi = w[i] & 0xF0F0F0F0u;         // elements 1,3,5,7 (x16)
    o[2 * i] = __byte_perm(lo, hi, 0x5140);
    o[2 * i + 1] = __byte_perm(lo, hi, 0x7362);
  }
  o0 = make_uint4(o[0], o[1], o[2], o[3]);
  o1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// Widen one 16-byte chunk j (32 codes) of packed row r (64B-swizzled staging)
// into two 16-byte chunks of the 128B-swizzled int8 row.  Jobs are numbered
// row-major (4 per row), so the 8 threads of a shared-memory phase touch 8
// distinct bank groups both when reading and when writing.
__device__ __forceinline__ void convert_chunk(const uint8_t* stg, uint8_t* op, int r, int j) {
  const uint4 in = *reinterpret_cast<const uint4*>(stg + r * 64 + 16 * (j ^ ((r >> 1) & 3)));
  uint4 o0, o1;
  widen16(in, o0, o1);
  const int sw_out = r & 7;
  *reinterpret_cast<uint4*>(op + r * 128 + 16 * ((2 * j) ^ sw_out)) = o0;
  *reinterpret_cast<uint4*>(op + r * 128 + 16 * ((2 * j + 1) ^ sw_out)) = o1;
}

// The same widening split in two: job jb = 4 r + j reads chunk j of packed
// row r, and writes its two widened chunks.
__device__ __forceinline__ uint4 load_chunk(const uint8_t* stg, int jb) {
  const int r = jb >> 2, j = jb & 3;
  return *reinterpret_cast<const uint4*>(stg + r * 64 + 16 * (j ^ ((r >> 1) & 3)));
}
__device__ __forceinline__ void store_widened(uint8_t* op, int jb, uint4 in) {
  const int r = jb >> 2, j = jb & 3;
  uint4 o0, o1;
  widen16(in, o0, o1);
  const int sw_out = r & 7;
  *reinterpret_cast<uint4*>(op + r * 128 + 16 * ((2 * j) ^ sw_out)) = o0;
  *reinterpret_cast<uint4*>(op + r * 128 + 16 * ((2 * j + 1) ^ sw_out)) = o1;
}

__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* op = base;                                            // [kI4Ops][A 16K | B 32K]
  uint8_t* stg = op + (size_t)kI4Ops * (kI4OpA + kI4OpB);        // [kI4Stg][A 8K | B 16K]
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + (size_t)kI4Stg * (kI4StgA + kI4StgB));
  uint64_t* stg_full = bars;
  uint64_t* stg_empty = stg_full + kI4Stg;
  uint64_t* op_full = stg_empty + kI4Stg;
  uint64_t* op_empty = op_full + kI4Ops;
  uint64_t* acc_full = op_empty + kI4Ops;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KT = p.K / kI4BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kI4Stg; ++i) {
      mbar_init(&stg_full[i], 1);
      mbar_init(&stg_empty[i], kI4ConvWarps);
    }
    for (int i = 0; i < kI4Ops; ++i) {
      mbar_init(&op_full[i], kI4ConvWarps);
      mbar_init(&op_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      unsigned ph = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int m0 = (tile % p.tiles_m) * kBM, n0 = (tile / p.tiles_m) * kBN;
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&stg_empty[s], ph ^ 1, abort_flag)) goto done;
          uint8_t* sa = stg + (size_t)s * (kI4StgA + kI4StgB);
          mbar_arrive_expect_tx(&stg_full[s], kI4StgA + kI4StgB);
          tma_load_2d(sa, &tmap_x, kt * 64, m0, &stg_full[s]);
          tma_load_2d(sa + kI4StgA, &tmap_w, kt * 64, n0, &stg_full[s]);
          if (++s == kI4Stg) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_i8(kBM, kBN);
      int o = 0;
      unsigned oph = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
        const int ab = it & 1;
        const unsigned aph = (unsigned)((it >> 1) & 1);
        if (!wait_or_fail(&acc_empty[ab], aph ^ 1, abort_flag)) goto done;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(ab * kBN);
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&op_full[o], oph, abort_flag)) goto done;
          tc_fence_after();
          const uint8_t* a = op + (size_t)o * (kI4OpA + kI4OpB);
          const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + kI4OpA);
#pragma unroll
          for (int j = 0; j < kI4BK / 32; ++j)
            mma_i8(d, ad + 2 * j, bd + 2 * j, idesc, (kt | j) != 0);
          tc_commit(&op_empty[o]);
          if (++o == kI4Ops) { o = 0; oph ^= 1; }
        }
        tc_commit(&acc_full[ab]);
      }
    }
  } else if (warp < 2 + kI4ConvWarps) {
    // converters: (kBM + kBN) rows x 4 chunks per k-tile, split over the converter threads
    const int t = threadIdx.x - 64;
    int s = 0, o = 0;
    unsigned ph = 0, oph = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      for (int kt = 0; kt < KT; ++kt) {
        if (!wait_or_fail(&stg_full[s], ph, abort_flag)) goto done;
        if (!wait_or_fail(&op_empty[o], oph ^ 1, abort_flag)) goto done;
        const uint8_t* sa = stg + (size_t)s * (kI4StgA + kI4StgB);
        uint8_t* oa = op + (size_t)o * (kI4OpA + kI4OpB);
        constexpr int kJobs = (kBM + kBN) * 4, kConvThreads = 32 * kI4ConvWarps;
#pragma unroll
        for (int jb = t; jb < kJobs; jb += kConvThreads) {
          const int r = jb >> 2, j = jb & 3;
          if (r < kBM)
            convert_chunk(sa, oa, r, j);
          else
            convert_chunk(sa + kI4StgA, oa + kI4OpA, r - kBM, j);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&op_full[o]);
          mbar_arrive(&stg_empty[s]);
        }
        if (++s == kI4Stg) { s = 0; ph ^= 1; }
        if (++o == kI4Ops) { o = 0; oph ^= 1; }
      }
    }
  } else {
    // epilogue
    const int q = warp & 3;
    const float* xs = static_cast<const float*>(p.xscale);
    const float* ws = static_cast<const float*>(p.wscale);
    int it = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
      const int m0 = (tile % p.tiles_m) * kBM, n0 = (tile / p.tiles_m) * kBN;
      const int ab = it & 1;
      const unsigned aph = (unsigned)((it >> 1) & 1);
      if (!wait_or_fail(&acc_full[ab], aph, abort_flag)) goto done;
      tc_fence_after();
      const int row = m0 + 32 * q + lane;
      const float sx = (row < p.M) ? xs[row] : 0.f;
      epilogue_store<0>(p, tmem + (uint32_t)(ab * kBN), m0, n0, q, lane, sx, ws, 1.0f, &acc_empty[ab]);
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// NVFP4 x NVFP4 -> fp32 (kind::mxf4nvf4, block16 E4M3 scales)
// ---------------------------------------------------------------------------
// The 32-bit tensor-memory word of one row's scales for MMA j (K = 64) of
// k-tile kt, from the row's 16 staged scale bytes.  NVFP4: the four E4M3
// scales 4j..4j+3 of the k-tile.  MXFP4: the two E8M0 scales of the MMA,
// bytes 8*(kt & 1) + 2j and + 1 (the 16 bytes span two k-tiles), in the low
// half of the word.
template <bool MX>
__device__ __forceinline__ uint32_t sf_word(const uint4& row16, int j, int kt) {
  // j is a compile-time constant in the callers' unrolled loops; the k-tile
  // parity only selects between two statically indexed words, so the staged
  // scales stay in registers
  const uint32_t w[4] = {row16.x, row16.y, row16.z, row16.w};
  if (!MX) return w[j];
  const uint32_t h = (kt & 1) ? w[2 + (j >> 1)] : w[j >> 1];
  return (j & 1) ? (h >> 16) : (h & 0xFFFFu);
}

constexpr int kF4BK = 256;                 // K elements per k-tile (128 packed bytes per row)
constexpr int kF4St = 3;
constexpr int kF4OpA = kBM * 128, kF4OpB = kBN * 128;
constexpr int kF4SfA = kBM * 16, kF4SfB = kBN * 16;          // 16 E4M3 scales per row per k-tile
constexpr int kF4Stage = kF4OpA + kF4OpB + kF4SfA + kF4SfB;
constexpr int kEpiStage = kBM * 128 * 2;   // bf16 staging: two 64-column boxes of 128 rows (32 KB)
constexpr size_t kF4Smem = 1024 + (size_t)kF4St * kF4Stage + kEpiStage + 256;
constexpr uint32_t kF4SfCol0 = 256;        // TMEM columns [256, 256 + 48*stages) hold the scales
constexpr uint32_t kF4SfCols = 48;         // per stage: SFA 16 columns, SFB 32 columns

template <bool MX>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_sx, const __grid_constant__ CUtensorMap tmap_sw,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  griddep_wait();
  griddep_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* op = base;
  uint8_t* epi_stage = op + (size_t)kF4St * kF4Stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_stage + kEpiStage);
  uint64_t* op_full = bars;
  uint64_t* op_empty = op_full + kF4St;
  uint64_t* sf_full = op_empty + kF4St;
  uint64_t* acc_full = sf_full + kF4St;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KT = p.K / kF4BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kF4St; ++i) {
      mbar_init(&op_full[i], 1);
      mbar_init(&op_empty[i], 1);
      mbar_init(&sf_full[i], 4);
    }
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_empty[0], 4);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_sx);
    prefetch_tmap(&tmap_sw);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      unsigned ph = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int m0 = (tile % p.tiles_m) * kBM, n0 = (tile / p.tiles_m) * kBN;
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&op_empty[s], ph ^ 1, abort_flag)) goto done;
          uint8_t* sa = op + (size_t)s * kF4Stage;
          mbar_arrive_expect_tx(&op_full[s], kF4Stage);
          tma_load_2d(sa, &tmap_x, kt * 128, m0, &op_full[s]);
          tma_load_2d(sa + kF4OpA, &tmap_w, kt * 128, n0, &op_full[s]);
          const int sx0 = MX ? (kt >> 1) * 16 : kt * 16;  // 16-byte aligned scale column
          tma_load_2d(sa + kF4OpA + kF4OpB, &tmap_sx, sx0, m0, &op_full[s]);
          tma_load_2d(sa + kF4OpA + kF4OpB + kF4SfA, &tmap_sw, sx0, n0, &op_full[s]);
          if (++s == kF4St) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_fp4(kBM, kBN, MX);
      int s = 0;
      unsigned ph = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
        if (!wait_or_fail(&acc_empty[0], (unsigned)(it & 1) ^ 1, abort_flag)) goto done;
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&op_full[s], ph, abort_flag)) goto done;
          if (!wait_or_fail(&sf_full[s], ph, abort_flag)) goto done;
          tc_fence_after();
          const uint8_t* a = op + (size_t)s * kF4Stage;
          const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + kF4OpA);
          const uint32_t sf = tmem + kF4SfCol0 + (uint32_t)s * kF4SfCols;
#pragma unroll
          for (int j = 0; j < kF4BK / 64; ++j)
            mma_fp4<MX>(tmem, ad + 2 * j, bd + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j, (kt | j) != 0);
          tc_commit(&op_empty[s]);
          if (++s == kF4St) { s = 0; ph ^= 1; }
        }
        tc_commit(&acc_full[0]);
      }
    }
  } else if (warp < 6) {
    // scale movers: the stage's scales arrived by TMA with the operands; this
    // warp copies the rows of its TMEM lane quadrant q into tensor memory.
    const int q = warp & 3;
    int s = 0;
    unsigned ph = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      for (int kt = 0; kt < KT; ++kt) {
        // op_full of this round implies the MMAs of the previous round on this
        // stage (and so their reads of its scale columns) have completed
        if (!wait_or_fail(&op_full[s], ph, abort_flag)) goto done;
        const uint8_t* sfa = op + (size_t)s * kF4Stage + kF4OpA + kF4OpB;
        const uint8_t* sfb = sfa + kF4SfA;
        uint4 ua[4], ub[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) ua[i] = *reinterpret_cast<const uint4*>(sfa + (lane + 32 * i) * 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) ub[i] = *reinterpret_cast<const uint4*>(sfb + (lane + 32 * i) * 16);
        uint32_t da[16], db0[16], db1[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int i = 0; i < 4; ++i) da[4 * j + i] = sf_word<MX>(ua[i], j, kt);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = 8 * j + i;
            if (c < 16)
              db0[c] = sf_word<MX>(ub[i], j, kt);
            else
              db1[c - 16] = sf_word<MX>(ub[i], j, kt);
          }
        }
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + kF4SfCol0 + (uint32_t)s * kF4SfCols;
        tmem_st16(tq, da);
        tmem_st16(tq + 16, db0);
        tmem_st16(tq + 32, db1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[s]);
        if (++s == kF4St) { s = 0; ph ^= 1; }
      }
    }
  } else {
    const int q = warp & 3;
    const float g = MX ? 1.0f : (*p.xg) * (*p.wg);
    int it = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++it) {
      const int m0 = (tile % p.tiles_m) * kBM, n0 = (tile / p.tiles_m) * kBN;
      if (!wait_or_fail(&acc_full[0], (unsigned)(it & 1), abort_flag)) goto done;
      tc_fence_after();
      if (p.tma_store)
        epilogue_bf16_tma(p, &tmap_y, tmem, m0, n0, q, lane, threadIdx.x - 192, g, epi_stage, &acc_empty[0]);
      else
        epilogue_store<1>(p, tmem, m0, n0, q, lane, 1.0f, nullptr, g, &acc_empty[0]);
    }
  }
done:
  if (threadIdx.x == 192) bulk_wait0();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// NVFP4 on two SMs (cta_group::2, 256 x 256 tiles).  Each CTA loads its own 128
// rows of X and its own 128 of the tile's 256 rows of W; those copies count on
// the even CTA's barrier, whose MMA consumes both halves.  Each CTA's scales
// come by a local copy; its scale warps move them into its own tensor memory,
// one 32-bit column per 32 rows and 64-wide K slice, replicated in the four
// lane quadrants: SFA of its own 128 X rows, and SFB of ALL 256 W rows of the
// tile (each SM's tensor core multiplies its rows by every column of the tile,
// so it reads the scales of both W halves from its own tensor memory).  Then
// they arrive on the even CTA's operand barrier, which so completes once the
// k-tile's operands have landed and its scales are in both CTAs' tensor
// memory: the MMA thread waits on one barrier per k-tile.
// ---------------------------------------------------------------------------
constexpr int kN2St = 5;
constexpr int kN2OpA = 128 * 128, kN2OpB = 128 * 128, kN2SfA = 128 * 16, kN2SfB = 256 * 16;
constexpr int kN2Stage = kN2OpA + kN2OpB + kN2SfA + kN2SfB;       // 38 KB
constexpr size_t kN2Smem = 1024 + (size_t)kN2St * kN2Stage + kEpiStage + 256;
constexpr uint32_t kN2SfCols = 48;                                // per stage: SFA 16 + SFB 32 columns
constexpr int kN2SfWarps = 8;                                     // scale movers (warps 2..9)
constexpr int kN2Threads = 32 * (2 + kN2SfWarps + 4);

template <bool MX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kN2Threads, 1)
    gemm_fp4_2sm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ CUtensorMap tmap_sx, const __grid_constant__ CUtensorMap tmap_sw,
                          const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  griddep_wait();
  griddep_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* op = base;
  uint8_t* epi_stage = op + (size_t)kN2St * kN2Stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_stage + kEpiStage);
  uint64_t* op_full = bars;                 // even CTA: both CTAs' X/W copies and scales in TMEM
  uint64_t* op_empty = op_full + kN2St;     // both: multicast MMA commit
  uint64_t* sf_full = op_empty + kN2St;     // local: this CTA's scale copies
  uint64_t* acc_full = sf_full + kN2St;
  uint64_t* acc_empty = acc_full + 1;       // even CTA: both epilogues
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KT = p.K / kF4BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kN2St; ++i) {
      // the producer's arrival with the copies' bytes, and one per scale mover
      // warp that wrote this k-tile's scales (4 quadrants x 2 CTAs)
      mbar_init(&op_full[i], 1 + 8);
      mbar_init(&op_empty[i], 1);
      mbar_init(&sf_full[i], 1);
    }
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_empty[0], 8);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_sx);
    prefetch_tmap(&tmap_sw);
  }
  if (warp == 1) {
    tmem_alloc_2cta(tmem_slot, 512);
    tmem_relinquish_2cta();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      unsigned ph = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs) {
        const int m0 = (tile % p.tiles_m) * 256 + 128 * (int)rank;
        const int nb = (tile / p.tiles_m) * 256 + 128 * (int)rank;
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&op_empty[s], ph ^ 1, abort_flag)) goto done;
          uint8_t* sa = op + (size_t)s * kN2Stage;
          if (leader) mbar_arrive_expect_tx(&op_full[s], 2 * (kN2OpA + kN2OpB));
          const uint32_t fb = mapa_u32(&op_full[s], 0);
          tma_load_2d_2cta(sa, &tmap_x, kt * 128, m0, fb);
          tma_load_2d_2cta(sa + kN2OpA, &tmap_w, kt * 128, nb, fb);
          mbar_arrive_expect_tx(&sf_full[s], kN2SfA + kN2SfB);
          const int sx0 = MX ? (kt >> 1) * 16 : kt * 16;  // 16-byte aligned scale column
          tma_load_2d(sa + kN2OpA + kN2OpB, &tmap_sx, sx0, m0, &sf_full[s]);
          tma_load_2d(sa + kN2OpA + kN2OpB + kN2SfA, &tmap_sw, sx0, nb - 128 * (int)rank, &sf_full[s]);
          if (++s == kN2St) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_fp4(256, kBN, MX);
      int s = 0;
      unsigned ph = 0;
      int it = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs, ++it) {
        if (!wait_or_fail(&acc_empty[0], (unsigned)(it & 1) ^ 1, abort_flag)) goto done;
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&op_full[s], ph, abort_flag)) goto done;  // operands and scales
          tc_fence_after();
          const uint8_t* a = op + (size_t)s * kN2Stage;
          const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + kN2OpA);
          const uint32_t sf = tmem + kF4SfCol0 + (uint32_t)s * kN2SfCols;
#pragma unroll
          for (int j = 0; j < kF4BK / 64; ++j)
            mma_fp4_2cta<MX>(tmem, ad + 2 * j, bd + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j, (kt | j) != 0);
          tc_commit_2cta_mc(&op_empty[s], 0x3);
          if (++s == kN2St) { s = 0; ph ^= 1; }
        }
        tc_commit_2cta_mc(&acc_full[0], 0x3);
      }
    }
  } else if (warp < 2 + kN2SfWarps) {
    // scale movers: two warps per lane quadrant take alternate k-tiles
    const int q = warp & 3;
    const int par = (warp - 2) >> 2;
    int s = 0;
    unsigned ph = 0;
    int n = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs) {
      for (int kt = 0; kt < KT; ++kt, ++n) {
        if ((n & 1) != par) {
          if (++s == kN2St) { s = 0; ph ^= 1; }
          continue;
        }
        // the scale copy of this round follows the producer's wait on op_empty, so
        // the MMAs of the previous round (which read these columns) are done
        if (!wait_or_fail(&sf_full[s], ph, abort_flag)) goto done;
        const uint8_t* sfa = op + (size_t)s * kN2Stage + kN2OpA + kN2OpB;
        const uint8_t* sfb = sfa + kN2SfA;
        uint4 ua[4], ub[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) ua[i] = *reinterpret_cast<const uint4*>(sfa + (lane + 32 * i) * 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) ub[i] = *reinterpret_cast<const uint4*>(sfb + (lane + 32 * i) * 16);
        tc_fence_after();
        uint32_t da[16], db0[16], db1[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int i = 0; i < 4; ++i) da[4 * j + i] = sf_word<MX>(ua[i], j, kt);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = 8 * j + i;
            if (c < 16)
              db0[c] = sf_word<MX>(ub[i], j, kt);
            else
              db1[c - 16] = sf_word<MX>(ub[i], j, kt);
          }
        }
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + kF4SfCol0 + (uint32_t)s * kN2SfCols;
        tmem_st16(tq, da);
        tmem_st16(tq + 16, db0);
        tmem_st16(tq + 32, db1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_u32(&op_full[s], 0));
        if (++s == kN2St) { s = 0; ph ^= 1; }
      }
    }
  } else {
    const int q = warp & 3;
    const float g = MX ? 1.0f : (*p.xg) * (*p.wg);
    int it = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++it) {
      const int m0 = (tile % p.tiles_m) * 256 + 128 * (int)rank;
      const int n0 = (tile / p.tiles_m) * kBN;
      if (!wait_or_fail(&acc_full[0], (unsigned)(it & 1), abort_flag)) goto done;
      tc_fence_after();
      const uint32_t ae = mapa_u32(&acc_empty[0], 0);
      if (p.tma_store)
        epilogue_bf16_tma(p, &tmap_y, tmem, m0, n0, q, lane, threadIdx.x - 32 * (2 + kN2SfWarps), g, epi_stage,
                          &acc_empty[0], ae);
      else
        epilogue_store<1>(p, tmem, m0, n0, q, lane, 1.0f, nullptr, g, &acc_empty[0], ae);
    }
  }
done:
  if (threadIdx.x == 32 * (2 + kN2SfWarps)) bulk_wait0();
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2cta(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// INT4 x INT4 on two SMs with A in tensor memory (kind::i8, cta_group::2).
//
// Widening nibbles to int8 through shared memory costs a store and a tensor
// core read of every widened byte; with both operands there, the stores, the
// staging writes and the MMA reads together exceed the shared-memory
// bandwidth that an M = 256 MMA leaves.  Here only B goes through shared
// memory: four warps, one per TMEM lane quadrant, widen the A rows in
// registers and write them into TMEM with tcgen05.st (32 columns per k-tile),
// and the MMA reads A from there.  TMEM: accumulator columns [0, 256), A
// stages from column 256 (32 columns each).  With the accumulator single
// buffered, the epilogue releases it as soon as its last columns are read
// and stores bf16 through shared memory with TMA.
//
// Warps: 0 TMA producer, 1 MMA issuer (even CTA), 2..9 B converters,
// 10..13 A converters, 14..21 epilogue.
//
// The same kernel serves 8-bit activation codes (A8: W4A8, W6A6, W8A8; the
// 6-bit codes are int8 bytes in [-31, 31]): the A rows are staged as int8
// (128B-swizzled) and the A warps copy them into TMEM unchanged.  With 8-bit
// weight codes (W8) the B tiles need no widening: TMA writes them straight
// into the 128B-swizzled operand ring, signalling the even CTA's barrier
// (cta_group::2 copies), and the B converter warps sit idle.  acc holds
// 2^shift * sum qx qw with shift = 8 (W4A4: both sides widened as 16 q),
// 4 (A8 x W4) or 0 (A8 x W8).
// ---------------------------------------------------------------------------
constexpr int kI3BWarps = 8;
constexpr int kI3AWarp0 = 2 + kI3BWarps;      // 10
constexpr int kI3EpiWarp0 = kI3AWarp0 + 4;    // 14
constexpr int kI3EpiWarps = 8;                // two per TMEM lane quadrant, 128 columns each
constexpr int kI3Threads = 32 * (kI3EpiWarp0 + kI3EpiWarps);
constexpr int kI3OpB = 128 * 128;
constexpr uint32_t kI3ACol0 = 256;
template <bool A8, bool W8>
struct I3 {
  static constexpr int StgA = A8 ? 128 * 128 : 128 * 64;  // A tile per k-tile: int8 or packed nibbles
  static constexpr int StgB = W8 ? 0 : 128 * 64;          // packed W (W8: straight into the operand ring)
  static constexpr int Stg = A8 ? 4 : 6;                  // staging depth within 227 KB
  static constexpr int Ops = W8 ? 6 : 4;                   // operand ring: B in smem, A in TMEM (32 columns each)
  static constexpr int BArr = W8 ? 0 : kI3BWarps;         // B converter arrivals per k-tile and CTA
  static constexpr int Shift = A8 ? (W8 ? 0 : 4) : (W8 ? 4 : 8);  // A4 x W8: 16 qx against the int8 codes of W
  static constexpr size_t Smem = 1024 + (size_t)Ops * kI3OpB + (size_t)Stg * (StgA + StgB) + 2 * kEpiStage + 256;
  static_assert(Smem <= 232448, "fits the 227 KB of shared memory a CTA may use");
};
constexpr size_t kI3Smem = I3<false, false>::Smem;

// Integer bf16 epilogue through shared memory for one 128-column half `ch` of
// the CTA's 128 x 256 accumulator, by the four warps (one per lane quadrant)
// that own that half: y = (acc >> SHIFT) * sx[row] * sw[col], the arithmetic
// of epilogue_store.  For W4A4 acc >> 8 (|.| < 2^22 for K <= 65536) becomes a
// float exactly through the 1.5 * 2^23 magic number; wider codes convert with
// cvt (exact below 2^24, rounded to nearest above).  `stage` is this half's 32 KB
// of staging (two 128B-swizzled 64-column boxes); one thread stores it with
// TMA (which clips rows >= M and columns >= N).  Named barrier 1 + ch.
template <int SHIFT>
__device__ __forceinline__ void epilogue_int4_bf16_tma(const GemmParams& p, const CUtensorMap* ytmap, uint32_t tacc,
                                                       int m0, int n0, int q, int ch, int lane, float sx,
                                                       const float* ws, uint8_t* stage,
                                                       uint32_t acc_empty_cluster) {
  const uint32_t tq = tacc + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * ch);
  const int row = 32 * q + lane;  // row within the CTA's 128
  const bool issuer = (q == 0 && lane == 0);
  if (issuer) bulk_wait_read0();  // the previous tile's TMA store has read the staging buffer
  named_sync(1 + ch, 128);
#pragma unroll 1
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t r[32];
    tmem_ld32(tq + (uint32_t)(32 * cc), r);
    tmem_wait_ld();
    if (cc == 3) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_cluster);  // this warp's accumulator lanes are read
    }
    const int c0 = n0 + 128 * ch + 32 * cc;
    float sw[32];
    if (c0 + 32 <= p.N) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 t = *reinterpret_cast<const float4*>(ws + c0 + j);
        sw[j] = t.x;
        sw[j + 1] = t.y;
        sw[j + 2] = t.z;
        sw[j + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) sw[j] = (c0 + j < p.N) ? ws[c0 + j] : 0.f;
    }
    uint8_t* box = stage + (cc >> 1) * (kBM * 128);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 8 * k + 2 * e;
        float i0, i1;
        if (SHIFT == 8) {
          i0 = __int_as_float(((int)r[j] >> 8) + 0x4B400000) - kRoundMagic;
          i1 = __int_as_float(((int)r[j + 1] >> 8) + 0x4B400000) - kRoundMagic;
        } else {
          i0 = __int2float_rn((int)r[j] >> SHIFT);
          i1 = __int2float_rn((int)r[j + 1] >> SHIFT);
        }
        __nv_bfloat162 b = __floats2bfloat162_rn(i0 * sx * sw[j], i1 * sx * sw[j + 1]);
        w[e] = *reinterpret_cast<uint32_t*>(&b);
      }
      const int c16 = 4 * (cc & 1) + k;
      *reinterpret_cast<uint4*>(box + row * 128 + 16 * (c16 ^ (row & 7))) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  fence_proxy_async_smem();
  named_sync(1 + ch, 128);
  if (issuer) {
    tma_store_2d(ytmap, stage, n0 + 128 * ch, m0);
    tma_store_2d(ytmap, stage + kBM * 128, n0 + 128 * ch + 64, m0);
    bulk_commit();
  }
}

template <bool A8, bool W8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kI3Threads, 1)
    gemm_int_2sm_ts_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
  griddep_wait();
  griddep_trigger();
  using C = I3<A8, W8>;
  constexpr int kI3Stg = C::Stg, kI3StgA = C::StgA, kI3StgB = C::StgB, kI3Ops = C::Ops;
  static_assert(kI3ACol0 + 32 * kI3Ops <= 512, "A stages fit the TMEM allocation");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* opb = base;                                         // [kI3Ops][B 16K], 128B-swizzled int8
  uint8_t* stg = opb + (size_t)kI3Ops * kI3OpB;                // [kI3Stg][A | B]: nibbles 64B-swizzled, int8 128B-swizzled
  uint8_t* epi = stg + (size_t)kI3Stg * (kI3StgA + kI3StgB);   // bf16 output staging, one 32 KB half per column half
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi + 2 * kEpiStage);
  uint64_t* stg_full = bars;
  uint64_t* stg_empty = stg_full + kI3Stg;
  uint64_t* op_full = stg_empty + kI3Stg;     // used in the even CTA only
  uint64_t* op_empty = op_full + kI3Ops;
  uint64_t* acc_full = op_empty + kI3Ops;
  uint64_t* acc_empty = acc_full + 1;         // used in the even CTA only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KT = p.K / kI4BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kI3Stg; ++i) {
      mbar_init(&stg_full[i], 1);
      mbar_init(&stg_empty[i], C::BArr + 4);
    }
    for (int i = 0; i < kI3Ops; ++i) {
      // A warps of both CTAs, B converters of both CTAs or (W8) the even
      // CTA's producer with the transaction bytes of both B copies
      mbar_init(&op_full[i], 2 * (C::BArr + 4) + (W8 ? 1 : 0));
      mbar_init(&op_empty[i], 1);
    }
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_empty[0], 2 * kI3EpiWarps);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
    if (p.tma_store) prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    tmem_alloc_2cta(tmem_slot, 512);
    tmem_relinquish_2cta();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0, o = 0;
      unsigned ph = 0, oph = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs) {
        const int m0 = (tile % p.tiles_m) * 256 + 128 * (int)rank;
        const int nb = (tile / p.tiles_m) * 256 + 128 * (int)rank;
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&stg_empty[s], ph ^ 1, abort_flag)) goto done;
          uint8_t* sa = stg + (size_t)s * (kI3StgA + kI3StgB);
          mbar_arrive_expect_tx(&stg_full[s], kI3StgA + kI3StgB);
          tma_load_2d(sa, &tmap_x, kt * (A8 ? 128 : 64), m0, &stg_full[s]);
          if (W8) {
            // the operand slot is free once the MMAs that read it have completed
            if (!wait_or_fail(&op_empty[o], oph ^ 1, abort_flag)) goto done;
            if (leader) mbar_arrive_expect_tx(&op_full[o], 2 * kI3OpB);
            tma_load_2d_2cta(opb + (size_t)o * kI3OpB, &tmap_w, kt * 128, nb, mapa_u32(&op_full[o], 0));
            if (++o == kI3Ops) { o = 0; oph ^= 1; }
          } else {
            tma_load_2d(sa + kI3StgA, &tmap_w, kt * 64, nb, &stg_full[s]);
          }
          if (++s == kI3Stg) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_i8(256, 256);
      int o = 0;
      unsigned oph = 0;
      int it = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs, ++it) {
        if (!wait_or_fail(&acc_empty[0], (unsigned)((it & 1) ^ 1), abort_flag)) goto done;
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_or_fail(&op_full[o], oph, abort_flag)) goto done;
          tc_fence_after();
          const uint64_t bd = smem_desc_sw128(opb + (size_t)o * kI3OpB);
          const uint32_t ta = tmem + kI3ACol0 + 32u * (uint32_t)o;
#pragma unroll
          for (int j = 0; j < kI4BK / 32; ++j) mma_i8_2cta_ts(tmem, ta + 8u * (uint32_t)j, bd + 2 * j, idesc, (kt | j) != 0);
          tc_commit_2cta_mc(&op_empty[o], 0x3);
          if (++o == kI3Ops) { o = 0; oph ^= 1; }
        }
        tc_commit_2cta_mc(&acc_full[0], 0x3);
      }
    }
  } else if (warp < kI3AWarp0) {
    // B: packed rows -> 128B-swizzled int8 in shared memory (idle for W8)
    if (W8) goto done;
    const int t = threadIdx.x - 64;
    int s = 0, o = 0;
    unsigned ph = 0, oph = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs) {
      for (int kt = 0; kt < KT; ++kt) {
        if (!wait_or_fail(&stg_full[s], ph, abort_flag)) goto done;
        if (!wait_or_fail(&op_empty[o], oph ^ 1, abort_flag)) goto done;
        const uint8_t* sb = stg + (size_t)s * (kI3StgA + kI3StgB) + kI3StgA;
        uint8_t* ob = opb + (size_t)o * kI3OpB;
static_assert(128 * 4 == 2 * 32 * kI3BWarps, "two widening jobs per thread");
        uint4 in[2];  // both reads issued before the first store
#pragma unroll
        for (int u = 0; u < 2; ++u) in[u] = load_chunk(sb, t + 32 * kI3BWarps * u);
#pragma unroll
        for (int u = 0; u < 2; ++u) store_widened(ob, t + 32 * kI3BWarps * u, in[u]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster(mapa_u32(&op_full[o], 0));
          mbar_arrive(&stg_empty[s]);
        }
        if (++s == kI3Stg) { s = 0; ph ^= 1; }
        if (++o == kI3Ops) { o = 0; oph ^= 1; }
      }
    }
  } else if (warp < kI3EpiWarp0) {
    // A: one row per thread, widened in registers, written to this warp's TMEM lanes
    const int quad = warp & 3;
    const int row = 32 * quad + lane;
    const uint32_t trow = tmem + ((uint32_t)(32 * quad) << 16) + kI3ACol0;
    int s = 0, o = 0;
    unsigned ph = 0, oph = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs) {
      for (int kt = 0; kt < KT; ++kt) {
        if (!wait_or_fail(&stg_full[s], ph, abort_flag)) goto done;
        if (!wait_or_fail(&op_empty[o], oph ^ 1, abort_flag)) goto done;
        tc_fence_after();
        uint32_t w[32];
        if (A8) {
          // 128 int8 codes, 16-byte chunk j at 16 (j ^ (row mod 8))
          const uint8_t* sa = stg + (size_t)s * (kI3StgA + kI3StgB) + row * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 in = *reinterpret_cast<const uint4*>(sa + 16 * (j ^ (row & 7)));
            w[4 * j + 0] = in.x;
            w[4 * j + 1] = in.y;
            w[4 * j + 2] = in.z;
            w[4 * j + 3] = in.w;
          }
        } else {
        const uint8_t* sa = stg + (size_t)s * (kI3StgA + kI3StgB) + row * 64;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 in = *reinterpret_cast<const uint4*>(sa + 16 * (j ^ ((row >> 1) & 3)));
          uint4 o0, o1;
          widen16(in, o0, o1);
          w[8 * j + 0] = o0.x;
          w[8 * j + 1] = o0.y;
          w[8 * j + 2] = o0.z;
          w[8 * j + 3] = o0.w;
          w[8 * j + 4] = o1.x;
          w[8 * j + 5] = o1.y;
          w[8 * j + 6] = o1.z;
          w[8 * j + 7] = o1.w;
        }
        }
        tmem_st32(trow + 32u * (uint32_t)o, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster(mapa_u32(&op_full[o], 0));
          mbar_arrive(&stg_empty[s]);
        }
        if (++s == kI3Stg) { s = 0; ph ^= 1; }
        if (++o == kI3Ops) { o = 0; oph ^= 1; }
      }
    }
  } else {
    const int q = warp & 3;
    const int ch = (warp - kI3EpiWarp0) >> 2;  // column half of the accumulator
    const float* xs = static_cast<const float*>(p.xscale);
    const float* ws = static_cast<const float*>(p.wscale);
    int it = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++it) {
      const int m0 = (tile % p.tiles_m) * 256 + 128 * (int)rank;
      const int n0 = (tile / p.tiles_m) * 256;
      if (!wait_or_fail(&acc_full[0], (unsigned)(it & 1), abort_flag)) goto done;
      tc_fence_after();
      const int row = m0 + 32 * q + lane;
      const float sx = (row < p.M) ? xs[row] : 0.f;
      if (p.tma_store) {
        epilogue_int4_bf16_tma<C::Shift>(p, &tmap_y, tmem, m0, n0, q, ch, lane, sx, ws,
                                         epi + (size_t)ch * kEpiStage, mapa_u32(&acc_empty[0], 0));
      } else if (ch == 0) {
        epilogue_store<0>(p, tmem, m0, n0, q, lane, sx, ws, 1.0f, &acc_empty[0], mapa_u32(&acc_empty[0], 0));
      } else {
        __syncwarp();  // the other half's warps do the whole slab on this path
        if (lane == 0) mbar_arrive_cluster(mapa_u32(&acc_empty[0], 0));
      }
    }
    if (q == 0 && lane == 0) bulk_wait0();  // stores out of shared memory complete before the CTA exits
  }
done:
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync();  // no CTA leaves while the pair's MMAs may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_2cta(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D byte tensor [rows, cols] (row pitch = cols bytes), box [box_rows, box_cols].
inline bool make_tmap_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                         uint32_t box_cols, CUtensorMapSwizzle sw) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 Y [rows, cols] with row pitch ld elements, 64 x 128 boxes, 128B swizzle.
inline bool make_tmap_y_bf16(CUtensorMap* m, void* ptr, uint64_t rows, uint64_t cols, uint64_t ld) {
  EncodeTiledFn f = encode_fn();
  if (!f) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kBM};
  cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

inline int gemm_num_sms() {
  int dev = 0, v = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
  return v > 0 ? v : 148;
}

// Raise a GEMM kernel's dynamic shared-memory limit once per (kernel, device).
inline bool gemm_ensure_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, uint64_t>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0;
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

// NVFP4 (MX = false: E4M3 scales [rows, K/16]) or MXFP4 (MX = true: E8M0
// scales [rows, K/32]) launch: 2-SM kernel above 128 rows, else 1-SM.
template <bool MX>
rq_status launch_fp4(GemmParams p, const uint8_t* xc, const void* xs, const uint8_t* wc, const void* ws, void* Y,
                     int64_t M, int64_t N, int64_t K, int64_t ldy, rq_out out, cudaStream_t st) {
  const uint64_t sf_cols = (uint64_t)K / (MX ? 32 : 16);
  CUtensorMap tx, tw, tsx, tsw, ty;
  std::memset(&ty, 0, sizeof(ty));
  p.tma_store = (out == RQ_OUT_BF16 && p.vec_ok) ? 1 : 0;
  if (p.tma_store && !make_tmap_y_bf16(&ty, Y, (uint64_t)M, (uint64_t)N, (uint64_t)ldy)) return RQ_ERR_CUDA;
  if (M > kBM) {
    // two SMs per 256 x 256 tile
    if (!make_tmap_u8(&tx, xc, (uint64_t)M, (uint64_t)K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_u8(&tw, wc, (uint64_t)N, (uint64_t)K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_u8(&tsx, xs, (uint64_t)M, sf_cols, 128, 16, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap_u8(&tsw, ws, (uint64_t)N, sf_cols, 256, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
      return RQ_ERR_CUDA;
    p.tiles_m = (int)((M + 255) / 256);
    p.tiles_n = (int)((N + kBN - 1) / kBN);
    p.num_tiles = p.tiles_m * p.tiles_n;
    const int sms = gemm_num_sms() & ~1;
    const int grid2 = 2 * p.num_tiles < sms ? 2 * p.num_tiles : sms;
    if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_fp4_2sm_kernel<MX>), (int)kN2Smem)) return RQ_ERR_CUDA;
    (void)launch_pdl(gemm_fp4_2sm_kernel<MX>, dim3(grid2), dim3(kN2Threads), kN2Smem, st, tx, tw, tsx, tsw, ty, p);
    return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
  }
  if (!make_tmap_u8(&tx, xc, (uint64_t)M, (uint64_t)K / 2, kBM, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_u8(&tw, wc, (uint64_t)N, (uint64_t)K / 2, kBN, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_u8(&tsx, xs, (uint64_t)M, sf_cols, kBM, 16, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_u8(&tsw, ws, (uint64_t)N, sf_cols, kBN, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return RQ_ERR_CUDA;
  const int grid = p.num_tiles < gemm_num_sms() ? p.num_tiles : gemm_num_sms();
  if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_fp4_kernel<MX>), (int)kF4Smem)) return RQ_ERR_CUDA;
  (void)launch_pdl(gemm_fp4_kernel<MX>, dim3(grid), dim3(kGemmThreads), kF4Smem, st, tx, tw, tsx, tsw, ty, p);
  return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

inline rq_status gemm_dispatch(const uint8_t* xc, const void* xs, const float* xg, const uint8_t* wc, const void* ws,
                               const float* wg, int64_t M, int64_t N, int64_t K, rq_format fmt, void* Y, int64_t ldy,
                               rq_out out, cudaStream_t st) {
  if (M < 0 || N < 0 || K <= 0 || ldy < N) return RQ_ERR_INVALID_ARG;
  if (fmt != RQ_INT4 && fmt != RQ_NVFP4 && fmt != RQ_MXFP4) return RQ_ERR_INVALID_ARG;
  if (out != RQ_OUT_F32 && out != RQ_OUT_BF16 && out != RQ_OUT_I32_ACC) return RQ_ERR_INVALID_ARG;
  if (fmt != RQ_INT4 && out == RQ_OUT_I32_ACC) return RQ_ERR_INVALID_ARG;
  if (M > 0 && N > 0) {
    if (!xc || !xs || !wc || !ws || !Y) return RQ_ERR_INVALID_ARG;
    if (fmt == RQ_NVFP4 && (!xg || !wg)) return RQ_ERR_INVALID_ARG;
  }
  if (K > 65536 || M > (int64_t)1 << 30 || N > (int64_t)1 << 30) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt == RQ_INT4 && K % kI4BK != 0) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt == RQ_NVFP4 && K % kF4BK != 0) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (fmt == RQ_MXFP4 && K % 512 != 0) return RQ_ERR_UNSUPPORTED_SHAPE;  // scale rows of K/32 bytes, 16-byte multiples
  if (M == 0 || N == 0) return RQ_OK;
  const size_t esz = out == RQ_OUT_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(xc) | reinterpret_cast<uintptr_t>(wc)) & 15) return RQ_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(Y) % esz != 0) return RQ_ERR_ALIGNMENT;
  if (fmt == RQ_INT4 && ((reinterpret_cast<uintptr_t>(xs) & 3) || (reinterpret_cast<uintptr_t>(ws) & 15)))
    return RQ_ERR_ALIGNMENT;
  if (fmt != RQ_INT4 && ((reinterpret_cast<uintptr_t>(xs) | reinterpret_cast<uintptr_t>(ws)) & 15))
    return RQ_ERR_ALIGNMENT;

  GemmParams p;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.xscale = xs;
  p.wscale = ws;
  p.xg = xg;
  p.wg = wg;
  p.y = Y;
  p.ldy = ldy;
  p.out = (int)out;
  p.vec_ok = ((reinterpret_cast<uintptr_t>(Y) % 16) == 0 && (ldy * (int64_t)esz) % 16 == 0) ? 1 : 0;
  p.tma_store = 0;
  p.acc_shift = 8;
  p.tiles_m = (int)((M + kBM - 1) / kBM);
  p.tiles_n = (int)((N + kBN - 1) / kBN);
  p.num_tiles = p.tiles_m * p.tiles_n;
  const int grid = p.num_tiles < gemm_num_sms() ? p.num_tiles : gemm_num_sms();

  CUtensorMap tx, tw;
  if (fmt == RQ_INT4) {
    if (!make_tmap_u8(&tx, xc, (uint64_t)M, (uint64_t)K / 2, kBM, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_tmap_u8(&tw, wc, (uint64_t)N, (uint64_t)K / 2, kBN, 64, CU_TENSOR_MAP_SWIZZLE_64B))
      return RQ_ERR_CUDA;
    if (M > kBM) {
      // two SMs per 256 x 256 tile
      CUtensorMap tx2, tw2;
      if (!make_tmap_u8(&tx2, xc, (uint64_t)M, (uint64_t)K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
          !make_tmap_u8(&tw2, wc, (uint64_t)N, (uint64_t)K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_64B))
        return RQ_ERR_CUDA;
      p.tiles_m = (int)((M + 255) / 256);
      p.tiles_n = (int)((N + kBN - 1) / kBN);
      p.num_tiles = p.tiles_m * p.tiles_n;
      const int sms = gemm_num_sms() & ~1;
      const int grid2 = 2 * p.num_tiles < sms ? 2 * p.num_tiles : sms;
      CUtensorMap ty;
      std::memset(&ty, 0, sizeof(ty));
      p.tma_store = (out == RQ_OUT_BF16 && p.vec_ok) ? 1 : 0;
      if (p.tma_store && !make_tmap_y_bf16(&ty, Y, (uint64_t)M, (uint64_t)N, (uint64_t)ldy)) return RQ_ERR_CUDA;
      if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_int_2sm_ts_kernel<false, false>), (int)kI3Smem))
        return RQ_ERR_CUDA;
      (void)launch_pdl(gemm_int_2sm_ts_kernel<false, false>, dim3(grid2), dim3(kI3Threads), kI3Smem, st, tx2, tw2, ty, p);
      return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
    }
    if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_int4_kernel), (int)kI4Smem)) return RQ_ERR_CUDA;
    gemm_int4_kernel<<<grid, kI4Threads, kI4Smem, st>>>(tx, tw, p);
  } else {
    return fmt == RQ_MXFP4 ? launch_fp4<true>(p, xc, xs, wc, ws, Y, M, N, K, ldy, out, st)
                           : launch_fp4<false>(p, xc, xs, wc, ws, Y, M, N, K, ldy, out, st);
  }
  return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

// Integer GEMM with 8-bit activation codes (W4A8, W6A6, W8A8 and the mixed
// 6/8-bit pairs): always the two-SM kernel (any M; a pair's second 128 rows
// are clipped by TMA and the epilogue when M <= 128).  W4A4 goes through
// gemm_dispatch.
inline rq_status int_gemm_dispatch(const uint8_t* xc, const float* xs, rq_format xfmt, const uint8_t* wc,
                                   const float* ws, rq_format wfmt, int64_t M, int64_t N, int64_t K, void* Y,
                                   int64_t ldy, rq_out out, cudaStream_t st) {
  auto is_int = [](rq_format f) { return f == RQ_INT4 || f == RQ_INT6 || f == RQ_INT8; };
  const bool a4w8 = xfmt == RQ_INT4 && wfmt == RQ_INT4_BYTES;  // W4A4 with the weight codes one per byte
  if (!a4w8 && (!is_int(xfmt) || !is_int(wfmt))) return RQ_ERR_INVALID_ARG;
  if (xfmt == RQ_INT4 && wfmt == RQ_INT4)
    return gemm_dispatch(xc, xs, nullptr, wc, ws, nullptr, M, N, K, RQ_INT4, Y, ldy, out, st);
  if (xfmt == RQ_INT4 && !a4w8) return RQ_ERR_UNSUPPORTED_SHAPE;  // 4-bit activations with wider weights
  const bool w8 = wfmt != RQ_INT4;
  if (M < 0 || N < 0 || K <= 0 || ldy < N) return RQ_ERR_INVALID_ARG;
  if (out != RQ_OUT_F32 && out != RQ_OUT_BF16 && out != RQ_OUT_I32_ACC) return RQ_ERR_INVALID_ARG;
  if (M > 0 && N > 0 && (!xc || !xs || !wc || !ws || !Y)) return RQ_ERR_INVALID_ARG;
  if (K > 65536 || M > (int64_t)1 << 30 || N > (int64_t)1 << 30) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (K % 128 != 0) return RQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return RQ_OK;
  const size_t esz = out == RQ_OUT_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(xc) | reinterpret_cast<uintptr_t>(wc)) & 15) return RQ_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(Y) % esz != 0) return RQ_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(xs) & 3) || (reinterpret_cast<uintptr_t>(ws) & 15)) return RQ_ERR_ALIGNMENT;

  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.xscale = xs;
  p.wscale = ws;
  p.y = Y;
  p.ldy = ldy;
  p.out = (int)out;
  p.vec_ok = ((reinterpret_cast<uintptr_t>(Y) % 16) == 0 && (ldy * (int64_t)esz) % 16 == 0) ? 1 : 0;
  p.acc_shift = a4w8 ? I3<false, true>::Shift : (w8 ? I3<true, true>::Shift : I3<true, false>::Shift);
  p.tiles_m = (int)((M + 255) / 256);
  p.tiles_n = (int)((N + kBN - 1) / kBN);
  p.num_tiles = p.tiles_m * p.tiles_n;
  const int sms = gemm_num_sms() & ~1;
  const int grid2 = 2 * p.num_tiles < sms ? 2 * p.num_tiles : sms;

  CUtensorMap tx, tw, ty;
  std::memset(&ty, 0, sizeof(ty));
  if (a4w8) {  // packed X nibbles, staged 64B-swizzled for the A converters
    if (!make_tmap_u8(&tx, xc, (uint64_t)M, (uint64_t)K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_64B)) return RQ_ERR_CUDA;
  } else if (!make_tmap_u8(&tx, xc, (uint64_t)M, (uint64_t)K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return RQ_ERR_CUDA;
  }
  if (w8) {
    if (!make_tmap_u8(&tw, wc, (uint64_t)N, (uint64_t)K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) return RQ_ERR_CUDA;
  } else {
    if (!make_tmap_u8(&tw, wc, (uint64_t)N, (uint64_t)K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_64B)) return RQ_ERR_CUDA;
  }
  p.tma_store = (out == RQ_OUT_BF16 && p.vec_ok) ? 1 : 0;
  if (p.tma_store && !make_tmap_y_bf16(&ty, Y, (uint64_t)M, (uint64_t)N, (uint64_t)ldy)) return RQ_ERR_CUDA;
  if (a4w8) {
    if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_int_2sm_ts_kernel<false, true>),
                          (int)I3<false, true>::Smem))
      return RQ_ERR_CUDA;
    (void)launch_pdl(gemm_int_2sm_ts_kernel<false, true>, dim3(grid2), dim3(kI3Threads), I3<false, true>::Smem, st, tx,
                     tw, ty, p);
  } else if (w8) {
    if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_int_2sm_ts_kernel<true, true>),
                          (int)I3<true, true>::Smem))
      return RQ_ERR_CUDA;
    (void)launch_pdl(gemm_int_2sm_ts_kernel<true, true>, dim3(grid2), dim3(kI3Threads), I3<true, true>::Smem, st, tx, tw, ty, p);
  } else {
    if (!gemm_ensure_smem(reinterpret_cast<const void*>(gemm_int_2sm_ts_kernel<true, false>),
                          (int)I3<true, false>::Smem))
      return RQ_ERR_CUDA;
    (void)launch_pdl(gemm_int_2sm_ts_kernel<true, false>, dim3(grid2), dim3(kI3Threads), I3<true, false>::Smem, st, tx, tw, ty, p);
  }
  return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}

}  // namespace rq
