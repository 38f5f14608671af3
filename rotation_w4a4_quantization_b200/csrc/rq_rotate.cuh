// Fused randomized-Hadamard rotation + 4-bit quantization + packing (sm_100a).
//
// What it computes ("Rotations for 4-Bit Activations: QuaRot, SpinQuant, and
// Friends", sections "A rotation changes nothing, and that is the point",
// "What it buys in 4 bits, and what it doesn't", "Gotchas"):
//   X~ = X . Q,  Q = blockdiag(diag(s_blk) . H_B / sqrt(B)),  B = 128 or B = K,
// then one of
//   INT4  : per-row symmetric, s = amax/7, q = rint(x/s)          (tokens / output channels)
//   NVFP4 : E2M1 codes, one E4M3 scale per 16 values, fp32 tensor scale g
//   KV4   : per-vector asymmetric, z = min, s = (max-min)/15 (fp16 scale and zero)
//   F32   : the rotated values themselves (parity checks)
//   AMAX  : only the global max |X~| (first pass of dynamic NVFP4)
// and packs two codes per byte, element 2i in the low nibble.
//
// Design (B200):
// * A CTA owns a tile of R rows.  One thread owns one 128-wide block of one
//   row and keeps it in 128 registers, so all seven butterfly stages of the
//   128-point fast Walsh-Hadamard transform run in registers (no shuffles).
// * Rows reach shared memory through TMA bulk copies (cp.async.bulk, no tensor
//   map, no multicast) into a STAGES-deep ring guarded by mbarriers; one
//   elected thread issues the copies, merging rows that are contiguous in HBM.
// * Bank conflicts: thread u reads 16-byte chunk (j XOR m) into register slot j,
//   m = u mod 8, so the 8 threads of every shared-memory phase hit 8 different
//   bank groups.  Permuting the input by XOR with M = 8m multiplies the
//   Hadamard output k by chi(k) = (-1)^popcount(k & M) (H . P_M = diag(chi) . H),
//   so output k of the registers is chi(k) * y(k) in natural order; chi is
//   folded into the per-chunk multipliers of the quantizer (free).
// * The sign diagonal is applied to the packed bf16 pairs with one XOR per
//   pair, using a per-CTA table of sign masks in shared memory.
// * Full-width rotations (B = K = 128*NB, NB <= 32) use the Kronecker split
//   H_K = H_NB (x) H_128: after the in-register 128-point transform, the
//   block's outputs are transposed through shared memory (the consumed input
//   stage, XOR-swizzled, in two halves) and the NB-point transform across
//   blocks runs in registers again.
// * Rounding to integers uses the 1.5*2^23 "magic" add (the FPU's
//   round-to-nearest-even), whose low mantissa bits are the two's-complement
//   code; packing gathers low bytes with PRMT.
#pragma once

#include "rq_common.cuh"

namespace rq {

enum RotMode : int { kModeInt4 = 0, kModeNvfp4 = 1, kModeF32 = 2, kModeAmax = 3, kModeKv4 = 4 };

struct RotParams {
  const uint8_t* x;    // bf16 input (bytes)
  int64_t rows;        // total rows (vectors of K channels)
  int K;               // channels per row
  int nb;              // K / 128
  // row -> address: t = row % S, bh = row / S, h = bh % H, b = bh / H
  int64_t S, H;
  int64_t sB, sH, sS;  // byte strides
  const int8_t* signs; // [K]
  uint8_t* codes;      // [rows, K/2]
  float* scales_f32;   // INT4: [rows]
  uint8_t* scales_e4m3;// NVFP4: [rows, K/16]
  __half* kv_scale;    // KV4: [rows]
  __half* kv_zero;     // KV4: [rows]
  float* out_f32;      // F32: [rows, ldo]
  int64_t ldo;
  const float* g_in;   // NVFP4 static: the per-tensor scale (device scalar)
  float* g_out;        // NVFP4: the per-tensor scale used (written by CTA 0)
  unsigned* amax_word; // NVFP4 dynamic: max |X~| as fp32 bits (AMAX writes, NVFP4 reads)
  int R;               // rows per tile
  int64_t num_tiles;
  int stages;
  int nvfp4_dynamic;   // 1: g from amax_word, 0: g from g_in
  float cfull;         // 1/sqrt(K) for full-width rotations (rounded once from the exact value)
};

struct RotSmemLayout {
  // [stages][R*K*2] input ring | sign masks [nb*64] u32 | row amax [2][R] u32 | mbarriers [stages] | flag
  static __host__ __device__ size_t stage_bytes(int R, int K) { return (size_t)R * K * 2; }
  static __host__ __device__ size_t total(int R, int K, int stages) {
    size_t b = stage_bytes(R, K) * stages;
    b += (size_t)(K / 128) * 64 * 4;
    b += 2 * (size_t)R * 4;
    b = (b + 7) & ~(size_t)7;
    b += (size_t)stages * 8 + 16;
    return b;
  }
};

__device__ __forceinline__ const uint8_t* row_addr(const RotParams& p, int64_t row) {
  const int64_t t = row % p.S;
  const int64_t bh = row / p.S;
  const int64_t h = bh % p.H;
  const int64_t b = bh / p.H;
  return p.x + b * p.sB + h * p.sH + t * p.sS;
}

// Issue the bulk copies of tile `tile` into `dst` (one elected thread).
__device__ __forceinline__ void issue_tile_load(const RotParams& p, int64_t tile, uint8_t* dst, uint64_t* bar) {
  const int64_t r0 = tile * p.R;
  const int nrows = (int)min((int64_t)p.R, p.rows - r0);
  const unsigned row_bytes = (unsigned)p.K * 2u;
  mbar_arrive_expect_tx(bar, row_bytes * (unsigned)nrows);
  const uint8_t* run_src = row_addr(p, r0);
  unsigned run_bytes = row_bytes;
  int run_row = 0;
  for (int r = 1; r < nrows; ++r) {
    const uint8_t* a = row_addr(p, r0 + r);
    if (a == run_src + run_bytes && run_bytes + row_bytes <= (1u << 19)) {
      run_bytes += row_bytes;
    } else {
      bulk_g2s(dst + (size_t)run_row * row_bytes, run_src, run_bytes, bar);
      run_src = a;
      run_bytes = row_bytes;
      run_row = r;
    }
  }
  bulk_g2s(dst + (size_t)run_row * row_bytes, run_src, run_bytes, bar);
}

// 128-point fast Walsh-Hadamard transform in registers (unnormalized).
__device__ __forceinline__ void fwht128(float (&v)[128]) {
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = a + b;
    v[i + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < 128; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 128; i += 2) {
      if ((i & h) == 0) {
        const float2 a = make_float2(v[i], v[i + 1]);
        const float2 b = make_float2(v[i + h], v[i + h + 1]);
        const float2 s = __fadd2_rn(a, b);
        const float2 d = __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
        v[i] = s.x;
        v[i + 1] = s.y;
        v[i + h] = d.x;
        v[i + h + 1] = d.y;
      }
    }
  }
}

// chi for 8-element chunk `chunk` of a thread with XOR key m: +-1 as a sign bit.
__device__ __forceinline__ uint32_t chi_signbit(int chunk, int m) {
  return (uint32_t)(__popc((unsigned)(chunk & m)) & 1) << 31;
}

__device__ __forceinline__ float with_sign(float x, uint32_t signbit) {
  return __uint_as_float(__float_as_uint(x) ^ signbit);
}

// Load this thread's 128-wide block (XOR-permuted chunks), apply the signs.
__device__ __forceinline__ void load_block(const uint8_t* blk, const uint32_t* smask, int m, float (&v)[128]) {
  const uint4* src = reinterpret_cast<const uint4*>(blk);
  const uint4* msk = reinterpret_cast<const uint4*>(smask);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int c = j ^ m;
    uint4 w = src[c];
    const uint4 s = msk[c];
    w.x ^= s.x;
    w.y ^= s.y;
    w.z ^= s.z;
    w.w ^= s.w;
    v[8 * j + 0] = __uint_as_float(w.x << 16);
    v[8 * j + 1] = __uint_as_float(w.x & 0xFFFF0000u);
    v[8 * j + 2] = __uint_as_float(w.y << 16);
    v[8 * j + 3] = __uint_as_float(w.y & 0xFFFF0000u);
    v[8 * j + 4] = __uint_as_float(w.z << 16);
    v[8 * j + 5] = __uint_as_float(w.z & 0xFFFF0000u);
    v[8 * j + 6] = __uint_as_float(w.w << 16);
    v[8 * j + 7] = __uint_as_float(w.w & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float absmax128(const float (&v)[128]) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 128; i += 4) {
    a0 = fmaxf(a0, fabsf(v[i]));
    a1 = fmaxf(a1, fabsf(v[i + 1]));
    a2 = fmaxf(a2, fabsf(v[i + 2]));
    a3 = fmaxf(a3, fabsf(v[i + 3]));
  }
  return fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
}

// Reduce a non-negative float max over the threads of one row and return it
// to all of them.  Rows are nb consecutive threads.
__device__ __forceinline__ float row_max(float a, int nb, int tid, int r, unsigned* slot_base, bool valid) {
  uint32_t bits = valid ? __float_as_uint(a) : 0u;
  if ((nb & 31) == 0) {
    bits = __reduce_max_sync(0xFFFFFFFFu, bits);
    if ((tid & 31) == 0) atomicMax(slot_base + r, bits);
  } else if ((32 % nb) == 0) {
    for (int o = 1; o < nb; o <<= 1) bits = max(bits, __shfl_xor_sync(0xFFFFFFFFu, bits, o));
    if ((tid % nb) == 0 && valid) slot_base[r] = bits;
  } else {
    if (valid) atomicMax(slot_base + r, bits);
  }
  __syncthreads();
  return __uint_as_float(slot_base[r]);
}

// INT4 per-row quantization of v (true value = v * c * chi) and packing.
// amax_true: the row's max |x~|.  Writes 64 bytes at dst.
__device__ __forceinline__ void quant_int4_store(const float (&v)[128], float c, float amax_true, int m,
                                                 uint8_t* dst) {
  // r = 7/amax; zero rows -> r = 0 -> all codes 0
  const float r = amax_true > 0.f ? __fdiv_rn(7.0f, amax_true) : 0.0f;
  const float cr = c * r;
  uint32_t words[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {  // chunk j = 8 elements -> one word
    const float mul = with_sign(cr, chi_signbit(j, m));
    float q[8];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 t = __ffma2_rn(make_float2(v[8 * j + e], v[8 * j + e + 1]), make_float2(mul, mul),
                                  make_float2(kRoundMagic, kRoundMagic));
      q[e] = t.x;
      q[e + 1] = t.y;
    }
    words[j] = pack8_magic(q);
  }
  uint4* out = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) out[j] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
}

// NVFP4 quantization of v (true value = v * c * chi): 8 groups of 16.
// Writes 64 bytes of codes and 8 bytes of E4M3 scales.
__device__ __forceinline__ void quant_nvfp4_store(const float (&v)[128], float c, float g, float inv6g, int m,
                                                  uint8_t* dst_codes, uint8_t* dst_scales) {
  uint32_t words[16];
  uint32_t sc_lo = 0, sc_hi = 0;
#pragma unroll
  for (int gi = 0; gi < 8; ++gi) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      a0 = fmaxf(a0, fabsf(v[16 * gi + e]));
      a1 = fmaxf(a1, fabsf(v[16 * gi + e + 1]));
    }
    const float amax_b = fmaxf(a0, a1) * c;              // true block max
    const uint32_t scode = f32_to_e4m3(amax_b * inv6g);   // S_b = E4M3(amax_b / (6 g))
    const float sdec = e4m3_to_f32(scode);
    const float denom = sdec * g;
    const float inv = denom > 0.f ? __frcp_rn(denom) : 0.0f;
    const float ci = c * inv;
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
      const int j = 2 * gi + hlf;
      const float mul = with_sign(ci, chi_signbit(j, m));
      const float* s = &v[8 * j];
      words[j] = pack8_e2m1(s[0] * mul, s[1] * mul, s[2] * mul, s[3] * mul, s[4] * mul, s[5] * mul, s[6] * mul,
                            s[7] * mul);
    }
    if (gi < 4)
      sc_lo |= scode << (8 * gi);
    else
      sc_hi |= scode << (8 * (gi - 4));
  }
  uint4* out = reinterpret_cast<uint4*>(dst_codes);
#pragma unroll
  for (int j = 0; j < 4; ++j) out[j] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
  *reinterpret_cast<uint2*>(dst_scales) = make_uint2(sc_lo, sc_hi);
}

// KV4: asymmetric per-vector quantization (true value = v * c * chi).
__device__ __forceinline__ void quant_kv4_store(const float (&v)[128], float c, int m, uint8_t* dst_codes,
                                                __half* dst_scale, __half* dst_zero) {
  float lo = 3.0e38f, hi = -3.0e38f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float cmin = v[8 * j], cmax = v[8 * j];
#pragma unroll
    for (int e = 1; e < 8; ++e) {
      cmin = fminf(cmin, v[8 * j + e]);
      cmax = fmaxf(cmax, v[8 * j + e]);
    }
    if (chi_signbit(j, m)) {
      lo = fminf(lo, -cmax);
      hi = fmaxf(hi, -cmin);
    } else {
      lo = fminf(lo, cmin);
      hi = fmaxf(hi, cmax);
    }
  }
  lo *= c;
  hi *= c;
  const float s = __fdiv_rn(hi - lo, 15.0f);
  const __half s_h = __float2half_rn(s);
  const __half z_h = __float2half_rn(lo);
  const float sf = __half2float(s_h);
  const float zf = __half2float(z_h);
  const float inv = sf > 0.f ? __frcp_rn(sf) : 0.0f;
  const float ci = c * inv;
  const float off = -zf * inv;
  // t = (x - z) / s is monotone in the true value; check the extremes to see
  // whether clamping to [0, 15] can be needed for this vector.
  const float tlo = fmaf(lo, inv, off), thi = fmaf(hi, inv, off);
  const bool need_clamp = !(tlo > -0.5f && thi < 15.5f);
  uint32_t words[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float mul = with_sign(ci, chi_signbit(j, m));
    float q[8];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float2 t = __ffma2_rn(make_float2(v[8 * j + e], v[8 * j + e + 1]), make_float2(mul, mul), make_float2(off, off));
      if (need_clamp) {
        t.x = fminf(fmaxf(t.x, 0.0f), 15.0f);
        t.y = fminf(fmaxf(t.y, 0.0f), 15.0f);
      }
      t = __fadd2_rn(t, make_float2(kRoundMagic, kRoundMagic));
      q[e] = t.x;
      q[e + 1] = t.y;
    }
    words[j] = pack8_magic(q);
  }
  uint4* out = reinterpret_cast<uint4*>(dst_codes);
#pragma unroll
  for (int j = 0; j < 4; ++j) out[j] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
  *dst_scale = s_h;
  *dst_zero = z_h;
}

__device__ __forceinline__ void store_f32_block(const float (&v)[128], float c, int m, float* dst) {
  float4* out = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float mul = with_sign(c, chi_signbit(j, m));
    out[2 * j] = make_float4(v[8 * j] * mul, v[8 * j + 1] * mul, v[8 * j + 2] * mul, v[8 * j + 3] * mul);
    out[2 * j + 1] = make_float4(v[8 * j + 4] * mul, v[8 * j + 5] * mul, v[8 * j + 6] * mul, v[8 * j + 7] * mul);
  }
}

// Kernel prologue shared by both variants: smem carve-up, barrier init, sign
// table, first loads.  Returns false if this CTA has no work.
struct RotSmem {
  uint8_t* ring;
  uint32_t* smask;
  unsigned* row_amax;  // [2][R]
  uint64_t* full;
  int* flag;
};

__device__ __forceinline__ RotSmem carve(uint8_t* base, const RotParams& p) {
  RotSmem s;
  s.ring = base;
  size_t off = RotSmemLayout::stage_bytes(p.R, p.K) * p.stages;
  s.smask = reinterpret_cast<uint32_t*>(base + off);
  off += (size_t)p.nb * 64 * 4;
  s.row_amax = reinterpret_cast<unsigned*>(base + off);
  off += 2 * (size_t)p.R * 4;
  off = (off + 7) & ~(size_t)7;
  s.full = reinterpret_cast<uint64_t*>(base + off);
  off += (size_t)p.stages * 8;
  s.flag = reinterpret_cast<int*>(base + off);
  return s;
}

__device__ __forceinline__ void prologue(const RotParams& p, RotSmem& s) {
  const int tid = threadIdx.x;
  // sign mask table: pair (2q, 2q+1) of channel block b -> XOR mask on the bf16x2 word
  for (int i = tid; i < p.nb * 64; i += blockDim.x) {
    const int b = i >> 6, q = i & 63;
    const int8_t s0 = p.signs[b * 128 + 2 * q], s1 = p.signs[b * 128 + 2 * q + 1];
    s.smask[i] = (s0 < 0 ? 0x8000u : 0u) | (s1 < 0 ? 0x80000000u : 0u);
  }
  if (tid < 2 * p.R) s.row_amax[tid] = 0u;
  if (tid == 0) {
    for (int st = 0; st < p.stages; ++st) mbar_init(&s.full[st], 1);
    fence_mbar_init();
    const size_t sb = RotSmemLayout::stage_bytes(p.R, p.K);
    int64_t tile = blockIdx.x;
    for (int st = 0; st < p.stages && tile < p.num_tiles; ++st, tile += gridDim.x)
      issue_tile_load(p, tile, s.ring + st * sb, &s.full[st]);
  }
  __syncthreads();
}

// Wait for stage `st` with parity; thread 0 waits (bounded) and publishes.
__device__ __forceinline__ bool wait_stage(RotSmem& s, int st, unsigned parity) {
  if (threadIdx.x == 0) *s.flag = mbar_wait_bounded(&s.full[st], parity) ? 1 : 0;
  __syncthreads();
  return *s.flag != 0;
}

// After a timeout: wait (bounded) for the copies this CTA issued, then return.
__device__ __forceinline__ void drain_after_timeout(RotSmem& s, const RotParams& p, int64_t i_fail) {
  if (threadIdx.x != 0) return;
  // stages that may still have copies in flight: tiles i_fail .. i_fail+stages-1
  for (int k = 0; k < p.stages; ++k) {
    const int64_t i = i_fail + k;
    const int64_t tile = blockIdx.x + i * gridDim.x;
    if (tile >= p.num_tiles) break;
    (void)mbar_wait_bounded(&s.full[i % p.stages], (unsigned)((i / p.stages) & 1));
  }
}

// ---------------------------------------------------------------------------
// Block-diagonal (B = 128) rotation: every mode.
// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(384, 1) rotate_block_kernel(const RotParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RotSmem s = carve(smem_raw, p);
  prologue(p, s);

  const int tid = threadIdx.x;
  const int nb = p.nb;
  const int r = tid / nb;
  const int b = tid - r * nb;
  const int m = tid & 7;
  const float c = 0.08838834764831845f;  // 1/sqrt(128)
  const size_t sb = RotSmemLayout::stage_bytes(p.R, p.K);

  float g = 0.f, inv6g = 0.f;
  if (MODE == kModeNvfp4) {
    if (p.nvfp4_dynamic) {
      const float amax = __uint_as_float(*((volatile unsigned*)p.amax_word));
      g = __fdiv_rn(amax, 2688.0f);
    } else {
      g = *p.g_in;
    }
    inv6g = g > 0.f ? __frcp_rn(6.0f * g) : 0.0f;
    if (blockIdx.x == 0 && tid == 0 && p.g_out) *p.g_out = g;
  }
  float amax_acc = 0.f;

  int64_t i = 0;
  for (int64_t tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++i) {
    const int st = (int)(i % p.stages);
    if (!wait_stage(s, st, (unsigned)((i / p.stages) & 1))) {
      drain_after_timeout(s, p, i + 1);
      return;
    }
    const int64_t r0 = tile * p.R;
    const int nrows = (int)min((int64_t)p.R, p.rows - r0);
    const bool valid = r < nrows;
    unsigned* slot = s.row_amax + (i & 1) * p.R;
    if (MODE == kModeInt4 && tid < p.R) slot[tid] = 0u;

    float v[128];
    if (valid) {
      load_block(s.ring + st * sb + (size_t)r * p.K * 2 + (size_t)b * 256, s.smask + b * 64, m, v);
    }
    __syncthreads();  // stage consumed; row slots reset
    if (tid == 0) {
      const int64_t nt = tile + (int64_t)p.stages * gridDim.x;
      if (nt < p.num_tiles) {
        fence_proxy_async_smem();
        issue_tile_load(p, nt, s.ring + st * sb, &s.full[st]);
      }
    }
    if (valid) fwht128(v);
    const int64_t row = r0 + r;

    if (MODE == kModeInt4) {
      const float a = valid ? absmax128(v) * c : 0.f;
      const float amax_row = row_max(a, nb, tid, r, slot, valid);
      if (valid) {
        quant_int4_store(v, c, amax_row, m, p.codes + row * (p.K / 2) + (size_t)b * 64);
        if (b == 0) p.scales_f32[row] = __fdiv_rn(amax_row, 7.0f);
      }
    } else if (MODE == kModeNvfp4) {
      if (valid)
        quant_nvfp4_store(v, c, g, inv6g, m, p.codes + row * (p.K / 2) + (size_t)b * 64,
                          p.scales_e4m3 + row * (p.K / 16) + (size_t)b * 8);
    } else if (MODE == kModeF32) {
      if (valid) store_f32_block(v, c, m, p.out_f32 + row * p.ldo + (size_t)b * 128);
    } else if (MODE == kModeAmax) {
      if (valid) amax_acc = fmaxf(amax_acc, absmax128(v) * c);
    } else if (MODE == kModeKv4) {
      if (valid) quant_kv4_store(v, c, m, p.codes + row * 64, p.kv_scale + row, p.kv_zero + row);
    }
  }
  if (MODE == kModeAmax) {
    const unsigned bits = __reduce_max_sync(__activemask(), __float_as_uint(amax_acc));
    if ((tid & 31) == 0) atomicMax(p.amax_word, bits);
  }
}

// ---------------------------------------------------------------------------
// Full-width rotation, K = 128 * NB (NB = 2..32): INT4 and F32.
// ---------------------------------------------------------------------------
template <int MODE, int NB>
__global__ void __launch_bounds__(256, 1) rotate_full_kernel(const RotParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RotSmem s = carve(smem_raw, p);
  prologue(p, s);

  constexpr int COLS = 64 / NB;   // i-columns per thread per half
  const int tid = threadIdx.x;
  const int r = tid / NB;
  const int b = tid - r * NB;     // phase 1: block; phase 2: column group t'
  const int m = tid & 7;
  const float cfull = p.cfull;
  const size_t sb = RotSmemLayout::stage_bytes(p.R, p.K);

  int64_t i = 0;
  for (int64_t tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++i) {
    const int st = (int)(i % p.stages);
    if (!wait_stage(s, st, (unsigned)((i / p.stages) & 1))) {
      drain_after_timeout(s, p, i + 1);
      return;
    }
    const int64_t r0 = tile * p.R;
    const int nrows = (int)min((int64_t)p.R, p.rows - r0);
    const bool valid = r < nrows;
    unsigned* slot = s.row_amax + (i & 1) * p.R;
    if (MODE == kModeInt4 && tid < p.R) slot[tid] = 0u;
    uint8_t* stage = s.ring + st * sb;

    float v[128];
    if (valid) load_block(stage + (size_t)r * p.K * 2 + (size_t)b * 256, s.smask + b * 64, m, v);
    __syncthreads();  // stage consumed: reuse it as the transpose buffer
    if (valid) fwht128(v);

    // y[bb][col] for this thread's 2*COLS columns (half h: columns 64h + b*COLS + c)
    float y[2][NB][COLS];
    float* zrow = reinterpret_cast<float*>(stage) + (size_t)r * NB * 64;  // [NB][64] per row
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (valid) {
        // write half h of this block's outputs: 16 chunks of 4 floats, XOR-swizzled by the writer index
        float* zb = zrow + (size_t)b * 64;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float mul = with_sign(cfull, chi_signbit(8 * h + (q >> 1), m));
          const int k = 64 * h + 4 * q;
          *reinterpret_cast<float4*>(zb + 4 * (q ^ (tid & 7))) =
              make_float4(v[k] * mul, v[k + 1] * mul, v[k + 2] * mul, v[k + 3] * mul);
        }
      }
      __syncthreads();
      if (valid) {
#pragma unroll
        for (int bb = 0; bb < NB; ++bb) {
          const int wtid = r * NB + bb;  // writer thread of block bb
          const float* zb = zrow + (size_t)bb * 64;
#pragma unroll
          for (int pp = 0; pp < COLS / 2; ++pp) {
            const int P = b * (COLS / 2) + pp;  // float2 index within the half row
            const int q = P >> 1;
            const float2 t = *reinterpret_cast<const float2*>(zb + 4 * (q ^ (wtid & 7)) + 2 * (P & 1));
            y[h][bb][2 * pp] = t.x;
            y[h][bb][2 * pp + 1] = t.y;
          }
        }
      }
      __syncthreads();
      if (valid) {
        // NB-point transform across blocks, per column
#pragma unroll
        for (int hh = 1; hh < NB; hh <<= 1) {
#pragma unroll
          for (int bb = 0; bb < NB; ++bb) {
            if ((bb & hh) == 0) {
#pragma unroll
              for (int cc = 0; cc < COLS; cc += 2) {
                const float2 a = make_float2(y[h][bb][cc], y[h][bb][cc + 1]);
                const float2 d = make_float2(y[h][bb + hh][cc], y[h][bb + hh][cc + 1]);
                const float2 sum = __fadd2_rn(a, d);
                const float2 dif = __ffma2_rn(d, make_float2(-1.0f, -1.0f), a);
                y[h][bb][cc] = sum.x;
                y[h][bb][cc + 1] = sum.y;
                y[h][bb + hh][cc] = dif.x;
                y[h][bb + hh][cc + 1] = dif.y;
              }
            }
          }
        }
      }
    }
    if (tid == 0) {
      const int64_t nt = tile + (int64_t)p.stages * gridDim.x;
      if (nt < p.num_tiles) {
        fence_proxy_async_smem();
        issue_tile_load(p, nt, stage, &s.full[st]);
      }
    }
    const int64_t row = r0 + r;
    if (MODE == kModeInt4) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int bb = 0; bb < NB; ++bb)
#pragma unroll
          for (int cc = 0; cc < COLS; cc += 2) {
            a0 = fmaxf(a0, fabsf(y[h][bb][cc]));
            a1 = fmaxf(a1, fabsf(y[h][bb][cc + 1]));
          }
      const float amax_row = row_max(valid ? fmaxf(a0, a1) : 0.f, NB, tid, r, slot, valid);
      if (valid) {
        const float rr = amax_row > 0.f ? __fdiv_rn(7.0f, amax_row) : 0.0f;
        uint8_t* crow = p.codes + row * (p.K / 2);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int bb = 0; bb < NB; ++bb) {
            // COLS values -> COLS/2 bytes at byte offset bb*64 + 32h + b*COLS/2
            uint32_t byt[COLS / 2];
#pragma unroll
            for (int cc = 0; cc < COLS; cc += 2) {
              const float2 t = __ffma2_rn(make_float2(y[h][bb][cc], y[h][bb][cc + 1]), make_float2(rr, rr),
                                          make_float2(kRoundMagic, kRoundMagic));
              byt[cc / 2] = (__float_as_uint(t.x) & 0xFu) | ((__float_as_uint(t.y) & 0xFu) << 4);
            }
            uint8_t* dst = crow + bb * 64 + 32 * h + b * (COLS / 2);
            if (COLS / 2 == 1) {
              dst[0] = (uint8_t)byt[0];
            } else if (COLS / 2 == 2) {
              *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(byt[0] | (byt[1 % (COLS / 2)] << 8));
            } else {
#pragma unroll
              for (int w4 = 0; w4 < COLS / 8; ++w4) {
                const uint32_t word = byt[(4 * w4) % (COLS / 2)] | (byt[(4 * w4 + 1) % (COLS / 2)] << 8) |
                                      (byt[(4 * w4 + 2) % (COLS / 2)] << 16) | (byt[(4 * w4 + 3) % (COLS / 2)] << 24);
                reinterpret_cast<uint32_t*>(dst)[w4] = word;
              }
            }
          }
        if (b == 0) p.scales_f32[row] = __fdiv_rn(amax_row, 7.0f);
      }
    } else if (MODE == kModeF32) {
      if (valid) {
        float* orow = p.out_f32 + row * p.ldo;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int bb = 0; bb < NB; ++bb)
#pragma unroll
            for (int cc = 0; cc < COLS; cc += 2)
              *reinterpret_cast<float2*>(orow + bb * 128 + 64 * h + b * COLS + cc) =
                  make_float2(y[h][bb][cc], y[h][bb][cc + 1]);
      }
    }
    __syncthreads();  // row slots / stage reuse ordering before the next tile
  }
}

}  // namespace rq
