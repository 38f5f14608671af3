// Fused randomized-Hadamard rotation + 4-bit quantization + packing (sm_100a).
//
// What it computes ("Rotations for 4-Bit Activations: QuaRot, SpinQuant, and
// Friends", sections "A rotation changes nothing, and that is the point",
// "What it buys in 4 bits, and what it doesn't", "Gotchas"):
//   X~ = X . Q,  Q = blockdiag(diag(s_blk) . H_B / sqrt(B)),  B = 128 or B = K,
// then one of
//   INT4  : per-row symmetric, s = amax/7, q = rint(x/s)          (tokens / output channels)
//   NVFP4 : E2M1 codes, one E4M3 scale per 16 values, fp32 tensor scale g
//   MXFP4 : E2M1 codes, one E8M0 (power-of-two) scale per 32 values
//   KV4   : per-vector asymmetric, z = min, s = (max-min)/15 (fp16 scale and zero)
//   F32   : the rotated values themselves (parity checks)
//   AMAX  : only the global max |X~| (first pass of dynamic NVFP4)
// and packs two codes per byte, element 2i in the low nibble.
//
// Design (B200):
// * One thread owns one 128-wide block of one row and keeps it in 128
//   registers, so all seven butterfly stages of the 128-point fast
//   Walsh-Hadamard transform run in registers (no shuffles).
// * Work is organised in warp groups, not CTAs: a group is the G warps that
//   cover one row (G = 1 for K <= 4096, where a warp may hold 32/(K/128) rows;
//   G = K/4096 rounded up otherwise).  Each group owns a ring of shared-memory
//   stages filled by TMA bulk copies (cp.async.bulk, no tensor map, no
//   multicast) and guarded by its own mbarriers, so groups never wait on one
//   another; the only synchronisation is __syncwarp or a named barrier over
//   the group's warps.  Rows that are contiguous in HBM go in one copy.
// * Bank conflicts: thread u reads 16-byte chunk (j XOR m) into register slot j,
//   m = u mod 8, so the 8 threads of every shared-memory phase hit 8 different
//   bank groups.  Permuting the input by XOR with M = 8m multiplies the
//   Hadamard output k by chi(k) = (-1)^popcount(k & M) (H . P_M = diag(chi) . H),
//   so output k of the registers is chi(k) * y(k) in natural order; chi is
//   folded into the per-chunk multipliers of the quantizer (free).
// * The sign diagonal is applied to the packed bf16 pairs with one XOR per
//   pair, using a per-CTA table of sign masks in shared memory.
// * Full-width rotations (B = K = 128*NB, NB <= 32) use the Kronecker split
//   H_K = H_NB (x) H_128: after the in-register 128-point transform, each warp
//   transposes its rows' block outputs through its own consumed stage buffer
//   (XOR-swizzled, in two halves) and runs the NB-point transform across blocks
//   in registers again.
// * Rounding to integers uses the 1.5*2^23 "magic" add (the FPU's
//   round-to-nearest-even), whose low mantissa bits are the two's-complement
//   code; packing gathers low bytes with PRMT.
#pragma once

#include "rq_common.cuh"

namespace rq {

// Threads per CTA of the full-width variant (8 warps; 218 registers, no spills).
#ifndef RQ_FULL_WIDTH_THREADS
#define RQ_FULL_WIDTH_THREADS 256
#endif

enum RotMode : int {
  kModeInt4 = 0, kModeNvfp4 = 1, kModeF32 = 2, kModeAmax = 3, kModeKv4 = 4, kModeMxfp4 = 5,
  kModeInt8 = 6,  // 6- or 8-bit symmetric codes, one per byte (qmax 31 or 127)
  kModeAsym4 = 7  // asymmetric 4-bit per group of 128 along K: fp16 (scale, zero) per group
};

struct RotParams {
  const uint8_t* x;    // bf16 input (bytes)
  int64_t rows;        // total rows (vectors of K channels)
  int K;               // channels per row
  int nb;              // K / 128
  // row -> address: t = row % S, bh = row / S, h = bh % H, b = bh / H
  int64_t S, H;
  int64_t sB, sH, sS;  // byte strides
  int contiguous;      // 1: row r starts at x + r * K * 2
  const int8_t* signs; // [K]
  uint8_t* codes;      // [rows, K/2]
  float* scales_f32;   // INT4 / INT6 / INT8: [rows]
  float qmax;          // INT6 / INT8: 31 or 127
  uint8_t* scales_e4m3;// NVFP4: [rows, K/16]; MXFP4: E8M0 [rows, K/32]
  __half* kv_scale;    // KV4: [rows]; ASYM4: (scale, zero) pairs [rows, K/128]
  __half* kv_zero;     // KV4: [rows]
  float* out_f32;      // F32: [rows, ldo]
  int64_t ldo;
  const float* g_in;   // NVFP4 static: the per-tensor scale (device scalar)
  float* g_out;        // NVFP4: the per-tensor scale used (written by CTA 0)
  unsigned* amax_word; // NVFP4 dynamic: max |X~| as fp32 bits (AMAX writes, NVFP4 reads)
  int nvfp4_dynamic;   // 1: g from amax_word, 0: g from g_in
  float cfull;         // 1/sqrt(K) for full-width rotations (rounded once from the exact value)
  int logb;            // block-diagonal rotations: log2 of the block, 7 (128), 5 (32) or 4 (16)
  float cblk;          // 1/sqrt(2^logb), rounded once
  // geometry (host-chosen)
  int G;               // warps per group
  int RPS;             // rows per stage
  int GPC;             // groups per CTA
  int stages;          // ring depth per group
  int64_t num_tiles;   // ceil(rows / RPS)
};

struct RotSmemLayout {
  // [GPC][stages][RPS*K*2] rings | sign masks [nb*64] u32 | amax slots [GPC][G] u32 | mbarriers [GPC][stages]
  static __host__ __device__ size_t stage_bytes(int RPS, int K) { return (size_t)RPS * K * 2; }
  static __host__ __device__ size_t rings(int RPS, int K, int stages, int GPC) {
    return stage_bytes(RPS, K) * stages * GPC;
  }
  static __host__ __device__ size_t total(int RPS, int K, int stages, int GPC, int G) {
    size_t b = rings(RPS, K, stages, GPC);
    b += (size_t)(K / 128) * 64 * 4;
    b += (size_t)GPC * G * 4;
    b = (b + 7) & ~(size_t)7;
    b += (size_t)GPC * stages * 8;
    return b;
  }
};

// Issue the bulk copies of tile `tile` (RPS rows) into `dst` (one elected thread).
__device__ __forceinline__ void issue_tile_load(const RotParams& p, int64_t tile, uint8_t* dst, uint64_t* bar) {
  const int64_t r0 = tile * p.RPS;
  const int nrows = (int)min((int64_t)p.RPS, p.rows - r0);
  const unsigned row_bytes = (unsigned)p.K * 2u;
  mbar_arrive_expect_tx(bar, row_bytes * (unsigned)nrows);
  if (p.contiguous) {
    bulk_g2s(dst, p.x + r0 * (int64_t)row_bytes, row_bytes * (unsigned)nrows, bar);
    return;
  }
  // general strides: walk (b, h, t) incrementally from the first row
  int64_t t = r0 % p.S;
  int64_t bh = r0 / p.S;
  int64_t h = bh % p.H;
  int64_t b = bh / p.H;
  for (int r = 0; r < nrows; ++r) {
    bulk_g2s(dst + (size_t)r * row_bytes, p.x + b * p.sB + h * p.sH + t * p.sS, row_bytes, bar);
    if (++t == p.S) {
      t = 0;
      if (++h == p.H) {
        h = 0;
        ++b;
      }
    }
  }
}


// 16 int8 signs (+1 / -1) -> 8 XOR masks, one per bf16 pair (bit 15 / bit 31).
__device__ __forceinline__ void sign_masks16(const uint4 sg, uint32_t* dst) {
  const uint32_t w[4] = {sg.x, sg.y, sg.z, sg.w};
  uint32_t mk[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // byte k of w[j] is the sign of channel 4j + k; negative <=> bit 7 set
    const uint32_t neg = w[j] & 0x80808080u;
    mk[2 * j] = ((neg & 0x80u) << 8) | ((neg & 0x8000u) << 16);
    mk[2 * j + 1] = ((neg & 0x800000u) >> 8) | (neg & 0x80000000u);
  }
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(mk[0], mk[1], mk[2], mk[3]);
  d[1] = make_uint4(mk[4], mk[5], mk[6], mk[7]);
}

// Build the CTA's sign-mask table (nb*64 words) from the K signs.  The first
// (up to 2 per thread) sign loads are issued before `issue` runs -- the
// caller's first tile copies -- so they do not queue behind those copies; the
// conversion follows.
template <typename IssueFn>
__device__ __forceinline__ void build_sign_table(const int8_t* signs, int nb, uint32_t* smask, IssueFn issue) {
  const uint4* s4 = reinterpret_cast<const uint4*>(signs);
  const int n = nb * 8;
  uint4 sg[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int i = threadIdx.x + k * blockDim.x;
    if (i < n) sg[k] = __ldg(s4 + i);
  }
  issue();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int i = threadIdx.x + k * blockDim.x;
    if (i < n) sign_masks16(sg[k], smask + 8 * i);
  }
  for (int i = threadIdx.x + 2 * blockDim.x; i < n; i += blockDim.x) sign_masks16(__ldg(s4 + i), smask + 8 * i);
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

// The same transform over independent blocks of 2^logb consecutive values
// (logb = 4 or 5: the format-sized blocks of 16 / 32; 7 is fwht128).
template <int LOGB>
__device__ __forceinline__ void fwht_blocks(float (&v)[128]) {
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = a + b;
    v[i + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < (1 << LOGB); h <<= 1) {
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

// LOGB = 0 is the identity: blocks of one channel, Q = diag(s) (the
// unrotated arm, signs only).
template <int LOGB>
__device__ __forceinline__ void fwht_block_diag(float (&v)[128]) {
  if constexpr (LOGB == 7)
    fwht128(v);
  else if constexpr (LOGB > 0)
    fwht_blocks<LOGB>(v);
}

// A lane reads its block's 8-element chunks in the order j ^ m so that the
// lanes of a shared-memory phase hit distinct banks (m = lane mod 8 makes the
// reads conflict-free).  The bits of m inside one rotation block (chunk-index
// bits below log2(B/8)) turn into the output sign pattern chi of the
// transform; bits above it only swap whole blocks of 16 or 32 values, so
// register chunk j then holds output chunk j ^ mo with mo = those bits, and
// the stores put it there (kPermuted).  That is done for 16-wide blocks (a
// 4-way conflict otherwise); 32-wide blocks keep m inside the block (2-way
// conflicts), which measured faster than scattering their stores.
// With no rotation (LOGB = 0) a block is one channel: every bit of m lies
// above it, so the whole key permutes the stores, as for 16-wide blocks.
template <int LOGB>
struct ChunkOrder {
  static constexpr bool kPermuted = LOGB <= 4;
  static constexpr int T = LOGB >= 7 ? 15 : (LOGB <= 3 ? 0 : (1 << (LOGB - 3)) - 1);
};
struct ChunkKeys {
  int m;     // read order key
  int mchi;  // the part of m inside a block (sign pattern)
  int mo;    // the part of m above a block (output chunk permutation)
};
template <int LOGB>
__device__ __forceinline__ ChunkKeys chunk_keys(int lane) {
  constexpr int T = ChunkOrder<LOGB>::T;
  const int m = ChunkOrder<LOGB>::kPermuted ? (lane & 7) : (lane & T & 7);
  return ChunkKeys{m, m & T, m & ~T & 7};
}

// Store the four code words of chunks 4 j4 .. 4 j4 + 3 (4 bytes each) in place,
// or (PERM) each at chunk j ^ mo.
template <bool PERM>
__device__ __forceinline__ void store_words4(uint8_t* dst, int j4, int mo, uint32_t w0, uint32_t w1, uint32_t w2,
                                             uint32_t w3) {
  if (!PERM) {
    reinterpret_cast<uint4*>(dst)[j4] = make_uint4(w0, w1, w2, w3);
  } else {
    const uint32_t w[4] = {w0, w1, w2, w3};
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) *reinterpret_cast<uint32_t*>(dst + 4 * ((4 * j4 + jj) ^ mo)) = w[jj];
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

// INT4 per-row quantization of v (true value = v * c * chi) and packing.
// amax_true: the row's max |x~|.  Writes 64 bytes at dst.
template <bool PERM = false>
__device__ __forceinline__ void quant_int4_store(const float (&v)[128], float c, float amax_true, int m, int mo,
                                                 uint8_t* dst) {
  // r = 7/amax; zero rows -> r = 0 -> all codes 0
  const float r = amax_true > 0.f ? __fdiv_rn(7.0f, amax_true) : 0.0f;
  const float cr = c * r;
  uint4* out = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    uint32_t w[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {  // chunk j = 8 elements -> one word
      const int j = 4 * j4 + jj;
      const float mul = with_sign(cr, chi_signbit(j, m));
      float q[8];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float2 t = __ffma2_rn(make_float2(v[8 * j + e], v[8 * j + e + 1]), make_float2(mul, mul),
                                    make_float2(kRoundMagic, kRoundMagic));
        q[e] = t.x;
        q[e + 1] = t.y;
      }
      w[jj] = pack8_magic(q);
    }
    store_words4<PERM>(dst, j4, mo, w[0], w[1], w[2], w[3]);
  }
  (void)out;
}

// Per-row symmetric quantization without a rotation (blocks of one channel:
// v holds the sign-flipped inputs themselves, exact bf16 values), codes
// rint(x / s) with s = fp32(amax / qmax) the stored scale.  bf16 inputs often
// sit exactly on, or within fp32 rounding of, a midpoint k + 1/2 of x / s, where
// a product with the reciprocal may round either way; there the quotient is
// formed in fp64 (x / s exactly as the plain definition divides).  BITS = 4
// packs two codes per byte (64 bytes per 128 values), BITS = 8 stores one
// code per byte (128 bytes).
template <bool PERM, int BITS>
__device__ __forceinline__ void quant_int_exact_store(const float (&v)[128], float amax_true, float qmax, int mo,
                                                      uint8_t* dst) {
  const float s = __fdiv_rn(amax_true, qmax);
  const float r = amax_true > 0.f ? __fdiv_rn(qmax, amax_true) : 0.0f;
  const int qlo = -(int)qmax - 1, qhi = (int)qmax;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    int q[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = v[8 * j + e];
      const float t = x * r;
      int qi = __float2int_rn(t);
      const float d = fabsf(t - floorf(t) - 0.5f);
      if (d <= 0x1p-18f * fmaxf(1.0f, fabsf(t)) && s > 0.f) qi = __double2int_rn((double)x / (double)s);
      q[e] = min(max(qi, qlo), qhi);
    }
    const int d = PERM ? (j ^ mo) : j;
    if (BITS == 4) {
      uint32_t w = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) w |= ((uint32_t)q[e] & 0xFu) << (4 * e);
      *reinterpret_cast<uint32_t*>(dst + 4 * d) = w;
    } else {
      uint32_t w0 = 0, w1 = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w0 |= ((uint32_t)q[e] & 0xFFu) << (8 * e);
        w1 |= ((uint32_t)q[e + 4] & 0xFFu) << (8 * e);
      }
      *reinterpret_cast<uint2*>(dst + 8 * d) = make_uint2(w0, w1);
    }
  }
}

// The E2M1 code (sign in bit 3, magnitude code 0..7 for 0, .5, 1, 1.5, 2, 3,
// 4, 6) of an fp64 value, rounded to nearest with ties to the even code and
// saturating at 6; a value that rounds to magnitude 0 gives +0.  Each
// comparison is against a midpoint of the grid: ">" where the lower neighbour
// has the even code, ">=" where the upper one has.
__device__ __forceinline__ uint32_t e2m1_code_f64(double x) {
  const double a = fabs(x);
  const uint32_t m = (uint32_t)(a > 0.25) + (uint32_t)(a >= 0.75) + (uint32_t)(a > 1.25) + (uint32_t)(a >= 1.75) +
                     (uint32_t)(a > 2.5) + (uint32_t)(a >= 3.5) + (uint32_t)(a > 5.0);
  return (x < 0.0 && m != 0) ? (m | 8u) : m;
}

// True when the fp32 value t (a quotient x / (S g)) lies within a relative
// 2^-18 of an E2M1 rounding midpoint (0.25, 0.75, 1.25, 1.75 below 2; 2.5,
// 3.5 below 4; 5 below 6; the test also fires, harmlessly, at 7 and above).
__device__ __forceinline__ bool near_e2m1_midpoint(float t) {
  const float a = fabsf(t);
  const float u = a < 2.0f ? 2.0f * a : (a < 4.0f ? a : 0.5f * a);
  return fabsf(u - floorf(u) - 0.5f) <= 0x1p-18f * fmaxf(1.0f, u);
}

// 6- / 8-bit per-row quantization of v (true value = v * c * chi): codes
// rint(x * qmax / amax) in [-qmax, qmax], one two's-complement byte each.
// Writes 128 bytes at dst.
template <bool PERM = false>
__device__ __forceinline__ void quant_int8_store(const float (&v)[128], float c, float amax_true, float qmax, int m,
                                                 int mo, uint8_t* dst) {
  const float r = amax_true > 0.f ? __fdiv_rn(qmax, amax_true) : 0.0f;
  const float cr = c * r;
  uint4* out = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j2 = 0; j2 < 8; ++j2) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // chunk j = 8 elements -> two words
      const int j = 2 * j2 + h;
      const float mul = with_sign(cr, chi_signbit(j, m));
      uint32_t q[8];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float2 t = __ffma2_rn(make_float2(v[8 * j + e], v[8 * j + e + 1]), make_float2(mul, mul),
                                    make_float2(kRoundMagic, kRoundMagic));
        q[e] = __float_as_uint(t.x);
        q[e + 1] = __float_as_uint(t.y);
      }
      w[2 * h] = gather_low_bytes(q[0], q[1], q[2], q[3]);
      w[2 * h + 1] = gather_low_bytes(q[4], q[5], q[6], q[7]);
    }
    if (!PERM) {
      out[j2] = make_uint4(w[0], w[1], w[2], w[3]);
    } else {  // chunk j (8 bytes) at chunk j ^ mo
      *reinterpret_cast<uint2*>(dst + 8 * ((2 * j2) ^ mo)) = make_uint2(w[0], w[1]);
      *reinterpret_cast<uint2*>(dst + 8 * ((2 * j2 + 1) ^ mo)) = make_uint2(w[2], w[3]);
    }
  }
}

// NVFP4 quantization of v (true value = v * c * chi): 8 groups of 16.
// Writes 64 bytes of codes and 8 bytes of E4M3 scales.  EXACT (the unrotated
// arm, v = the sign-flipped bf16 inputs, c = 1, chi = +1): a code whose fp32
// quotient lies near an E2M1 midpoint is decided again from the fp64 quotient
// x / (S g), the plain definition (bf16 inputs hit such midpoints often).
template <bool PERM = false, bool EXACT = false>
__device__ __forceinline__ void quant_nvfp4_store(const float (&v)[128], float c, float g, float inv6g, int m,
                                                  int mo, uint8_t* dst_codes, uint8_t* dst_scales) {
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
      if (EXACT && denom > 0.f) {
        const double dd = (double)sdec * (double)g;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (near_e2m1_midpoint(s[e] * mul)) {
            const uint32_t code = e2m1_code_f64((double)s[e] / dd);
            words[j] = (words[j] & ~(0xFu << (4 * e))) | (code << (4 * e));
          }
      }
    }
    if (PERM) {
      dst_scales[gi ^ (mo >> 1)] = (uint8_t)scode;  // group gi = chunks 2 gi, 2 gi + 1
    } else if (gi < 4) {
      sc_lo |= scode << (8 * gi);
    } else {
      sc_hi |= scode << (8 * (gi - 4));
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
    store_words4<PERM>(dst_codes, j, mo, words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
  if (!PERM) *reinterpret_cast<uint2*>(dst_scales) = make_uint2(sc_lo, sc_hi);
}

// MXFP4 quantization of v (true value = v * c * chi): 4 groups of 32 with an
// E8M0 scale 2^e each, e = floor(log2(amax)) - 2 clamped to [-127, 127].
// floor(log2(amax)) is the exponent field of the fp32 amax (a zero or
// subnormal amax gives -127 - 2 and clamps to -127).  x / 2^e is exact, so the
// only rounding left is the E2M1 conversion.  Writes 64 bytes of codes and 4
// bytes of scales.
template <bool PERM = false>
__device__ __forceinline__ void quant_mxfp4_store(const float (&v)[128], float c, int m, int mo, uint8_t* dst_codes,
                                                  uint8_t* dst_scales) {
  uint32_t words[16];
  uint32_t sc = 0;
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      a0 = fmaxf(a0, fabsf(v[32 * gi + e]));
      a1 = fmaxf(a1, fabsf(v[32 * gi + e + 1]));
    }
    const float amax_b = fmaxf(a0, a1) * c;  // true block max
    int ex = (int)((__float_as_uint(amax_b) >> 23) & 0xFFu) - 127 - 2;
    ex = min(max(ex, -127), 127);
    if (PERM)
      dst_scales[gi ^ (mo >> 2)] = (uint8_t)(ex + 127);  // group gi = chunks 4 gi .. 4 gi + 3
    else
      sc |= (uint32_t)(ex + 127) << (8 * gi);
    // 2^-ex: a normal fp32 for ex <= 126; 2^-127 is the subnormal 0x00400000
    const float inv = ex == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - ex) << 23);
    const float ci = c * inv;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int j = 4 * gi + q4;
      const float mul = with_sign(ci, chi_signbit(j, m));
      const float* s = &v[8 * j];
      words[j] = pack8_e2m1(s[0] * mul, s[1] * mul, s[2] * mul, s[3] * mul, s[4] * mul, s[5] * mul, s[6] * mul,
                            s[7] * mul);
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
    store_words4<PERM>(dst_codes, j, mo, words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
  if (!PERM) *reinterpret_cast<uint32_t*>(dst_scales) = sc;
}

// Global address of row `row`'s first input element.
__device__ __forceinline__ const uint8_t* row_src(const RotParams& p, int64_t row) {
  if (p.contiguous) return p.x + row * (int64_t)p.K * 2;
  const int64_t t = row % p.S, bh = row / p.S;
  return p.x + (bh / p.H) * p.sB + (bh % p.H) * p.sH + t * p.sS;
}

// True when v may lie within 2^-LOG2BAND of `am` (am >= |v| > 0 in practice)
// of a midpoint between two neighbouring fp16 values, so that an error of that
// size could change its fp16 rounding.  Integer arithmetic on the fp32 bits:
// in the fp16 normal range a midpoint is where the 13 fraction bits fp16 drops
// read 0x1000, and 2^-LOG2BAND am is at most 2^(23 - LOG2BAND + 1 + ea - ev)
// units in the last place of v (ea, ev the exponent fields).  Values outside
// the fp16 normal range are reported as near (the caller then decides exactly).
template <int LOG2BAND>
__device__ __forceinline__ bool near_fp16_midpoint(float v, float am) {
  const uint32_t b = __float_as_uint(v) & 0x7FFFFFFFu;
  const int ev = (int)(b >> 23), ea = (int)((__float_as_uint(am) >> 23) & 0xFFu);
  if (ev < 127 - 14 || ev > 127 + 15) return true;
  const int d = (int)(b & 0x1FFFu) - 0x1000;
  const int span = ea - ev;  // >= 0 when am >= |v|
  return span > 10 || (d < 0 ? -d : d) <= ((1 << (24 - LOG2BAND)) << (span > 0 ? span : 0));
}

// 1 / sqrt(2^LOGB) in fp64 (LOGB = 0, 4, 5, 7).
template <int LOGB>
__device__ __forceinline__ double inv_sqrt_block_f64() {
  if constexpr (LOGB == 0) return 1.0;
  else if constexpr (LOGB == 4) return 0.25;
  else if constexpr (LOGB == 5) return 0.125 * 1.4142135623730951;   // 2^-2.5 = 2^-3 sqrt(2)
  else return 0.0625 * 1.4142135623730951;                            // 2^-3.5 = 2^-4 sqrt(2)
}

// One group of 128 channels rotated in fp64 by the whole warp: lane l takes
// channels 4l .. 4l+3 of the group's bf16 inputs at `src` (the tile's
// shared-memory stage) and of its sign masks, and the fast Walsh-Hadamard butterflies of the
// 2^LOGB-wide blocks run in fp64 (the first two stages within a lane, the
// others across lanes), scaled by 1/sqrt(2^LOGB).  On return y[e] is rotated
// channel 4 lane + e, and lo / hi are the group's min / max (the same in every
// lane).  The sum of a block's +-x is exact in fp64 for inputs whose
// magnitudes span less than 2^45, so y is the true rotation to within one
// fp64 rounding.
template <int LOGB>
__device__ __forceinline__ void rotated_group_f64(const uint8_t* src, const uint32_t* smask_grp, int lane,
                                                  double (&v)[4], double& lo, double& hi) {
  const uint2 raw = *(reinterpret_cast<const uint2*>(src) + lane);
  const uint2 mk = *reinterpret_cast<const uint2*>(smask_grp + 2 * lane);
  const uint32_t a = raw.x ^ mk.x, b = raw.y ^ mk.y;
  v[0] = (double)__uint_as_float(a << 16);
  v[1] = (double)__uint_as_float(a & 0xFFFF0000u);
  v[2] = (double)__uint_as_float(b << 16);
  v[3] = (double)__uint_as_float(b & 0xFFFF0000u);
  if constexpr (LOGB >= 1) {  // h = 1
    const double t0 = v[0], t2 = v[2];
    v[0] = t0 + v[1];
    v[1] = t0 - v[1];
    v[2] = t2 + v[3];
    v[3] = t2 - v[3];
  }
  if constexpr (LOGB >= 2) {  // h = 2
    const double t0 = v[0], t1 = v[1];
    v[0] = t0 + v[2];
    v[2] = t0 - v[2];
    v[1] = t1 + v[3];
    v[3] = t1 - v[3];
  }
#pragma unroll
  for (int j = 0; j + 2 < LOGB; ++j) {  // h = 4 * 2^j: the partner is lane ^ 2^j
    const bool upper = (lane >> j) & 1;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double o = __shfl_xor_sync(0xFFFFFFFFu, v[e], 1 << j);
      v[e] = upper ? o - v[e] : v[e] + o;
    }
  }
  const double c = inv_sqrt_block_f64<LOGB>();
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] *= c;
  double mn = fmin(fmin(v[0], v[1]), fmin(v[2], v[3]));
  double mx = fmax(fmax(v[0], v[1]), fmax(v[2], v[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fmin(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
    mx = fmax(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  }
  lo = mn;
  hi = mx;
}

// Where one group of 128 channels lives: its bf16 inputs (the shared-memory
// stage), its sign masks (shared) and its stored codes, scale and zero (global).
struct KvGroup {
  const uint8_t* src;
  const uint32_t* smask;
  uint8_t* codes;
  __half* scale;
  __half* zero;
};

// The second look of quant_kv4_store: for each lane L in `pending` the warp
// rotates L's group in fp64 (rotated_group_f64) and, where the fp16 roundings
// of the exact min and (max - min)/15 differ from the ones lane L stored for
// that group (`szb`: its fp16 scale bits << 16 | zero bits, taken from lane L
// by a shuffle), rewrites its scale, zero and codes from the fp64 values.
// Called by every lane of the warp; group_of(L) gives lane L's group and is
// evaluated (by the whole warp) only for the pending lanes, so none of its
// address arithmetic runs in the common case.  Nothing here reads global
// memory: a look costs its arithmetic, not a round trip.
template <int LOGB, typename GroupFn>
__device__ __forceinline__ void kv4_second_look(unsigned pending, uint32_t szb, GroupFn group_of) {
  const int lane = threadIdx.x & 31;
  __syncwarp();  // this warp's stores of its groups come before any rewrite below
  while (pending) {
    const int L = __ffs(pending) - 1;
    pending &= pending - 1;
    const KvGroup gr = group_of(L);
    const uint32_t szbits = __shfl_sync(0xFFFFFFFFu, szb, L);
    double y[4], dlo, dhi;
    rotated_group_f64<LOGB>(gr.src, gr.smask, lane, y, dlo, dhi);
    const __half zx = __double2half(dlo);
    const __half sx = __double2half((dhi - dlo) / 15.0);
    const uint32_t xbits = ((uint32_t)__half_as_ushort(sx) << 16) | __half_as_ushort(zx);
    if (xbits != szbits) {  // the same in every lane
      const double sd = (double)__half2float(sx), zd = (double)__half2float(zx);
      uint32_t nib = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int q = 0;
        if (sd > 0.0) q = min(max(__double2int_rn((y[e] - zd) / sd), 0), 15);
        nib |= (uint32_t)q << (4 * e);
      }
      *reinterpret_cast<uint16_t*>(gr.codes + 2 * lane) = (uint16_t)nib;  // channels 4 lane .. 4 lane + 3
      if (lane == 0) {
        *gr.scale = sx;
        *gr.zero = zx;
      }
    }
  }
}

// kv4_second_look out of line, for the rotate kernel: lane L's group follows
// the kernel's thread mapping (rows of RPS per stage starting at r0; a group
// is the lane's 128-wide block, or the vector itself for KV4).  Kept out of
// line so that its code -- rarely run -- does not crowd the instruction cache
// of the unrolled main loop.
template <int LOGB, bool KV>
__device__ __noinline__ void kv4_second_look_rows(unsigned pending, uint32_t szb, const RotParams p, int64_t r0,
                                                  int wig, int RPS, const uint32_t* smask, const uint8_t* stage) {
  const int nb = p.nb;
  kv4_second_look<LOGB>(pending, szb, [&](int L) {
    // KV4: one head vector per lane (K = 128, 32 rows per stage)
    const int rL = KV ? L : (RPS > 1 ? L / nb : 0);
    const int bL = KV ? 0 : (RPS > 1 ? L - rL * nb : wig * 32 + L);
    const int64_t rowL = r0 + rL;
    KvGroup gr;
    gr.src = stage + (size_t)rL * p.K * 2 + (size_t)bL * 256;
    gr.smask = smask + bL * 64;
    if (KV) {
      gr.codes = p.codes + rowL * 64;
      gr.scale = p.kv_scale + rowL;
      gr.zero = p.kv_zero + rowL;
    } else {
      gr.codes = p.codes + rowL * (p.K / 2) + (size_t)bL * 64;
      gr.scale = p.kv_scale + 2 * (rowL * nb + bL);
      gr.zero = gr.scale + 1;
    }
    return gr;
  });
}

// KV4 and per-group asymmetric INT4: asymmetric quantization of one group of
// 128 channels (true value = v * c * chi): z = min, s = (max - min)/15, both
// stored as fp16, q = clamp(rint((x - z)/s), 0, 15).
//
// The fp32 butterflies leave the group's min within about 2^-23 of its
// largest magnitude and (max - min)/15 within about 2^-25 (the largest errors
// seen over 6e5 Gaussian and outlier groups; the bound of a 7-level summation
// is a few times that), which can decide the fp16 rounding of z or s when
// either lies that close to a midpoint between two fp16 values.  So after
// the group is stored, the lanes for which that is possible (a band of at
// least 2^-22 of the largest magnitude around z, 2^-24 around s, found from
// the fp32 bits alone: about 0.3 % of groups) have their
// group rotated again in fp64 by the whole warp (rotated_group_f64); where the
// fp16 roundings of the exact min and scale differ from the stored ones (about
// 2 groups in 10^4), the warp rewrites the group's z, s and codes from the
// fp64 values (kv4_second_look).  This function stores the group (only where
// `valid`), sets `szb` to the stored bits (scale << 16 | zero) and returns
// whether this lane's group needs the second look; the caller then runs
// kv4_second_look with the whole warp, from the tile's shared-memory stage.
template <bool PERM>
__device__ __forceinline__ bool quant_kv4_store(const float (&v)[128], float c, int m, int mo, bool valid,
                                                uint8_t* dst_codes, __half* dst_scale, __half* dst_zero,
                                                uint32_t& szb) {
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
  // whether z or s lies near an fp16 midpoint (the second look, after the stores)
  const float am = fmaxf(fabsf(lo), fabsf(hi));
  const bool unsure = valid && (near_fp16_midpoint<22>(lo, am) || near_fp16_midpoint<24>(s, am));
  szb = ((uint32_t)__half_as_ushort(s_h) << 16) | __half_as_ushort(z_h);
  if (valid) {
    *dst_scale = s_h;
    *dst_zero = z_h;
  }
#pragma unroll
  for (int j4 = 0; j4 < 4; ++j4) {
    uint32_t w[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * j4 + jj;
      const float mul = with_sign(ci, chi_signbit(j, m));
      float q[8];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        float2 t = __ffma2_rn(make_float2(v[8 * j + e], v[8 * j + e + 1]), make_float2(mul, mul),
                              make_float2(off, off));
        if (need_clamp) {
          t.x = fminf(fmaxf(t.x, 0.0f), 15.0f);
          t.y = fminf(fmaxf(t.y, 0.0f), 15.0f);
        }
        t = __fadd2_rn(t, make_float2(kRoundMagic, kRoundMagic));
        q[e] = t.x;
        q[e + 1] = t.y;
      }
      w[jj] = pack8_magic(q);
    }
    if (valid) store_words4<PERM>(dst_codes, j4, mo, w[0], w[1], w[2], w[3]);
  }
  return unsure;
}

template <bool PERM = false>
__device__ __forceinline__ void store_f32_block(const float (&v)[128], float c, int m, int mo, float* dst) {
  float4* out = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float mul = with_sign(c, chi_signbit(j, m));
    const int d = PERM ? (j ^ mo) : j;
    out[2 * d] = make_float4(v[8 * j] * mul, v[8 * j + 1] * mul, v[8 * j + 2] * mul, v[8 * j + 3] * mul);
    out[2 * d + 1] = make_float4(v[8 * j + 4] * mul, v[8 * j + 5] * mul, v[8 * j + 6] * mul, v[8 * j + 7] * mul);
  }
}


// Synchronise the G warps of a group (named barrier 1 + group index).
__device__ __forceinline__ void group_sync(int G, int grp) {
  if (G == 1) {
    __syncwarp();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(32 * G) : "memory");
  }
}

// Group-wide AND of a predicate (all threads of the group get the result).
__device__ __forceinline__ bool group_all(bool v, int G, int grp) {
  if (G == 1) return __all_sync(0xFFFFFFFFu, v);
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(1 + grp), "r"(32 * G)
      : "memory");
  return out != 0;
}

// Max of a non-negative float over the threads of one row; every thread of
// the row gets it.  Rows are `seg` consecutive lanes when RPS > 1 (seg = nb, a
// power of two below 32), a whole warp when G == 1, or the group's G warps.
__device__ __forceinline__ float row_max(float a, int RPS, int nb, int G, int grp, int wig, unsigned* slots) {
  uint32_t bits = __float_as_uint(a);
  if (RPS > 1) {
    for (int o = 1; o < nb; o <<= 1) bits = max(bits, __shfl_xor_sync(0xFFFFFFFFu, bits, o));
    return __uint_as_float(bits);
  }
  bits = __reduce_max_sync(0xFFFFFFFFu, bits);
  if (G == 1) return __uint_as_float(bits);
  if ((threadIdx.x & 31) == 0) slots[grp * G + wig] = bits;
  group_sync(G, grp);
  uint32_t m = 0;
  for (int w = 0; w < G; ++w) m = max(m, ((volatile unsigned*)slots)[grp * G + w]);
  return __uint_as_float(m);
}

// Full-width second phase for one half (h) of every block's outputs: the rows'
// outputs are transposed through `zbuf` (this warp's consumed stage) and the
// NB-point transform runs across blocks.  Thread (r, b): on entry v holds
// chi-signed block outputs of block b of row r; on exit y[bb][c] holds
// y(bb*128 + 64h + b*COLS + c) for all NB blocks bb.
template <int NB>
__device__ __forceinline__ void full_phase2(const float (&v)[128], float (&y)[NB][64 / NB], int h, float* zbuf,
                                            int r, int b, int lane, int m, float cfull, bool valid) {
  constexpr int COLS = 64 / NB;
  float* zrow = zbuf + (size_t)r * NB * 64;
  {
    float* zb = zrow + (size_t)b * 64;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float mul = with_sign(cfull, chi_signbit(8 * h + (q >> 1), m));
      const int k = 64 * h + 4 * q;
      *reinterpret_cast<float4*>(zb + 4 * (q ^ (lane & 7))) =
          make_float4(v[k] * mul, v[k + 1] * mul, v[k + 2] * mul, v[k + 3] * mul);
    }
  }
  __syncwarp();
  {
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
      const int wl = (NB >= 8) ? (bb & 7) : ((r * NB + bb) & 7);  // XOR key of the lane that wrote block bb
      const float* zb = zrow + (size_t)bb * 64;
#pragma unroll
      for (int pp = 0; pp < COLS / 2; ++pp) {
        const int P = b * (COLS / 2) + pp;
        const float2 t = *reinterpret_cast<const float2*>(zb + 4 * ((P >> 1) ^ wl) + 2 * (P & 1));
        y[bb][2 * pp] = t.x;
        y[bb][2 * pp + 1] = t.y;
      }
    }
  }
  __syncwarp();
  {
#pragma unroll
    for (int hh = 1; hh < NB; hh <<= 1) {
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        if ((bb & hh) == 0) {
#pragma unroll
          for (int cc = 0; cc < COLS; cc += 2) {
            const float2 a = make_float2(y[bb][cc], y[bb][cc + 1]);
            const float2 d = make_float2(y[bb + hh][cc], y[bb + hh][cc + 1]);
            const float2 s = __fadd2_rn(a, d);
            const float2 e = __ffma2_rn(d, make_float2(-1.0f, -1.0f), a);
            y[bb][cc] = s.x;
            y[bb][cc + 1] = s.y;
            y[bb + hh][cc] = e.x;
            y[bb + hh][cc + 1] = e.y;
          }
        }
      }
    }
  }
}

// INT4 quantize + store of the full-width layout: COLS values per (block, half).
template <int NB>
__device__ __forceinline__ void full_store_int4(const float (&y)[2][NB][64 / NB], float rr, uint8_t* crow, int b) {
  constexpr int COLS = 64 / NB;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
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
        for (int w4 = 0; w4 < COLS / 8; ++w4)
          reinterpret_cast<uint32_t*>(dst)[w4] =
              byt[(4 * w4) % (COLS / 2)] | (byt[(4 * w4 + 1) % (COLS / 2)] << 8) |
              (byt[(4 * w4 + 2) % (COLS / 2)] << 16) | (byt[(4 * w4 + 3) % (COLS / 2)] << 24);
      }
    }
}

// 6- / 8-bit quantize + store of the full-width layout: COLS bytes per (block, half).
template <int NB>
__device__ __forceinline__ void full_store_int8(const float (&y)[2][NB][64 / NB], float rr, uint8_t* crow, int b) {
  constexpr int COLS = 64 / NB;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
      uint32_t q[COLS];
#pragma unroll
      for (int cc = 0; cc < COLS; cc += 2) {
        const float2 t = __ffma2_rn(make_float2(y[h][bb][cc], y[h][bb][cc + 1]), make_float2(rr, rr),
                                    make_float2(kRoundMagic, kRoundMagic));
        q[cc] = __float_as_uint(t.x);
        q[cc + 1] = __float_as_uint(t.y);
      }
      uint8_t* dst = crow + bb * 128 + 64 * h + b * COLS;
      if (COLS == 2) {
        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)((q[0] & 0xFFu) | ((q[1 % COLS] & 0xFFu) << 8));
      } else {
        uint32_t wd[COLS / 4 > 0 ? COLS / 4 : 1];
#pragma unroll
        for (int w4 = 0; w4 < COLS / 4; ++w4)
          wd[w4] = gather_low_bytes(q[(4 * w4) % COLS], q[(4 * w4 + 1) % COLS], q[(4 * w4 + 2) % COLS],
                                    q[(4 * w4 + 3) % COLS]);
        if (COLS == 4) {
          *reinterpret_cast<uint32_t*>(dst) = wd[0];
        } else if (COLS == 8) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1 % (COLS / 4)]);
        } else {
#pragma unroll
          for (int u = 0; u < COLS / 16; ++u)
            reinterpret_cast<uint4*>(dst)[u] = make_uint4(wd[(4 * u) % (COLS / 4)], wd[(4 * u + 1) % (COLS / 4)],
                                                          wd[(4 * u + 2) % (COLS / 4)], wd[(4 * u + 3) % (COLS / 4)]);
        }
      }
    }
}

// ---------------------------------------------------------------------------
// The kernel.  NBF = 0: block-diagonal with blocks of 2^LOGB (128, 32 or 16),
// any mode.  NBF = 2..32: full-width rotation of K = 128*NBF (INT4, INT6/INT8
// and F32 modes).
// ---------------------------------------------------------------------------
template <int MODE, int NBF, int LOGB = 7>
__global__ void __launch_bounds__(NBF ? RQ_FULL_WIDTH_THREADS : 384, 1) rotate_kernel(const RotParams p) {
  griddep_wait();
  griddep_trigger();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G, RPS = p.RPS, nb = p.nb;
  const int grp = warp / G, wig = warp - grp * G;
  const size_t sbytes = RotSmemLayout::stage_bytes(RPS, p.K);
  uint8_t* ring = smem_raw + (size_t)grp * p.stages * sbytes;
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem_raw + RotSmemLayout::rings(RPS, p.K, p.stages, p.GPC));
  unsigned* slots = reinterpret_cast<unsigned*>(smask + nb * 64);
  uint64_t* bars_all = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(slots + p.GPC * G) + 7) & ~(uintptr_t)7);
  uint64_t* full = bars_all + grp * p.stages;

  // thread -> (row in stage, block)
  int r, b;
  bool active;
  if (RPS > 1) {
    r = lane / nb;
    b = lane - r * nb;
    active = r < RPS;
  } else {
    r = 0;
    b = wig * 32 + lane;
    active = b < nb;
  }
  constexpr bool PERM = NBF == 0 && ChunkOrder<LOGB>::kPermuted;
  const ChunkKeys ck = chunk_keys<NBF ? 7 : LOGB>(lane);
  const int m = ck.m, mchi = ck.mchi, mo = ck.mo;
  const bool producer = (wig == 0 && lane == 0);
  // 1/sqrt(block), rounded once; 1 without a rotation
  const float c = (NBF || LOGB == 7) ? 0.08838834764831845f : (LOGB == 0 ? 1.0f : p.cblk);
  // each CTA a contiguous run of num_tiles / grid tiles (rounded down or up),
  // dealt to its groups in turn, so that no SM gets a whole round more than
  // another (tiles dealt grid-wide in turn left some SMs a whole round more)
  const int64_t t_end = ((int64_t)blockIdx.x + 1) * p.num_tiles / gridDim.x;
  const int64_t TG = p.GPC;
  const int64_t gg = (int64_t)blockIdx.x * p.num_tiles / gridDim.x + grp;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.GPC * p.stages; ++i) mbar_init(&bars_all[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  build_sign_table(p.signs, nb, smask, [&]() {
    if (producer) {  // the first tile copies of this group
      int64_t tile = gg;
      for (int st = 0; st < p.stages && tile < t_end; ++st, tile += TG)
        issue_tile_load(p, tile, ring + st * sbytes, &full[st]);
    }
  });
  __syncthreads();

  float g = 0.f, inv6g = 0.f;
  if (MODE == kModeNvfp4) {
    g = p.nvfp4_dynamic ? __fdiv_rn(__uint_as_float(*((volatile unsigned*)p.amax_word)), 2688.0f) : *p.g_in;
    inv6g = g > 0.f ? __frcp_rn(6.0f * g) : 0.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0 && p.g_out) *p.g_out = g;
  }
  float amax_acc = 0.f;

  int64_t i = 0;
  for (int64_t tile = gg; tile < t_end; tile += TG, ++i) {
    const int st = (int)(i % p.stages);
    const bool ok = group_all(mbar_wait_bounded(&full[st], (unsigned)((i / p.stages) & 1)), G, grp);
    if (!ok) {
      if (producer) {  // let the copies this group issued land before leaving
        for (int k = 1; k < p.stages; ++k) {
          const int64_t i2 = i + k;
          if (gg + i2 * TG >= t_end) break;
          (void)mbar_wait_bounded(&full[i2 % p.stages], (unsigned)((i2 / p.stages) & 1));
        }
      }
      return;
    }
    const int64_t r0 = tile * RPS;
    const int nrows = (int)min((int64_t)RPS, p.rows - r0);
    const bool valid = active && r < nrows;
    uint8_t* stage = ring + st * sbytes;
    const int64_t row = r0 + r;

    float v[128];
    // every thread loads and transforms (no predication of the 128-register block);
    // threads without a row read an in-bounds block and store nothing
    const int bl = active ? b : 0;
    load_block(stage + (size_t)(active ? r : 0) * p.K * 2 + (size_t)bl * 256, smask + bl * 64, m, v);

    if (NBF == 0) {
      // stage consumed: refill it while this tile is computed.  KV4 and
      // per-group asymmetric INT4 keep it until after the tile's second look,
      // which reads its inputs from there.
      constexpr bool kKeepStage = MODE == kModeKv4 || MODE == kModeAsym4;
      const auto refill = [&]() {
        group_sync(G, grp);
        if (producer) {
          const int64_t nt = tile + (int64_t)p.stages * TG;
          if (nt < t_end) {
            fence_proxy_async_smem();
            issue_tile_load(p, nt, stage, &full[st]);
          }
        }
      };
      if (!kKeepStage) refill();
      fwht_block_diag<LOGB>(v);
      if (MODE == kModeInt4) {
        const float a = valid ? absmax128(v) * c : 0.f;
        const float amax_row = row_max(a, RPS, nb, G, grp, wig, slots);
        if (valid) {
          if constexpr (LOGB == 0)
            quant_int_exact_store<PERM, 4>(v, amax_row, 7.0f, mo, p.codes + row * (p.K / 2) + (size_t)b * 64);
          else
            quant_int4_store<PERM>(v, c, amax_row, mchi, mo, p.codes + row * (p.K / 2) + (size_t)b * 64);
          if (b == 0) p.scales_f32[row] = __fdiv_rn(amax_row, 7.0f);
        }
      } else if (MODE == kModeInt8) {
        const float a = valid ? absmax128(v) * c : 0.f;
        const float amax_row = row_max(a, RPS, nb, G, grp, wig, slots);
        if (valid) {
          if constexpr (LOGB == 0)
            quant_int_exact_store<PERM, 8>(v, amax_row, p.qmax, mo, p.codes + row * p.K + (size_t)b * 128);
          else
            quant_int8_store<PERM>(v, c, amax_row, p.qmax, mchi, mo, p.codes + row * p.K + (size_t)b * 128);
          if (b == 0) p.scales_f32[row] = __fdiv_rn(amax_row, p.qmax);
        }
      } else if (MODE == kModeNvfp4) {
        if (valid)
          quant_nvfp4_store<PERM, LOGB == 0>(v, c, g, inv6g, mchi, mo, p.codes + row * (p.K / 2) + (size_t)b * 64,
                                             p.scales_e4m3 + row * (p.K / 16) + (size_t)b * 8);
      } else if (MODE == kModeMxfp4) {
        if (valid)
          quant_mxfp4_store<PERM>(v, c, mchi, mo, p.codes + row * (p.K / 2) + (size_t)b * 64,
                                  p.scales_e4m3 + row * (p.K / 32) + (size_t)b * 4);
      } else if (MODE == kModeF32) {
        if (valid) store_f32_block<PERM>(v, c, mchi, mo, p.out_f32 + row * p.ldo + (size_t)b * 128);
      } else if (MODE == kModeAmax) {
        if (valid) amax_acc = fmaxf(amax_acc, absmax128(v) * c);
      } else if (MODE == kModeKv4 || MODE == kModeAsym4) {
        constexpr bool KV = MODE == kModeKv4;
        __half* sz = KV ? p.kv_scale + row : p.kv_scale + 2 * (row * nb + b);
        uint32_t szb;
        const bool unsure =
            KV ? quant_kv4_store<false>(v, c, m, 0, valid, p.codes + row * 64, sz, p.kv_zero + row, szb)
               : quant_kv4_store<PERM>(v, c, mchi, mo, valid, p.codes + row * (p.K / 2) + (size_t)b * 64, sz, sz + 1,
                                       szb);
        const unsigned pending = __ballot_sync(0xFFFFFFFFu, unsure);
        if (pending) kv4_second_look_rows<KV ? 7 : LOGB, KV>(pending, szb, p, r0, wig, RPS, smask, stage);
        refill();
      }
    } else {
      constexpr int NB = NBF ? NBF : 1;
      constexpr int COLS = 64 / NB;
      float y[2][NB][COLS];
      fwht128(v);
      __syncwarp();  // every lane has read the stage: reuse it as the transpose buffer
      float* zbuf = reinterpret_cast<float*>(stage);
      full_phase2<NB>(v, y[0], 0, zbuf, r, b, lane, m, p.cfull, valid);
      full_phase2<NB>(v, y[1], 1, zbuf, r, b, lane, m, p.cfull, valid);
      if (producer) {
        const int64_t nt = tile + (int64_t)p.stages * TG;
        if (nt < t_end) {
          fence_proxy_async_smem();
          issue_tile_load(p, nt, stage, &full[st]);
        }
      }
      if (MODE == kModeInt4 || MODE == kModeInt8) {
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
        const float amax_row = row_max(valid ? fmaxf(a0, a1) : 0.f, RPS, nb, 1, grp, 0, slots);
        if (valid && MODE == kModeInt4) {
          const float rr = amax_row > 0.f ? __fdiv_rn(7.0f, amax_row) : 0.0f;
          full_store_int4<NB>(y, rr, p.codes + row * (p.K / 2), b);
          if (b == 0) p.scales_f32[row] = __fdiv_rn(amax_row, 7.0f);
        } else if (valid) {
          const float rr = amax_row > 0.f ? __fdiv_rn(p.qmax, amax_row) : 0.0f;
          full_store_int8<NB>(y, rr, p.codes + row * p.K, b);
          if (b == 0) p.scales_f32[row] = __fdiv_rn(amax_row, p.qmax);
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
    }
  }
  if (MODE == kModeAmax) {
    const unsigned bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax_acc));
    if (lane == 0) atomicMax(p.amax_word, bits);
  }
}

// ---------------------------------------------------------------------------
// Full-width rotation of K = 4096 as a 64 x 64 two-pass transform, with the
// rows staged in shared memory.
//
// Sylvester's H_4096 is the Kronecker product of twelve H_2, one per bit of
// the element index n, so the bits can be transformed in any grouping.  The
// row is read as a 64 x 64 matrix X[a][b] with a = bits 3..8 of n and
// b = bits 0..2 and 9..11: H_64 along b in every matrix row, then H_64 along a
// in every column.  A team of 64 threads (two warps) owns one row at a time;
// eight teams per CTA, one CTA per SM.
//
// Staging: each CTA takes a contiguous run of rows (M / grid, rounded down or
// up) and, at kernel start, issues one bulk copy (cp.async.bulk, local memory,
// no multicast) per row into a ring of up to kF4kSlots shared-memory slots,
// building its sign table while they are in flight; so every CTA's reads are
// in the memory system from the start instead of one row per team at a time.
// Local row i goes to team i mod 8 and slot i mod S; once its team has read
// it into registers, the slot is refilled with row i + S (whichever team
// takes that one waits on the slot's mbarrier).
//
// Per row: thread a reads matrix row a (elements 8 a + 512 i + e) from the
// slot, signs and transforms it, and writes it to the team's fp32 transpose
// buffer; after a team barrier, thread b transforms column b.  The codes of
// its outputs (a = 0..63, b) go back through the team's code buffer as bytes,
// and thread t stores the codes of outputs 64 t .. 64 t + 63 with 16-byte
// stores.  Three team barriers per row (transpose, row max, codes).
// Shared-memory granules are XOR-swizzled so that the row writes, column
// reads and code transposes are free of bank conflicts (the code reads:
// two-way).  A team synchronises on its own named barrier (1..8).
// ---------------------------------------------------------------------------
constexpr int kR64Teams = 8;
constexpr int kR64Threads = 64 * kR64Teams;
constexpr int kF4kSlots = 7;                        // row slots per CTA
constexpr size_t kF4kRowBytes = 4096 * 2;
constexpr size_t kR64TeamBytes = 64 * 64 * 4 + 64 * 64 + 16;  // fp32 transpose | code bytes | row max slots
__host__ __device__ constexpr size_t f4k_smem_bytes(int slots) {
  // sign masks | team buffers | row slots | mbarriers (one per slot) | per-slot row tags | abort flag
  return 2048 * 4 + kR64Teams * kR64TeamBytes + (size_t)slots * kF4kRowBytes + (size_t)slots * 8 +
         (size_t)slots * 4 + 16;
}

__device__ __forceinline__ void team_sync(int team) {
  asm volatile("bar.sync %0, 64;" ::"r"(team + 1) : "memory");
}

// Team-wide AND of a predicate (every thread of the team gets the result).
__device__ __forceinline__ bool team_all(bool v, int team) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)v), "r"(team + 1)
      : "memory");
  return out != 0;
}

// 64-point fast Walsh-Hadamard transform in registers (unnormalized).
__device__ __forceinline__ void fwht64(float (&v)[64]) {
#pragma unroll
  for (int i = 0; i < 64; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = a + b;
    v[i + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < 64; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
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

// Four code bytes (two's complement, element order) -> two packed nibble bytes.
__device__ __forceinline__ uint32_t nibbles_of(uint32_t w0, uint32_t w1) {
  const uint32_t a = w0 & 0x0F0F0F0Fu, b = w1 & 0x0F0F0F0Fu;
  return __byte_perm(a | (a >> 4), b | (b >> 4), 0x6420);
}

template <int MODE>
__global__ void __launch_bounds__(kR64Threads, 1) rotate_full4096_kernel(const RotParams p, int slots) {
  griddep_wait();
  griddep_trigger();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem_raw);              // [2048] XOR masks, one per bf16 pair
  const int team = threadIdx.x >> 6, t = threadIdx.x & 63, lane = threadIdx.x & 31;
  uint8_t* tb = smem_raw + 2048 * 4 + (size_t)team * kR64TeamBytes;
  float* tr = reinterpret_cast<float*>(tb);             // [a][b] fp32, 16-byte granule g of row a at g ^ (a mod 16)
  uint8_t* cb = tb + 64 * 64 * 4;                       // [a][b] code bytes, 8-byte group g of row a at g ^ (a / 8)
  float* slot_max = reinterpret_cast<float*>(cb + 64 * 64);
  uint8_t* rows = smem_raw + 2048 * 4 + kR64Teams * kR64TeamBytes;  // [slots][8 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(rows + (size_t)slots * kF4kRowBytes);
  // the local row most recently issued into each slot.  Consecutive fills of a
  // slot go to different teams, so an mbarrier parity alone cannot tell a team
  // waiting for fill f from fill f - 2: a team first waits until the slot's
  // tag names its row -- the copy is issued, so fill f - 1 has completed (its
  // consumer issued this one) -- and only then for the fill's parity.
  int* tags = reinterpret_cast<int*>(bars + slots);
  int* abort_flag = tags + slots;
  // each CTA a contiguous run of M / grid rows (rounded down or up)
  const int64_t r_begin = (int64_t)blockIdx.x * p.rows / gridDim.x;
  const int nloc = (int)(((int64_t)blockIdx.x + 1) * p.rows / gridDim.x - r_begin);
  const int S = nloc < slots ? nloc : slots;  // slots in use (all rows when they fit)

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&bars[i], 1);
      tags[i] = i;
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  build_sign_table(p.signs, 32, smask, [&]() {
    if (threadIdx.x == 0) {  // the first S rows, one copy each
      for (int i = 0; i < S; ++i) {
        mbar_arrive_expect_tx(&bars[i], (unsigned)kF4kRowBytes);
        bulk_g2s(rows + (size_t)i * kF4kRowBytes, p.x + (r_begin + i) * p.sS, (unsigned)kF4kRowBytes, &bars[i]);
      }
    }
  });
  __syncthreads();

#pragma unroll 1
  for (int i = team; i < nloc; i += kR64Teams) {
    const int sl = i % S;
    const int64_t row = r_begin + i;
    uint8_t* buf = rows + (size_t)sl * kF4kRowBytes;
    bool ok = true;
    {
      const long long t0 = clock64();
      while (((volatile int*)tags)[sl] != i) {
        if (clock64() - t0 > kWaitLimitCycles) {
          atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
          ok = false;
          break;
        }
      }
    }
    ok = ok && mbar_wait_bounded(&bars[sl], (unsigned)((i / S) & 1));
    if (!team_all(ok, team)) {
      if (t == 0) atomicOr(abort_flag, 1);
      break;
    }
    float v[64];
    {
      const uint4* src = reinterpret_cast<const uint4*>(buf) + t;        // elements 8 t + 512 i + e
      const uint4* sm = reinterpret_cast<const uint4*>(smask) + t;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint4 w = src[64 * k];
        const uint4 sg = sm[64 * k];
        w.x ^= sg.x;
        w.y ^= sg.y;
        w.z ^= sg.z;
        w.w ^= sg.w;
        v[8 * k + 0] = __uint_as_float(w.x << 16);
        v[8 * k + 1] = __uint_as_float(w.x & 0xFFFF0000u);
        v[8 * k + 2] = __uint_as_float(w.y << 16);
        v[8 * k + 3] = __uint_as_float(w.y & 0xFFFF0000u);
        v[8 * k + 4] = __uint_as_float(w.z << 16);
        v[8 * k + 5] = __uint_as_float(w.z & 0xFFFF0000u);
        v[8 * k + 6] = __uint_as_float(w.w << 16);
        v[8 * k + 7] = __uint_as_float(w.w & 0xFFFF0000u);
      }
    }
    fwht64(v);
#pragma unroll
    for (int g = 0; g < 16; ++g)
      *reinterpret_cast<float4*>(tr + 64 * t + 4 * (g ^ (t & 15))) =
          make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
    team_sync(team);  // the transpose is written, and every thread has read the row out of its slot
    if (t == 0 && i + S < nloc) {  // refill the slot with row i + S
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bars[sl], (unsigned)kF4kRowBytes);
      bulk_g2s(buf, p.x + (row + S) * p.sS, (unsigned)kF4kRowBytes, &bars[sl]);
      ((volatile int*)tags)[sl] = i + S;
    }
#pragma unroll
    for (int k = 0; k < 64; ++k) v[k] = tr[64 * k + 4 * ((t >> 2) ^ (k & 15)) + (t & 3)];
    fwht64(v);
    // v[k] is output n = (t mod 8) + 8 k + 512 (t / 8)
    if (MODE == kModeF32) {
      float* orow = p.out_f32 + row * p.ldo + (t & 7) + 512 * (t >> 3);
#pragma unroll
      for (int k = 0; k < 64; ++k) orow[8 * k] = v[k] * 0.015625f;
      team_sync(team);  // every column read is done before the next row's writes
      continue;
    }
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int k = 0; k < 64; k += 4) {
      a0 = fmaxf(a0, fabsf(v[k]));
      a1 = fmaxf(a1, fabsf(v[k + 1]));
      a2 = fmaxf(a2, fabsf(v[k + 2]));
      a3 = fmaxf(a3, fabsf(v[k + 3]));
    }
    float am = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    if (lane == 0) slot_max[t >> 5] = am;
    team_sync(team);
    const float amax = fmaxf(slot_max[0], slot_max[1]) * 0.015625f;  // max |x~| (x~ = H x / 64, exact scaling)
    const float qmax = MODE == kModeInt4 ? 7.0f : p.qmax;
    const float rr = amax > 0.f ? __fdiv_rn(qmax, amax) : 0.0f;
    const float cr = rr * 0.015625f;
#pragma unroll
    for (int k = 0; k < 64; k += 2) {
      const float2 q = __ffma2_rn(make_float2(v[k], v[k + 1]), make_float2(cr, cr),
                                  make_float2(kRoundMagic, kRoundMagic));
      cb[64 * k + (t ^ (8 * (k >> 3)))] = (uint8_t)__float_as_uint(q.x);
      cb[64 * (k + 1) + (t ^ (8 * ((k + 1) >> 3)))] = (uint8_t)__float_as_uint(q.y);
    }
    team_sync(team);
    // outputs 64 t + 8 r + e sit at a = 8 (t mod 8) + r, b = 8 (t / 8) + e
    uint2 c[8];
#pragma unroll
    for (int r = 0; r < 8; ++r)
      c[r] = *reinterpret_cast<const uint2*>(cb + 64 * (8 * (t & 7) + r) + 8 * ((t >> 3) ^ (t & 7)));
    if (MODE == kModeInt4) {
      uint4* dst = reinterpret_cast<uint4*>(p.codes + row * 2048 + 32 * t);
      dst[0] = make_uint4(nibbles_of(c[0].x, c[0].y), nibbles_of(c[1].x, c[1].y), nibbles_of(c[2].x, c[2].y),
                          nibbles_of(c[3].x, c[3].y));
      dst[1] = make_uint4(nibbles_of(c[4].x, c[4].y), nibbles_of(c[5].x, c[5].y), nibbles_of(c[6].x, c[6].y),
                          nibbles_of(c[7].x, c[7].y));
    } else {
      uint4* dst = reinterpret_cast<uint4*>(p.codes + row * 4096 + 64 * t);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = make_uint4(c[2 * k].x, c[2 * k].y, c[2 * k + 1].x, c[2 * k + 1].y);
    }
    if (t == 0) p.scales_f32[row] = __fdiv_rn(amax, qmax);
  }
  __syncthreads();
  // after a timed-out wait, let this CTA's own copies in flight land before it exits
  if (*abort_flag && threadIdx.x == 0) {
    for (int sl = 0; sl < S; ++sl) (void)mbar_wait_bounded(&bars[sl], (unsigned)((tags[sl] / S) & 1));
  }
}

// ---------------------------------------------------------------------------
// NVFP4 with the dynamic per-tensor scale in ONE pass over HBM, for tensors that
// fit in the SMs' combined shared memory: a cooperative launch (all CTAs
// resident) where each CTA copies its rows into shared memory once, rotates
// them and takes the max |X~| of its rows, meets the other CTAs at a grid-wide
// barrier (atomic counter, bounded spin), and then quantizes its rotated rows
// with g = max/(6*448).
//
// Between the two passes the rotated values wait in tensor memory when they
// fit (stash = 1: at most 512 128-value units per CTA, i.e. 256 KB of fp32):
// each thread writes its unit's 128 registers into its warp's TMEM lane
// quadrant with tcgen05.st (column group warp / 4, or 3 for a second unit) and
// reads them back after the barrier, so the rows are rotated once.  With more
// units per CTA (stash = 0) the second pass rotates the rows again from
// shared memory.
// p.amax_word[0] gathers the max, p.amax_word[1] counts arrivals; both are
// zeroed by the host before the launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc512(uint32_t* dst_smem) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(dst_smem))
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free512(uint32_t taddr) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(taddr) : "memory");
}
// 128 fp32 registers of this thread to / from its lane, 128 consecutive columns
// from `taddr` (the warp's lane-quadrant base and first column).
__device__ __forceinline__ void tmem_store128(uint32_t taddr, const float (&v)[128]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float* q = &v[32 * k];
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr + 32u * (uint32_t)k),
        "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]), "f"(q[8]),
        "f"(q[9]), "f"(q[10]), "f"(q[11]), "f"(q[12]), "f"(q[13]), "f"(q[14]), "f"(q[15]), "f"(q[16]), "f"(q[17]),
        "f"(q[18]), "f"(q[19]), "f"(q[20]), "f"(q[21]), "f"(q[22]), "f"(q[23]), "f"(q[24]), "f"(q[25]),
        "f"(q[26]), "f"(q[27]), "f"(q[28]), "f"(q[29]), "f"(q[30]), "f"(q[31])
        : "memory");
  }
}
__device__ __forceinline__ void tmem_load128(uint32_t taddr, float (&v)[128]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float* q = &v[32 * k];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=f"(q[0]), "=f"(q[1]), "=f"(q[2]), "=f"(q[3]), "=f"(q[4]), "=f"(q[5]), "=f"(q[6]), "=f"(q[7]),
          "=f"(q[8]), "=f"(q[9]), "=f"(q[10]), "=f"(q[11]), "=f"(q[12]), "=f"(q[13]), "=f"(q[14]), "=f"(q[15]),
          "=f"(q[16]), "=f"(q[17]), "=f"(q[18]), "=f"(q[19]), "=f"(q[20]), "=f"(q[21]), "=f"(q[22]), "=f"(q[23]),
          "=f"(q[24]), "=f"(q[25]), "=f"(q[26]), "=f"(q[27]), "=f"(q[28]), "=f"(q[29]), "=f"(q[30]), "=f"(q[31])
        : "r"(taddr + 32u * (uint32_t)k)
        : "memory");
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

constexpr int kResThreads = 384;
constexpr int kResStashUnits = 512;  // 128 lanes x 4 column groups of 128

template <int LOGB>
__global__ void __launch_bounds__(kResThreads, 1) rotate_nvfp4_resident_kernel(const RotParams p, int rows_per_cta,
                                                                              int stash) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int nb = p.nb;
  const int64_t r0 = (int64_t)blockIdx.x * rows_per_cta;
  const int nrows = (int)max((int64_t)0, min((int64_t)rows_per_cta, p.rows - r0));
  const size_t row_bytes = (size_t)p.K * 2;
  uint8_t* rows = smem_raw;
  uint32_t* smask = reinterpret_cast<uint32_t*>(smem_raw + (size_t)rows_per_cta * row_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smask + nb * 64);  // one per row: a warp starts on its row once it lands
  unsigned* cta_max = reinterpret_cast<unsigned*>(bars + rows_per_cta);
  int* flag = reinterpret_cast<int*>(cta_max + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(flag + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr bool PERM = ChunkOrder<LOGB>::kPermuted;
  const ChunkKeys ck = chunk_keys<LOGB>(tid);
  const int m = ck.m;
  const float c = LOGB == 7 ? 0.08838834764831845f : (LOGB == 0 ? 1.0f : p.cblk);  // 1/sqrt(block), rounded once

  if (tid == 0) {
    for (int rr = 0; rr < nrows; ++rr) mbar_init(&bars[rr], 1);
    fence_mbar_init();
    *cta_max = 0u;
  }
  if (stash && warp == 0) tmem_alloc512(tmem_slot);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = stash ? *tmem_slot : 0u;
  // this warp's lanes; column group of its first and second unit
  const uint32_t tq = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  build_sign_table(p.signs, nb, smask, [&]() {
    if (tid == 0) {  // one copy per row, in row order
      for (int rr = 0; rr < nrows; ++rr) {
        mbar_arrive_expect_tx(&bars[rr], (unsigned)row_bytes);
        bulk_g2s(rows + (size_t)rr * row_bytes, p.x + (r0 + rr) * p.sS, (unsigned)row_bytes, &bars[rr]);
      }
    }
  });
  __syncthreads();

  // pass 1: rotate, max |X~| over this CTA's rows (and, stashing, park the values
  // in TMEM); each thread waits only for the row of its own unit
  const int units = nrows * nb;
  float amax = 0.f;
  bool ok = true;
  if (stash) {
#pragma unroll 1
    for (int i = 0; i < 2; ++i) {
      if (32 * warp + kResThreads * i >= units) break;  // warp-uniform: no unit for any lane
      const int u = tid + kResThreads * i;
      const bool have = u < units;
      const int r = have ? u / nb : 0, b = have ? u - r * nb : 0;
      if (have) ok = ok && mbar_wait_bounded(&bars[r], 0);
      float v[128];
      load_block(rows + (size_t)r * row_bytes + (size_t)b * 256, smask + b * 64, m, v);
      fwht_block_diag<LOGB>(v);
      if (have) amax = fmaxf(amax, absmax128(v) * c);
      tmem_store128(tq + 128u * (uint32_t)(i == 0 ? (warp >> 2) : 3), v);
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  } else {
    for (int u = tid; u < units; u += blockDim.x) {
      const int r = u / nb, b = u - r * nb;
      ok = ok && mbar_wait_bounded(&bars[r], 0);
      float v[128];
      load_block(rows + (size_t)r * row_bytes + (size_t)b * 256, smask + b * 64, m, v);
      fwht_block_diag<LOGB>(v);
      amax = fmaxf(amax, absmax128(v) * c);
    }
  }
  const unsigned wbits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax));
  if ((tid & 31) == 0) atomicMax(cta_max, wbits);
  const bool loaded = __syncthreads_and(ok) != 0;  // every row of this CTA landed

  // grid-wide barrier: publish this CTA's max, count arrivals, wait for all
  volatile unsigned* gmax = p.amax_word;
  volatile unsigned* count = p.amax_word + 1;
  if (tid == 0) {
    atomicMax(p.amax_word, *cta_max);
    __threadfence();
    atomicAdd(p.amax_word + 1, 1u);
    bool ok = true;
    const long long t0 = clock64();
    while (*count < gridDim.x) {
      __nanosleep(64);
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
        ok = false;
        break;
      }
    }
    __threadfence();
    *flag = (ok && loaded) ? 1 : 0;
  }
  __syncthreads();

  // pass 2: quantize with the tensor's scale (skipped after a timed-out barrier)
  if (*flag) {
    const float g = __fdiv_rn(__uint_as_float(*gmax), 2688.0f);
    const float inv6g = g > 0.f ? __frcp_rn(6.0f * g) : 0.0f;
    if (blockIdx.x == 0 && tid == 0 && p.g_out) *p.g_out = g;
    if (stash) {
#pragma unroll 1
      for (int i = 0; i < 2; ++i) {
        if (32 * warp + kResThreads * i >= units) break;
        const int u = tid + kResThreads * i;
        float v[128];
        tmem_load128(tq + 128u * (uint32_t)(i == 0 ? (warp >> 2) : 3), v);
        if (u < units) {
          const int r = u / nb, b = u - r * nb;
          const int64_t row = r0 + r;
          quant_nvfp4_store<PERM, LOGB == 0>(v, c, g, inv6g, ck.mchi, ck.mo,
                                             p.codes + row * (p.K / 2) + (size_t)b * 64,
                                             p.scales_e4m3 + row * (p.K / 16) + (size_t)b * 8);
        }
      }
    } else {
      for (int u = tid; u < units; u += blockDim.x) {
        const int r = u / nb, b = u - r * nb;
        const int64_t row = r0 + r;
        float v[128];
        load_block(rows + (size_t)r * row_bytes + (size_t)b * 256, smask + b * 64, m, v);
        fwht_block_diag<LOGB>(v);
        quant_nvfp4_store<PERM, LOGB == 0>(v, c, g, inv6g, ck.mchi, ck.mo,
                                           p.codes + row * (p.K / 2) + (size_t)b * 64,
                                           p.scales_e4m3 + row * (p.K / 16) + (size_t)b * 8);
      }
    }
  }
  if (stash) {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      tmem_free512(tmem);
    }
  }
}

}  // namespace rq
