// One decoding step of attention over the 4-bit KV cache (sm_100a).
//
// "QuaRot (rotation-based outlier removal, W4A4KV4)", "Activation scheme":
// keys and values are stored rotated and quantized to 4 bits (the KV4 of
// W4A4KV4, asymmetric with an fp16 scale and zero per vector as the SpinQuant
// page's "Activation scheme" has it).  For orthogonal Q, q.K^T = (q.Q).(K.Q)^T
// ("Rotations for 4-Bit Activations", "A rotation changes nothing"), so the
// query is rotated with the same per-head Q = diag(s).H_128/sqrt(128) and the
// scores need no de-rotation; the weighted sum of rotated values is rotated
// back at the end.  The cache is what rq_kv_rotate_quantize writes.
//
// Split-S ("flash-decoding") in two kernels:
// * kv4_attn_partial_kernel: one CTA (4 warps) per 256 cached tokens of one
//   (batch, head).  Warp 0 rotates q with shuffles (two butterfly stages in
//   registers, five across lanes) and folds 1/sqrt(128), the softmax scale and
//   log2(e) into it, so scores come out in the log2 domain for exp2.  Lane l
//   keeps the quarter l mod 4 of q~ (32 values) and, for each group of 32
//   tokens, reads the same quarter of 4 tokens' 64-byte code rows with
//   coalesced 16-byte loads.  A score is s.(q~ . c) + z.sum(q~): the codes are
//   never dequantized; a nibble becomes a float through PRMT into the
//   exponent of 2^23 and one packed subtraction.  The four lanes of a token add
//   their partial dots with two shuffles.  Online softmax per warp; the value
//   side accumulates w.c with w = p.s_v in the same lane layout, plus sum p.z_v.
//   The CTA merges its warps and writes (max, sum, o~[128]) per chunk.
// * kv4_attn_combine_kernel: one CTA per (batch, head) merges the chunks,
//   normalises, rotates the 128 values back (Hadamard across threads: shuffles
//   within warps, shared memory across them) and applies the signs.
#pragma once

#include "rq_common.cuh"

namespace rq {

constexpr int kAttnChunk = 256;     // cached tokens per CTA
constexpr int kAttnPart = 132;      // floats per chunk record: max, sum, 128 values, pad

struct AttnParams {
  const __nv_bfloat16* q;   // [BH, 128]
  const uint8_t* kc;        // [BH, S, 64]
  const __half* ks;         // [BH, S]
  const __half* kz;
  const uint8_t* vc;
  const __half* vs;
  const __half* vz;
  const int8_t* signs;      // [128]
  float qscale;             // softmax scale * log2(e) / sqrt(128)
  int64_t S;
  int nchunks;
  float* part;              // [BH, nchunks, kAttnPart]
  void* out;                // [BH, 128]
  int out_bf16;
};

// 4 nibbles of a 16-bit group -> float2 pairs, via PRMT into the low byte of
// 2^23's bit pattern and one packed subtraction of 2^23.
__device__ __forceinline__ float2 nib_pair(uint32_t e, int k) {
  // e holds one nibble per byte; byte k and byte k+1 -> (float, float)
  const uint32_t magic = 0x4B000000u;
  const uint32_t a = __byte_perm(e, magic, 0x7540 | k);          // [e.b_k, 0, 0, 0x4B]
  const uint32_t b = __byte_perm(e, magic, 0x7540 | (k + 1));
  return __fadd2_rn(make_float2(__uint_as_float(a), __uint_as_float(b)),
                    make_float2(-8388608.0f, -8388608.0f));
}

// acc (float2) += sum over the 32 nibbles of c (byte j: element 2j low, 2j+1
// high) times x[0..31], as packed pairs (x[2i], x[2i+1]).
__device__ __forceinline__ float dot32_nibbles(const uint4 c, const float (&x)[32]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // word i = elements 8i..8i+7; even ones in the low nibbles, odd in the high
    const uint32_t ev = w[i] & 0x0F0F0F0Fu;         // elements 8i, 8i+2, 8i+4, 8i+6
    const uint32_t od = (w[i] >> 4) & 0x0F0F0F0Fu;  // elements 8i+1, 8i+3, 8i+5, 8i+7
    const uint32_t lo = __byte_perm(ev, od, 0x5140);  // bytes: e0 o0 e1 o1 -> elements 8i..8i+3
    const uint32_t hi = __byte_perm(ev, od, 0x7362);  // elements 8i+4..8i+7
    const float2 f0 = nib_pair(lo, 0), f1 = nib_pair(lo, 2), f2 = nib_pair(hi, 0), f3 = nib_pair(hi, 2);
    acc0 = __ffma2_rn(f0, make_float2(x[8 * i], x[8 * i + 1]), acc0);
    acc1 = __ffma2_rn(f1, make_float2(x[8 * i + 2], x[8 * i + 3]), acc1);
    acc0 = __ffma2_rn(f2, make_float2(x[8 * i + 4], x[8 * i + 5]), acc0);
    acc1 = __ffma2_rn(f3, make_float2(x[8 * i + 6], x[8 * i + 7]), acc1);
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// o[0..31] += w * (the 32 nibbles of c), packed.
__device__ __forceinline__ void axpy32_nibbles(const uint4 c, float wgt, float (&o)[32]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  const float2 ww = make_float2(wgt, wgt);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t ev = w[i] & 0x0F0F0F0Fu;
    const uint32_t od = (w[i] >> 4) & 0x0F0F0F0Fu;
    const uint32_t lo = __byte_perm(ev, od, 0x5140);
    const uint32_t hi = __byte_perm(ev, od, 0x7362);
    const float2 f[4] = {nib_pair(lo, 0), nib_pair(lo, 2), nib_pair(hi, 0), nib_pair(hi, 2)};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 t = __ffma2_rn(f[k], ww, make_float2(o[8 * i + 2 * k], o[8 * i + 2 * k + 1]));
      o[8 * i + 2 * k] = t.x;
      o[8 * i + 2 * k + 1] = t.y;
    }
  }
}

__global__ void __launch_bounds__(128) kv4_attn_partial_kernel(const AttnParams p) {
  __shared__ float qs[128];
  __shared__ float qsum_s;
  __shared__ float wm[4], wl[4];
  __shared__ __align__(16) float wo[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.x / p.nchunks;   // one CTA per (batch*head, chunk)
  const int chunk = (int)(blockIdx.x - bh * p.nchunks);
  const float kNegInf = -__int_as_float(0x7f800000);

  if (warp == 0) {
    // q~ = (q . diag(s) . H_128) * qscale; lane l holds elements 4l..4l+3
    const uint2 qb = *reinterpret_cast<const uint2*>(p.q + bh * 128 + 4 * lane);
    const uint32_t sg = *reinterpret_cast<const uint32_t*>(p.signs + 4 * lane);
    float v[4];
    v[0] = __uint_as_float(qb.x << 16);
    v[1] = __uint_as_float(qb.x & 0xFFFF0000u);
    v[2] = __uint_as_float(qb.y << 16);
    v[3] = __uint_as_float(qb.y & 0xFFFF0000u);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if ((sg >> (8 * j + 7)) & 1u) v[j] = -v[j];
    // element bits 0, 1 in registers
    float a = v[0] + v[1], b = v[0] - v[1], c = v[2] + v[3], d = v[2] - v[3];
    v[0] = a + c; v[2] = a - c; v[1] = b + d; v[3] = b - d;
    // element bits 2..6 are lane bits 0..4
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const bool upper = (lane >> k) & 1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float o = __shfl_xor_sync(0xFFFFFFFFu, v[j], 1 << k);
        v[j] = upper ? (o - v[j]) : (v[j] + o);
      }
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[j] *= p.qscale;
      qs[4 * lane + j] = v[j];
      sum += v[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) qsum_s = sum;
  }
  __syncthreads();
  const int quarter = lane & 3;
  float qq[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) qq[j] = qs[32 * quarter + j];
  const float qsum = qsum_s;

  float m = kNegInf, l = 0.f, zacc = 0.f;
  float o[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j] = 0.f;

  const int64_t S = p.S;
  const int64_t row0 = bh * S;
#pragma unroll 1
  for (int g = 0; g < 2; ++g) {
    const int64_t t0 = (int64_t)chunk * kAttnChunk + warp * 64 + 32 * g;
    if (t0 >= S) break;
    // scale / zero of the group's tokens, one per lane
    const int64_t tl = t0 + lane < S ? t0 + lane : S - 1;
    const float ksl = __half2float(p.ks[row0 + tl]), kzl = __half2float(p.kz[row0 + tl]);
    const float vsl = __half2float(p.vs[row0 + tl]), vzl = __half2float(p.vz[row0 + tl]);
    uint4 kq[4], vq[4];
    int tok[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tok[i] = 8 * i + (lane >> 2);  // token within the group
      const int64_t t = t0 + tok[i] < S ? t0 + tok[i] : S - 1;
      kq[i] = *reinterpret_cast<const uint4*>(p.kc + (row0 + t) * 64 + 16 * quarter);
      vq[i] = *reinterpret_cast<const uint4*>(p.vc + (row0 + t) * 64 + 16 * quarter);
    }
    float sc[4];
    float gmax = kNegInf;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float dsum = dot32_nibbles(kq[i], qq);
      dsum += __shfl_xor_sync(0xFFFFFFFFu, dsum, 1);
      dsum += __shfl_xor_sync(0xFFFFFFFFu, dsum, 2);
      const float s_k = __shfl_sync(0xFFFFFFFFu, ksl, tok[i]);
      const float z_k = __shfl_sync(0xFFFFFFFFu, kzl, tok[i]);
      sc[i] = (t0 + tok[i] < S) ? fmaf(s_k, dsum, z_k * qsum) : kNegInf;
      gmax = fmaxf(gmax, sc[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xFFFFFFFFu, gmax, off));
    const float m_new = fmaxf(m, gmax);               // finite: the group has a valid token
    const float corr = exp2f(m - m_new);              // 0 on the first group (m = -inf)
    float psum = 0.f, zsum = 0.f;
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float pi = exp2f(sc[i] - m_new);          // 0 for masked tokens
      const float s_v = __shfl_sync(0xFFFFFFFFu, vsl, tok[i]);
      const float z_v = __shfl_sync(0xFFFFFFFFu, vzl, tok[i]);
      psum += pi;
      zsum = fmaf(pi, z_v, zsum);
      w[i] = pi * s_v;
    }
    // each token is held by the four lanes of its quarter group: count it once
    psum = quarter == 0 ? psum : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xFFFFFFFFu, psum, off);
    l = fmaf(l, corr, psum);
    zacc = fmaf(zacc, corr, zsum);
    m = m_new;
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] *= corr;
#pragma unroll
    for (int i = 0; i < 4; ++i) axpy32_nibbles(vq[i], w[i], o);
  }
  // merge the lanes of the same quarter (lane bits 2..4) and the z terms
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] += __shfl_xor_sync(0xFFFFFFFFu, o[j], off);
  }
  float zs = quarter == 0 ? zacc : 0.f;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) zs += __shfl_xor_sync(0xFFFFFFFFu, zs, off);
  if (lane < 4) {
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(&wo[warp][32 * lane + j]) =
          make_float4(o[j] + zs, o[j + 1] + zs, o[j + 2] + zs, o[j + 3] + zs);
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
  __syncthreads();
  // CTA merge: thread d owns element d
  const int d = threadIdx.x;
  float M = fmaxf(fmaxf(wm[0], wm[1]), fmaxf(wm[2], wm[3]));
  float L = 0.f, O = 0.f;
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const float f = wm[wi] == kNegInf ? 0.f : exp2f(wm[wi] - M);
    L = fmaf(wl[wi], f, L);
    O = fmaf(wo[wi][d], f, O);
  }
  float* rec = p.part + (bh * p.nchunks + chunk) * kAttnPart;
  rec[2 + d] = O;
  if (d == 0) {
    rec[0] = M;
    rec[1] = L;
  }
}

__global__ void __launch_bounds__(128) kv4_attn_combine_kernel(const AttnParams p) {
  __shared__ float buf[128];
  const int64_t bh = blockIdx.x;
  const int d = threadIdx.x, lane = d & 31, warp = d >> 5;
  const float* rec = p.part + bh * p.nchunks * kAttnPart;
  const float kNegInf = -__int_as_float(0x7f800000);
  float M = kNegInf;
  for (int c = 0; c < p.nchunks; ++c) M = fmaxf(M, rec[c * kAttnPart]);
  float L = 0.f, O = 0.f;
  for (int c = 0; c < p.nchunks; ++c) {
    const float mc = rec[c * kAttnPart];
    const float f = mc == kNegInf ? 0.f : exp2f(mc - M);
    L = fmaf(rec[c * kAttnPart + 1], f, L);
    O = fmaf(rec[c * kAttnPart + 2 + d], f, O);
  }
  float v = O / L;
  // rotate back: (o~ . H_128 / sqrt(128)) * s.  Bits 0..4 of d across lanes.
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const bool upper = (lane >> k) & 1;
    const float o = __shfl_xor_sync(0xFFFFFFFFu, v, 1 << k);
    v = upper ? (o - v) : (v + o);
  }
  // bits 5, 6 across warps through shared memory
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    buf[d] = v;
    __syncthreads();
    const float o = buf[d ^ (32 << k)];
    __syncthreads();
    v = ((warp >> k) & 1) ? (o - v) : (v + o);
  }
  v *= 0.08838834764831845f;  // 1/sqrt(128), rounded once
  if (p.signs[d] < 0) v = -v;
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[bh * 128 + d] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p.out)[bh * 128 + d] = v;
}

}  // namespace rq
