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
// * kv4_attn_partial_kernel: one CTA (4 warps) per 1024 cached tokens of one
//   (batch, head); the code rows stream through a three-stage shared-memory
//   ring of 128-token stages (cp.async.bulk; a "full" and a per-warp "read"
//   mbarrier per stage, bounded waits, no CTA-wide barrier in the loop), the
//   per-token fp16 scales and zeros through registers one stage ahead.  Warp 0
//   rotates q with shuffles (two butterfly stages in
//   registers, five across lanes) and folds 1/sqrt(128), the softmax scale and
//   log2(e) into it, so scores come out in the log2 domain for exp2.  Lane l
//   keeps the quarter l mod 4 of q~ (32 values) and, for each group of 32
//   tokens, reads the same quarter of 4 tokens' 64-byte code rows with
//   16-byte shared-memory loads.  A score is s.(q~ . c) + z.sum(q~): the codes are
//   never dequantized; a nibble's own bit pattern is read as an fp32
//   subnormal and multiplied by an operand pre-scaled by 2^100 (one PRMT per
//   nibble, no conversion arithmetic).  The four lanes of a token add
//   their partial dots with two shuffles.  Online softmax per warp; the value
//   side accumulates w.c with w = p.s_v in the same lane layout, plus sum p.z_v.
//   The CTA merges its warps and writes (max, sum, o~[128]) per chunk.
// * kv4_attn_combine_kernel: one CTA per (batch, head) merges the chunks,
//   normalises, rotates the 128 values back (Hadamard across threads: shuffles
//   within warps, shared memory across them) and applies the signs.
#pragma once

#include "rq_common.cuh"

namespace rq {

constexpr int kAttnChunk = 1024;    // cached tokens per CTA
constexpr int kAttnStageTok = 128;  // tokens per shared-memory stage (32 per warp)
constexpr int kAttnStages = 3;
constexpr int kAttnStageBytes = kAttnStageTok * 64 * 2;  // K codes | V codes
constexpr size_t kAttnSmem = (size_t)kAttnStages * kAttnStageBytes + 2 * kAttnStages * 8;
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

// A code nibble n is turned into a float for free: its bit pattern n is the
// fp32 subnormal n * 2^-149.  Multiplied by an operand pre-scaled by 2^100
// (kNibScale) the product x * n * 2^-49 is a normal number, exact up to the
// product's own rounding, and the sums are scaled back by 2^49 (kNibUnscale)
// once.  (The kernels are built without flush-to-zero, so the subnormal inputs
// are honoured; the pre-scaled operands stay far below the fp32 range.)
constexpr float kNibScale = 1.2676506002282294e30f;   // 2^100
constexpr float kNibUnscale = 562949953421312.0f;     // 2^49

// The nibbles of one 32-bit word as subnormal floats, paired for packed math:
// pair j = (element 2j, element 2j + 1) of the word (low nibble first).
__device__ __forceinline__ void word_nibbles(uint32_t w, float2 (&f)[4]) {
  const uint32_t ev = w & 0x0F0F0F0Fu;          // elements 0, 2, 4, 6
  const uint32_t od = (w >> 4) & 0x0F0F0F0Fu;   // elements 1, 3, 5, 7
#pragma unroll
  for (int j = 0; j < 4; ++j)
    f[j] = make_float2(__uint_as_float(__byte_perm(ev, 0u, 0x4440 | j)),
                       __uint_as_float(__byte_perm(od, 0u, 0x4440 | j)));
}

// sum over the 32 nibbles of c (word i: elements 8i..8i+7) times x[0..31],
// with x pre-scaled by 2^100; the result carries the 2^-49 factor.
__device__ __forceinline__ float dot32_nibbles(const uint4 c, const float (&x)[32]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f[4];
    word_nibbles(w[i], f);
    acc0 = __ffma2_rn(f[0], make_float2(x[8 * i], x[8 * i + 1]), acc0);
    acc1 = __ffma2_rn(f[1], make_float2(x[8 * i + 2], x[8 * i + 3]), acc1);
    acc0 = __ffma2_rn(f[2], make_float2(x[8 * i + 4], x[8 * i + 5]), acc0);
    acc1 = __ffma2_rn(f[3], make_float2(x[8 * i + 6], x[8 * i + 7]), acc1);
  }
  return (acc0.x + acc0.y) + (acc1.x + acc1.y);
}

// o[0..31] += w * (the 32 nibbles of c), w pre-scaled by 2^100 (o carries 2^-49).
__device__ __forceinline__ void axpy32_nibbles(const uint4 c, float wgt, float (&o)[32]) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  const float2 ww = make_float2(wgt, wgt);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f[4];
    word_nibbles(w[i], f);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 t = __ffma2_rn(f[k], ww, make_float2(o[8 * i + 2 * k], o[8 * i + 2 * k + 1]));
      o[8 * i + 2 * k] = t.x;
      o[8 * i + 2 * k + 1] = t.y;
    }
  }
}

// Bulk-copy the K and V code rows of stage-iteration n (tokens g0 + 128 n ...,
// at most 128, clipped at S) into stage buffer `buf`; one elected thread.
__device__ __forceinline__ void attn_issue(const AttnParams& p, int64_t row0, int64_t t, uint8_t* buf, uint64_t* bar) {
  const int64_t cnt = min((int64_t)kAttnStageTok, p.S - t);
  const unsigned bytes = (unsigned)(cnt * 64);
  mbar_arrive_expect_tx(bar, 2 * bytes);
  bulk_g2s(buf, p.kc + (row0 + t) * 64, bytes, bar);
  bulk_g2s(buf + kAttnStageTok * 64, p.vc + (row0 + t) * 64, bytes, bar);
}

__device__ __forceinline__ float4 attn_scales(const AttnParams& p, int64_t row0, int64_t t) {
  const int64_t tt = t < p.S ? t : p.S - 1;
  return make_float4(__half2float(p.ks[row0 + tt]), __half2float(p.kz[row0 + tt]), __half2float(p.vs[row0 + tt]),
                     __half2float(p.vz[row0 + tt]));
}

__global__ void __launch_bounds__(128) kv4_attn_partial_kernel(const AttnParams p) {
  griddep_wait();
  griddep_trigger();
  extern __shared__ __align__(128) uint8_t attn_smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(attn_smem + kAttnStages * kAttnStageBytes);
  uint64_t* empty = full + kAttnStages;  // one arrival per warp once it has read the stage
  __shared__ float qs[128];
  __shared__ float qsum_s;
  __shared__ float wm[4], wl[4];
  __shared__ __align__(16) float wo[4][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.x / p.nchunks;   // one CTA per (batch*head, chunk)
  const int chunk = (int)(blockIdx.x - bh * p.nchunks);
  const float kNegInf = -__int_as_float(0x7f800000);
  const int64_t S = p.S;
  const int64_t row0 = bh * S;
  const int64_t g0 = (int64_t)chunk * kAttnChunk;
  const int n_iter = (int)((min((int64_t)kAttnChunk, S - g0) + kAttnStageTok - 1) / kAttnStageTok);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAttnStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)  // the cache starts streaming before q is rotated
    for (int n = 0; n < kAttnStages && n < n_iter; ++n)
      attn_issue(p, row0, g0 + (int64_t)kAttnStageTok * n, attn_smem + n * kAttnStageBytes, &full[n]);
  float4 scl = attn_scales(p, row0, g0 + 32 * warp + lane);

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
  for (int j = 0; j < 32; ++j) qq[j] = qs[32 * quarter + j] * kNibScale;
  const float qsum = qsum_s;

  float m = kNegInf, l = 0.f, zacc = 0.f;
  float o[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j] = 0.f;

  bool timed_out = false;
  int n_stop = 0;
#pragma unroll 1
  for (int n = 0; n < n_iter; ++n) {
    const int st = n % kAttnStages;
    // warps drift apart by up to a stage; a warp that gives up on a wait
    // leaves the loop, the device error word records the timeout and the
    // CTA's partial result is not to be used
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[st], (unsigned)((n / kAttnStages) & 1)))) {
      timed_out = true;
      n_stop = n;
      break;
    }
    const float4 cur = scl;
    if (n + 1 < n_iter) scl = attn_scales(p, row0, g0 + (int64_t)kAttnStageTok * (n + 1) + 32 * warp + lane);
    const int64_t t0 = g0 + (int64_t)kAttnStageTok * n + 32 * warp;  // this warp's 32 tokens
    if (t0 < S) {
      const uint8_t* kb = attn_smem + st * kAttnStageBytes + 32 * warp * 64;
      const uint8_t* vb = kb + kAttnStageTok * 64;
      uint4 kq[4], vq[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // lane l: quarter l mod 4 of token 8i + l/4 -- the 512 bytes at 512 i + 16 l
        kq[i] = *reinterpret_cast<const uint4*>(kb + 512 * i + 16 * lane);
        vq[i] = *reinterpret_cast<const uint4*>(vb + 512 * i + 16 * lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
      float sc[4];
      float gmax = kNegInf;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = 8 * i + (lane >> 2);
        float dsum = dot32_nibbles(kq[i], qq);
        dsum += __shfl_xor_sync(0xFFFFFFFFu, dsum, 1);
        dsum += __shfl_xor_sync(0xFFFFFFFFu, dsum, 2);
        dsum *= kNibUnscale;
        const float s_k = __shfl_sync(0xFFFFFFFFu, cur.x, tok);
        const float z_k = __shfl_sync(0xFFFFFFFFu, cur.y, tok);
        sc[i] = (t0 + tok < S) ? fmaf(s_k, dsum, z_k * qsum) : kNegInf;
        gmax = fmaxf(gmax, sc[i]);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xFFFFFFFFu, gmax, off));
      const float m_new = fmaxf(m, gmax);               // finite: token t0 is valid
      const float corr = exp2f(m - m_new);              // 0 on the first group (m = -inf)
      float psum = 0.f, zsum = 0.f;
      float w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tok = 8 * i + (lane >> 2);
        const float pi = exp2f(sc[i] - m_new);          // 0 for masked tokens
        const float s_v = __shfl_sync(0xFFFFFFFFu, cur.z, tok);
        const float z_v = __shfl_sync(0xFFFFFFFFu, cur.w, tok);
        psum += pi;
        zsum = fmaf(pi, z_v, zsum);
        w[i] = pi * s_v * kNibScale;
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
    else if (lane == 0) {
      mbar_arrive(&empty[st]);  // no tokens of this warp in the stage
    }
    if (warp == 0 && n + kAttnStages < n_iter) {
      // lane 0 refills stage st once every warp has read it; the warp leaves
      // the loop together if that wait gives up
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait_bounded(&empty[st], (unsigned)((n / kAttnStages) & 1));
        if (ok) {
          fence_proxy_async_smem();
          attn_issue(p, row0, g0 + (int64_t)kAttnStageTok * (n + kAttnStages), attn_smem + st * kAttnStageBytes,
                     &full[st]);
        }
      }
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
        timed_out = true;
        n_stop = n;
        break;
      }
    }
  }
  if (timed_out && threadIdx.x == 0) {
    // stages n_stop+1 .. n_stop+kAttnStages-1 may still be in flight: let
    // them land before the CTA finishes (stage n_stop landed or gave up)
    for (int j = n_stop + 1; j < n_stop + kAttnStages && j < n_iter; ++j)
      (void)mbar_wait_bounded(&full[j % kAttnStages], (unsigned)((j / kAttnStages) & 1));
  }
  // merge the lanes of the same quarter (lane bits 2..4) and the z terms
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] += __shfl_xor_sync(0xFFFFFFFFu, o[j], off);
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j] *= kNibUnscale;
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
  griddep_wait();
  griddep_trigger();
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
