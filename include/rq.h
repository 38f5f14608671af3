/*
 * rq.h -- C ABI of librq: the online hot path of rotation-based W4A4
 * quantization (QuaRot / SpinQuant style) on NVIDIA B200 (sm_100a).
 *
 * The method ("Rotations for 4-Bit Activations: QuaRot, SpinQuant, and
 * Friends", section "A rotation changes nothing, and that is the point"):
 * a linear layer Y = X.W^T equals (X.Q).(W.Q)^T for any orthogonal Q, so X.Q
 * and W.Q are quantized instead of X and W.  Q is a randomized Hadamard matrix
 * scaled by 1/sqrt(n) -- a +-1 sign per channel followed by a Sylvester
 * Hadamard -- either over all K channels or block-diagonal in 128-wide blocks
 * (sections "The recipe" and "Gotchas"; QuaRot page, "Activation scheme").
 *
 *   Q = blockdiag_{K/B}( diag(s_blk) . H_B / sqrt(B) ),  B = 128 or B = K,
 *   H_B[i][j] = (-1)^popcount(i & j).
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are DEVICE pointers owned by the caller; the
 *    library never allocates, frees or retains them.  Host arrays are named
 *    *_host.  Matrices are row-major; leading dimensions are in elements.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and never synchronizes, except
 *    rq_get_device_error and rq_init.
 *  - The rotate, GEMM and attention kernels are launched with programmatic
 *    dependent launch: a kernel may be scheduled while the previous kernel on
 *    the stream drains, but it reads and writes no global memory before that
 *    kernel has completed, so stream order is kept.  Calls may be captured
 *    into CUDA graphs.
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call returns a status other than RQ_OK and leaves every output
 *    untouched.  RQ_ERR_CUDA reports a launch failure (cudaGetLastError).
 *  - Kernels that wait on barriers give up after about one second, record
 *    RQ_ERR_TIMEOUT in a device word and return; rq_get_device_error reads it.
 *  - Codes are packed two per byte, element 2i in the low nibble (bits 0-3),
 *    element 2i+1 in the high nibble.  INT4 codes are two's complement in
 *    [-7, 7]; KV4 codes unsigned in [0, 15]; NVFP4 codes are E2M1 with the
 *    sign in bit 3 (a value that rounds to zero is written as +0).
 *  - Inputs must be finite and, for KV4, within the fp16 range; NaN or Inf
 *    inputs give unspecified codes.
 */
#ifndef RQ_H_
#define RQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RQ_API __attribute__((visibility("default")))
#else
#define RQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef void* rq_stream_t; /* a cudaStream_t */

typedef enum {
  RQ_OK = 0,
  RQ_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
  RQ_ERR_UNSUPPORTED_SHAPE = 2, /* K, block or head_dim outside what the kernels support */
  RQ_ERR_ALIGNMENT = 3,         /* a pointer or leading dimension breaks the stated alignment */
  RQ_ERR_UNSUPPORTED_DEVICE = 4,/* not a compute-capability 10.0 GPU, or the sm_100a image does not load */
  RQ_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
  RQ_ERR_TIMEOUT = 6            /* a kernel gave up on a bounded wait (see rq_get_device_error) */
} rq_status;

typedef enum {
  RQ_INT4 = 0,  /* symmetric INT4, one fp32 scale per row */
  RQ_NVFP4 = 1, /* E2M1, one E4M3 scale per 16 values, fp32 per-tensor scale */
  RQ_MXFP4 = 2, /* E2M1, one E8M0 (power-of-two) scale per 32 values */
  RQ_INT8 = 3,  /* symmetric 8-bit, one int8 code per byte, one fp32 scale per row */
  RQ_INT6 = 4,  /* symmetric 6-bit (codes in [-31, 31]), one int8 byte each, one fp32 scale per row */
  RQ_INT4_ASYM = 5, /* asymmetric 4-bit per group of 128 along K: fp16 (scale, zero) per group */
  RQ_INT4_BYTES = 6 /* the RQ_INT4 codes and scales, one int8 byte per code (the layout the integer MMA reads) */
} rq_format;

typedef enum {
  RQ_OUT_F32 = 0,     /* Y as fp32 */
  RQ_OUT_BF16 = 1,    /* Y as bf16 (round to nearest even) */
  RQ_OUT_I32_ACC = 2  /* integer formats only: the raw int32 accumulators sum_k qx*qw, no scales */
} rq_out;

typedef enum {
  RQ_SCALE_DYNAMIC = 0, /* NVFP4 per-tensor scale from the rotated tensor's own max */
  RQ_SCALE_STATIC = 1   /* NVFP4 per-tensor scale supplied by the caller */
} rq_gscale;

/* Checks that `device` is a compute-capability 10.0 GPU and that this
 * library's sm_100a kernels load on it.  Synchronous.  Call once per device
 * before the other entry points (they do not call it themselves). */
RQ_API rq_status rq_init(int device);

/* Static description of a status code.  Never NULL. */
RQ_API const char* rq_status_string(rq_status status);

/* Bytes of device workspace rq_rotate_quantize / rq_prepare_weights need:
 * 16 for NVFP4 (the dynamic-scale max word), 0 for the other formats.  The workspace must
 * be 16-byte aligned; its contents need not be initialised. */
RQ_API size_t rq_workspace_bytes(rq_format fmt);

/*
 * rq_rotate_quantize: X~ = X.Q, then quantize and pack (the online activation
 * side; "What it buys in 4 bits, and what it doesn't": INT4 with one scale per
 * token, or NVFP4 with an FP8 scale for every block of 16 values; "The full
 * model in NVFP4, on vLLM" and "When to rotate": MXFP4, whose scales are
 * powers of two shared by 32 values).
 *
 *  X_dev      bf16 [M, ldx]; rows 16-byte aligned (X_dev and ldx*2 multiples of 16).
 *  M          rows (tokens), >= 0.  M = 0 is a no-op.
 *  K          channels; a multiple of 128, at most 32768.
 *  signs_dev  int8 [K], 16-byte aligned, each +1 or -1 (the random sign diagonal;
 *             any other value is read as -1 if negative and +1 otherwise).
 *  block      128, 32 or 16 for block-diagonal rotations (32 and 16: blocks
 *             sized to the MXFP4 / NVFP4 scale groups, "Gotchas", "Block size
 *             matters"), or 0 for a full-width rotation (then K must be a power
 *             of two in [256, 4096]; INT4, INT6 and INT8 only), or 1 for no
 *             rotation: blocks of one channel, Q = diag(s).  With all signs +1
 *             that quantizes X itself -- the unrotated arm that section "What
 *             it buys in 4 bits, and what it doesn't" compares the rotated
 *             product error against.  Every format takes 1, 16, 32 or 128.
 *  fmt        RQ_INT4:
 *               codes_dev  uint8 [M, K/2], scales_dev float [M]:
 *               s = amax/7 (fp32, amax = max |x~| of the row); q = rint(x~/s).
 *             RQ_NVFP4:
 *               codes_dev  uint8 [M, K/2] E2M1 codes,
 *               scales_dev uint8 [M, K/16] E4M3 block scales,
 *               gscale_dev float scalar g:
 *                 RQ_SCALE_DYNAMIC: written, g = fp32(amax(X~)) / 2688;
 *                 RQ_SCALE_STATIC : read.
 *               S_b = E4M3_rn_satfinite(amax_b / (6 g));
 *               e = E2M1_rn_satfinite(x~ / (S_b g)); S_b = 0 gives e = 0.
 *             RQ_MXFP4:
 *               codes_dev  uint8 [M, K/2] E2M1 codes,
 *               scales_dev uint8 [M, K/32] E8M0 block scales (4-byte aligned):
 *               per block b of 32, 2^e_b with e_b = floor(log2(amax_b)) - 2
 *               clamped to [-127, 127] (the OCP Microscaling shared-exponent
 *               rule; the pages name only powers of two); e = E2M1_rn_satfinite(x~ / 2^e_b).
 *               amax_b = 0 gives scale code 0 and e = 0.  gscale_dev and
 *               workspace_dev are unused (may be NULL).
 *             RQ_INT8 / RQ_INT6 (6- and 8-bit round to nearest: "QuaRot", field
 *             "Bits"; the 8-bit activations of W4A8: "SpinQuant", field
 *             "Activation scheme"):
 *               codes_dev  int8 [M, K], scales_dev float [M]:
 *               s = amax/qmax with qmax = 127 / 31; q = rint(x~/s).  gscale_dev
 *               and workspace_dev are unused (may be NULL).
 *             RQ_INT4_BYTES (a weight layout for rq_int_gemm):
 *               codes_dev  int8 [M, K], scales_dev float [M]: exactly the
 *               RQ_INT4 codes and scales, one code per byte instead of two.
 *               Twice the memory of packed INT4; the GEMM then reads the
 *               codes as int8 MMA operands with no widening.
 *             RQ_INT4_ASYM (per-group asymmetric INT4, "SpinQuant", field
 *             "Activation scheme"; block 16, 32 or 128):
 *               codes_dev  uint8 [M, K/2], unsigned nibbles q in [0, 15],
 *               scales_dev fp16 pairs [M, K/128][2] = (s_h, z_h) per group of
 *               128 channels (4-byte aligned): z = min, s = (max - min)/15 of
 *               the group's x~, s_h = fp16(s), z_h = fp16(z);
 *               q = clamp(rint((x~ - z_h)/s_h), 0, 15) (s_h = 0 gives q = 0);
 *               x^ = z_h + s_h q.  No GEMM in this library consumes these codes.
 *               z and s are rounded to fp16 from the exact min and max: a
 *               group whose fp32 min or scale lies near an fp16 rounding
 *               midpoint has both re-evaluated in fp64 (as in
 *               rq_kv_rotate_quantize).
 *  workspace_dev  rq_workspace_bytes(fmt) bytes (may be NULL when that is 0).
 *  codes_dev and scales_dev 16-byte aligned (8 for NVFP4 scales).
 * Values that sit within a few fp32 ulps of a rounding boundary may round
 * either way (the rotation is computed in fp32).
 */
RQ_API rq_status rq_rotate_quantize(const void* X_dev, int64_t M, int64_t K, int64_t ldx, const int8_t* signs_dev,
                             int block, rq_format fmt, rq_gscale gmode, uint8_t* codes_dev, void* scales_dev,
                             float* gscale_dev, void* workspace_dev, rq_stream_t stream);

/*
 * rq_prepare_weights: the offline side, W~ = W.Q then quantize and pack, with
 * the same Q as the activations so (X.Q)(W.Q)^T = X.W^T ("Where the rotations
 * go": offline rotations are folded into the weights).  A row of W is an
 * output channel, so INT4 gives one scale per output channel.  Same arguments,
 * layouts and errors as rq_rotate_quantize with X -> W [N, K]; NVFP4 always
 * uses the dynamic per-tensor scale (gscale_dev is written).
 */
RQ_API rq_status rq_prepare_weights(const void* W_dev, int64_t N, int64_t K, int64_t ldw, const int8_t* signs_dev,
                             int block, rq_format fmt, uint8_t* codes_dev, void* scales_dev, float* gscale_dev,
                             void* workspace_dev, rq_stream_t stream);

/*
 * rq_w4a4_gemm: Y[M, N] = deq(X codes) . deq(W codes)^T, the quantized
 * product of section "What it buys in 4 bits, and what it doesn't".
 *  RQ_INT4 : xscales_dev float [M], wscales_dev float [N] (16-byte aligned);
 *            acc = sum_k qx[m,k] qw[n,k] exactly in int32; Y = acc * sx[m] * sw[n].
 *            xgscale_dev / wgscale_dev unused (may be NULL).
 *  RQ_NVFP4: xscales_dev uint8 [M, K/16], wscales_dev uint8 [N, K/16] (E4M3, 16-byte aligned),
 *            xgscale_dev / wgscale_dev float scalars;
 *            Y = gx gw sum_b Sx[m,b] Sw[n,b] sum_{k in b} ex ew.
 *  RQ_MXFP4: xscales_dev uint8 [M, K/32], wscales_dev uint8 [N, K/32] (E8M0, 16-byte aligned);
 *            Y = sum_b 2^(sx[m,b]-127) 2^(sw[n,b]-127) sum_{k in b} ex ew; the global
 *            scale pointers are unused (may be NULL).  RQ_OUT_I32_ACC is INT4 only.
 *  xcodes_dev uint8 [M, K/2], wcodes_dev uint8 [N, K/2], both 16-byte aligned.
 *  K a multiple of 128 (INT4), 256 (NVFP4) or 512 (MXFP4: scale rows of K/32
 *  bytes are copied in 16-byte units), at most 65536; M, N >= 0.
 *  Y_dev [M, ldy] of fp32, bf16 or int32 per `out`; ldy >= N; Y_dev aligned to
 *  its element size (16-byte aligned rows are stored with vector stores).
 */
RQ_API rq_status rq_w4a4_gemm(const uint8_t* xcodes_dev, const void* xscales_dev, const float* xgscale_dev,
                       const uint8_t* wcodes_dev, const void* wscales_dev, const float* wgscale_dev, int64_t M,
                       int64_t N, int64_t K, rq_format fmt, void* Y_dev, int64_t ldy, rq_out out,
                       rq_stream_t stream);

/*
 * rq_int_gemm: Y[M, N] = deq(X codes) . deq(W codes)^T for integer codes of
 * different widths on the two sides: W4A8 ("SpinQuant", field "Activation
 * scheme"), W8A8 and W6A6 ("QuaRot", field "Bits"), and W4A4.
 *  xfmt  RQ_INT4 (xcodes uint8 [M, K/2], packed nibbles), RQ_INT6 or RQ_INT8
 *        (xcodes int8 [M, K]); xscales float [M].
 *  wfmt  the same for W [N, K]; wscales float [N].
 *  Supported pairs (xfmt, wfmt): (INT4, INT4) -- the rq_w4a4_gemm INT4 path --
 *  (INT4, INT4_BYTES) -- the same W4A4 product with the weights' INT4 codes
 *  stored one per byte (wcodes int8 [N, K], from rq_prepare_weights with
 *  RQ_INT4_BYTES), which the two-SM kernel feeds to the tensor cores without
 *  widening them --, (INT6/INT8, INT4) and (INT6/INT8, INT6/INT8).
 *  (INT4, INT6/INT8) returns RQ_ERR_UNSUPPORTED_SHAPE.
 *  acc = sum_k qx[m,k] qw[n,k] exactly in int32 (|acc| < 2^31 for K <= 65536);
 *  Y = float(acc) * sx[m] * sw[n] (float(acc) rounds to nearest above 2^24).
 *  Codes 16-byte aligned, xscales 4-byte and wscales 16-byte aligned; K a
 *  multiple of 128, at most 65536; M, N >= 0; Y_dev, ldy and `out` as for
 *  rq_w4a4_gemm (RQ_OUT_I32_ACC gives the raw accumulators).
 */
RQ_API rq_status rq_int_gemm(const uint8_t* xcodes_dev, const float* xscales_dev, rq_format xfmt,
                             const uint8_t* wcodes_dev, const float* wscales_dev, rq_format wfmt, int64_t M,
                             int64_t N, int64_t K, void* Y_dev, int64_t ldy, rq_out out, rq_stream_t stream);

/*
 * rq_kv_rotate_quantize: 4-bit KV cache entries ("QuaRot", "Activation
 * scheme": the rotation is applied to the KV cache too; "SpinQuant",
 * "Activation scheme": asymmetric INT4 for the KV cache).  Each head_dim
 * vector v of K or V [B, H, S, D] (D = 128) becomes v~ = v.diag(s).H_128/sqrt(128),
 * then z = min(v~), s = (max(v~) - min(v~))/15, stored as fp16 z_h, s_h, and
 * q = clamp(rint((v~ - z_h)/s_h), 0, 15) (s_h = 0 gives q = 0).  z_h and s_h
 * are the fp16 roundings of the exact min and scale: the rotation runs in
 * fp32, and a vector whose fp32 min or scale lies near an fp16 rounding
 * midpoint has its min and max re-evaluated in fp64 (about 0.3 % of
 * vectors), within the same kernel.
 *  KV_dev      bf16, element (b,h,t,d) at KV_dev + b*strides_host[0] + h*strides_host[1]
 *              + t*strides_host[2] + d (strides in elements; d contiguous; each
 *              vector 16-byte aligned).
 *  signs_dev   int8 [D], 16-byte aligned.
 *  codes_dev   uint8 [B, H, S, D/2] contiguous, 16-byte aligned.
 *  scale_dev, zero_dev  fp16 [B, H, S] contiguous.
 */
RQ_API rq_status rq_kv_rotate_quantize(const void* KV_dev, int64_t B, int64_t H, int64_t S, int64_t D,
                                const int64_t* strides_host, const int8_t* signs_dev, uint8_t* codes_dev,
                                void* scale_dev, void* zero_dev, rq_stream_t stream);

/*
 * rq_kv4_decode_attention: one decoding step of attention over the 4-bit KV
 * cache written by rq_kv_rotate_quantize ("QuaRot", "Activation scheme": the
 * KV cache is stored rotated; "Rotations for 4-Bit Activations", "A rotation
 * changes nothing": q.K^T = (q.Q).(K.Q)^T).  For each (b, h): the query is
 * rotated with the same per-head Q = diag(s).H_128/sqrt(128) as the cache,
 * the cached vectors dequantize as z + s*q, p = softmax(q~.K~^T * scale) over
 * the S cached tokens, and o = (p.V~).Q^T is returned in the original basis.
 *  q_dev       bf16 [B, H, 128] contiguous, 16-byte aligned.
 *  kcodes_dev, vcodes_dev   uint8 [B, H, S, 64] contiguous, 16-byte aligned;
 *  kscale_dev, kzero_dev, vscale_dev, vzero_dev   fp16 [B, H, S] contiguous
 *              (the layouts rq_kv_rotate_quantize writes).
 *  signs_dev   int8 [128], 16-byte aligned: the signs the cache was rotated with.
 *  softmax_scale  > 0, or 0 for 1/sqrt(128).
 *  out_dev     [B, H, 128] fp32 (RQ_OUT_F32) or bf16 (RQ_OUT_BF16).
 *  workspace_dev  rq_kv4_attention_workspace_bytes(B, H, S) bytes, 16-byte aligned.
 *  S >= 1 (S = 0 is RQ_ERR_INVALID_ARG); B = 0 or H = 0 is a no-op.
 * Two kernels: per-chunk partial softmax sums, then a merge that rotates back.
 */
RQ_API size_t rq_kv4_attention_workspace_bytes(int64_t B, int64_t H, int64_t S);
RQ_API rq_status rq_kv4_decode_attention(const void* q_dev, int64_t B, int64_t H, int64_t S, const uint8_t* kcodes_dev,
                                         const void* kscale_dev, const void* kzero_dev, const uint8_t* vcodes_dev,
                                         const void* vscale_dev, const void* vzero_dev, const int8_t* signs_dev,
                                         float softmax_scale, void* out_dev, rq_out out, void* workspace_dev,
                                         rq_stream_t stream);

/*
 * rq_rotate_f32: the rotation alone, X~ = X.Q as fp32 [M, ldo] (ldo a multiple
 * of 4, out_dev 16-byte aligned).  Same X, K, signs and block rules as
 * rq_rotate_quantize (block 0 allowed for K a power of two in [256, 4096]).
 * Intended for checking the rotation against a reference.
 */
RQ_API rq_status rq_rotate_f32(const void* X_dev, int64_t M, int64_t K, int64_t ldx, const int8_t* signs_dev, int block,
                        float* out_dev, int64_t ldo, rq_stream_t stream);

/*
 * rq_rotate_quantize_nvfp4_noalloc: rq_rotate_quantize with fmt = RQ_NVFP4,
 * block = 128 and RQ_SCALE_DYNAMIC, for callers that cannot allocate device
 * memory -- engines that hand every byte of the GPU to a fixed arena sized at
 * start-up, plugin interfaces that offer no workspace, and latency-sensitive
 * hosts that avoid cudaMalloc (which synchronizes the device) after start-up.
 * It allocates nothing and needs no workspace argument: the 16 bytes of scratch
 * the dynamic scale needs live in a 256-byte static device array inside the
 * library (held by every GPU that loads the library until the process exits).
 * Not part of the method on the pages; it only changes where the scratch lives.
 *  - Same arguments, layouts and results as rq_rotate_quantize (NVFP4, dynamic
 *    scale; gscale_dev is written).  The scratch need does not depend on M or
 *    K; a scratch need above the array's 256 bytes would be rejected with
 *    RQ_ERR_UNSUPPORTED_SHAPE before anything runs.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.  The cached address belongs to the device's primary
 *    context: after cudaDeviceReset on that device, do not call this entry
 *    point again in the same process.
 *  - Every call clears the scratch it uses before use, but all calls share the
 *    one array: calls that may overlap on the GPU (different streams, or
 *    different host threads) race on it and must be serialized by the caller.
 */
RQ_API rq_status rq_rotate_quantize_nvfp4_noalloc(const void* X_dev, int64_t M, int64_t K, int64_t ldx,
                                                  const int8_t* signs_dev, uint8_t* codes_dev, void* scales_dev,
                                                  float* gscale_dev, rq_stream_t stream);

/*
 * rq_selftest_wait_timeout: exercises the device-side timeout path (every
 * wait of this library's kernels on an mbarrier or a flag is bounded).
 * Launches one tiny kernel that waits on an mbarrier
 * nobody arrives at, for at most `limit_cycles` SM clock cycles (1 .. the
 * library's own limit of 2e9 cycles, ~1 s), then records RQ_ERR_TIMEOUT in
 * the device error word and returns; the context stays usable.  The next
 * rq_get_device_error on the stream reports RQ_ERR_TIMEOUT (and clears it).
 * Returns RQ_ERR_INVALID_ARG for a limit out of range, RQ_ERR_CUDA if the
 * launch fails.
 */
RQ_API rq_status rq_selftest_wait_timeout(int64_t limit_cycles, rq_stream_t stream);

/* Synchronizes `stream`, returns RQ_ERR_TIMEOUT if any kernel of this library
 * recorded a device-side timeout since the last call (and clears the record),
 * RQ_ERR_CUDA if the stream reports an error, else RQ_OK. */
RQ_API rq_status rq_get_device_error(rq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RQ_H_ */
