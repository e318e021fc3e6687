/*
 * kvq.h -- libkvq: rotate-then-quantize int4 KV-cache codec for NVIDIA B200
 * (sm_100a).  Plain C ABI: device pointers, sizes and a CUDA stream; no C++
 * or framework types.
 *
 * The method ("Quantization Speed Is Often a Kernel Problem", section
 * "First, the 17%"): every K/V vector x of length d is multiplied by a fixed
 * random +-1 sign vector D, rotated by an orthonormal transform R (SRFT, a
 * real-packed FFT; or SRHT, a Walsh-Hadamard transform, the control),
 * quantized to int4 with one absmax scale per group of g consecutive rotated
 * values, and stored as packed nibbles plus fp32 scales.  The inverse
 * dequantizes and rotates back.  Section "Fusing four steps into two kernels
 * is not enough": each direction is one fused kernel, so data never makes a
 * round trip through memory between the steps.
 *
 * Exact definitions used by every entry point:
 *   u = D x                                   (signs[i] in {+1, -1})
 *   SRFT: X_k = sum_n u_n exp(-2 pi i k n / d), and
 *         y[0] = Re X_0 / sqrt(d),  y[1] = Re X_{d/2} / sqrt(d),
 *         y[2k] = sqrt(2) Re X_k / sqrt(d), y[2k+1] = sqrt(2) Im X_k / sqrt(d)
 *         for 1 <= k < d/2  (the real packing of the rfft output).
 *   SRHT: y = H u / sqrt(d), H_ij = (-1)^popcount(i & j) (Sylvester order).
 *   group j = y[j*g .. j*g+g-1]:  s_j = max|y_i| / 7 (fp32),
 *         q_i = round_half_even(y_i / s_j) in [-7, 7]  (q = 0 when s_j = 0),
 *         ("Chapter 25 - Quantization: The Hardware View", sample symmetric
 *         quantizer: qmax = 7, codes clamped to [-8, 7]).
 *   packed byte b of a vector = (q_{2b} & 0xF) | ((q_{2b+1} & 0xF) << 4)
 *         (same chapter, "Why INT4 Packing Needs Special Code": w0 in the
 *         low nibble, w1 in the high nibble; two's complement nibbles).
 *   inverse: y_hat_i = s_j q_i, x_hat = D R^T y_hat, rounded to fp16.
 *
 * Arithmetic is fp32 on the device; the outputs match a float64 evaluation
 * of the definitions except for codes whose y/s lies within float32 error of
 * a rounding tie.
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers allocated and owned by the
 *     caller.  The library never allocates device memory and keeps no
 *     per-call state.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     return as soon as the work is enqueued.  Results are ready when the
 *     stream is synchronized.  The decode-step and attention calls are
 *     launched with programmatic dependent launch: their blocks may be
 *     scheduled while the previous kernel of the stream drains, but they
 *     touch no global memory before that kernel has completed, so stream
 *     order holds for their inputs and outputs as for any other launch.
 *   - Every argument check runs on the host before anything is launched; a
 *     failing check returns its status and enqueues nothing.  KVQ_ERR_CUDA
 *     reports a CUDA runtime error raised while enqueueing.
 *   - Inputs must be finite fp16 values; NaN/Inf are outside the contract.
 *   - Outputs must not alias inputs.
 *   - Supported shapes: d in {64, 128, 256}; group in {32, 64, 128, 256}
 *     with group <= d (group divides d).
 *   - Alignment: x, out, packed, x_new and the scales of the forward and
 *     inverse steps must be 16-byte aligned (whole tiles move by TMA copies);
 *     the decode step's scales cache needs 4 bytes.
 *   - fp16 data is passed as uint16_t bit patterns (IEEE-754 binary16).
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The library is built with hidden symbol visibility: only the functions
 * declared here are exported, so two builds loaded into one process (for
 * instance a test build beside the product one) share no internal state. */
#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *kvq_stream;

typedef enum {
  KVQ_ROT_SRFT = 0, /* sign-randomized real-packed FFT (the method) */
  KVQ_ROT_SRHT = 1  /* sign-randomized Walsh-Hadamard (the control) */
} kvq_rot;

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_NULL = 1,           /* a required pointer is NULL                */
  KVQ_ERR_BAD_DIM = 2,        /* d not in {64, 128, 256}                    */
  KVQ_ERR_BAD_GROUP = 3,      /* group not in {32,64,128,256} or > d        */
  KVQ_ERR_MISALIGNED = 4,     /* a pointer breaks the alignment rule        */
  KVQ_ERR_BAD_ROT = 5,        /* rot is neither SRFT nor SRHT               */
  KVQ_ERR_CUDA = 6,           /* CUDA runtime error while enqueueing        */
  KVQ_ERR_BAD_SIZE = 7,       /* negative or too large count / position     */
  KVQ_ERR_DEVICE_TIMEOUT = 8, /* a kernel gave up waiting for its own copy  */
  KVQ_ERR_UNSUPPORTED_DEVICE = 9, /* device is not compute capability 10.0 */
  KVQ_ERR_BAD_BITS = 10       /* code width not 3 (d >= 128), 4, 6 or 8     */
} kvq_status;

/*
 * Forward step ("First, the 17%"; "Fusing four steps into two kernels is not
 * enough": rotate plus quantize in one kernel).
 *
 *   x       [n_vec][d] fp16, row-major, 16-byte aligned (read)
 *   n_vec   number of vectors, 0 <= n_vec < 2^31 (0: no-op, returns KVQ_OK)
 *   d       vector length, 64 / 128 / 256
 *   group   scale group g, 32 / 64 / 128 / 256, g <= d
 *   signs   [d] int8 in {+1, -1}, device memory (read).  Values other than
 *           +-1 are not detected; any negative value acts as -1.
 *   rot     KVQ_ROT_SRFT or KVQ_ROT_SRHT
 *   packed  [n_vec][d/2] uint8, 16-byte aligned (written)
 *   scales  [n_vec][d/g] fp32, 16-byte aligned (written)
 *   stream  CUDA stream
 */
KVQ_API kvq_status kvq_rot_quant_fwd(const uint16_t *x, int64_t n_vec, int32_t d,
                                     int32_t group, const int8_t *signs, kvq_rot rot,
                                     uint8_t *packed, float *scales, kvq_stream stream);

/*
 * Inverse step ("First, the 17%": dequantized and rotated back when
 * attention reads it; "Fusing four steps...": dequantize plus inverse
 * rotate in one kernel).
 *
 *   packed  [n_vec][d/2] uint8, 16-byte aligned (read)
 *   scales  [n_vec][d/g] fp32, 16-byte aligned (read)
 *   out     [n_vec][d] fp16, 16-byte aligned (written): x_hat = D R^T (s q)
 *   other arguments as in kvq_rot_quant_fwd.
 */
KVQ_API kvq_status kvq_dequant_rot_inv(const uint8_t *packed, const float *scales,
                                       int64_t n_vec, int32_t d, int32_t group,
                                       const int8_t *signs, kvq_rot rot, uint16_t *out,
                                       kvq_stream stream);

/*
 * Forward and inverse steps with a per-channel factor lambda, the kernel
 * hook of "Quantization Speed Is Often a Kernel Problem", section "Before you
 * celebrate..." (first condition: per-channel lambda plus per-group
 * abs-max, inside the fused kernel).  The pages do not define how lambda is
 * calibrated, so it is an input:
 *   forward: u = D (lambda * x) (channel-wise), then as kvq_rot_quant_fwd;
 *   inverse: x_hat = (D R^T y_hat) / lambda (channel-wise, before the fp16
 *            rounding), i.e. the inverse step of the same scaled space.
 *   lambda  [d] fp32, 8-byte aligned DEVICE pointer (read); finite and
 *           non-zero (not checked on the device).  NULL -> KVQ_ERR_NULL.
 *   other arguments as in kvq_rot_quant_fwd / kvq_dequant_rot_inv.
 */
KVQ_API kvq_status kvq_rot_quant_fwd_lambda(const uint16_t *x, int64_t n_vec, int32_t d,
                                            int32_t group, const int8_t *signs,
                                            const float *lambda, kvq_rot rot,
                                            uint8_t *packed, float *scales,
                                            kvq_stream stream);
KVQ_API kvq_status kvq_dequant_rot_inv_lambda(const uint8_t *packed, const float *scales,
                                              int64_t n_vec, int32_t d, int32_t group,
                                              const int8_t *signs, const float *lambda,
                                              kvq_rot rot, uint16_t *out,
                                              kvq_stream stream);

/*
 * Forward and inverse steps with another code width b ("Quantization Speed
 * Is Often a Kernel Problem": "6-bit and 8-bit are lossless; 3-bit is worse";
 * "Chapter 25 - Quantization: The Hardware View", sample quantizer:
 * qmax = 2^(b-1) - 1):
 *   s_j = max|y_i| / (2^(b-1) - 1), q_i = round_half_even(y_i / s_j);
 *   packed row of a vector: d*b/8 bytes, a little-endian bitstream in which
 *   code i occupies bits [b i, b i + b) as b-bit two's complement (for b = 4
 *   this is the nibble layout above).
 *   bits    3 (d >= 128 only: a d = 64 row would be 24 bytes), 4, 6 or 8;
 *           anything else -> KVQ_ERR_BAD_BITS
 *   packed  [n_vec][d*bits/8] uint8, 16-byte aligned
 *   other arguments as in kvq_rot_quant_fwd / kvq_dequant_rot_inv.
 */
KVQ_API kvq_status kvq_rot_quant_fwd_bits(const uint16_t *x, int64_t n_vec, int32_t d,
                                          int32_t group, int32_t bits,
                                          const int8_t *signs, kvq_rot rot,
                                          uint8_t *packed, float *scales,
                                          kvq_stream stream);
KVQ_API kvq_status kvq_dequant_rot_inv_bits(const uint8_t *packed, const float *scales,
                                            int64_t n_vec, int32_t d, int32_t group,
                                            int32_t bits, const int8_t *signs,
                                            kvq_rot rot, uint16_t *out,
                                            kvq_stream stream);

/*
 * Decode step for one head-major cache, one launch ("A scene" and "First,
 * the 17%": every layer, every decoding step, the new K/V token is rotated
 * and quantized and the cache is dequantized for attention).
 *
 * For every head h < n_heads:
 *   1. forward step on x_new[h] -> packed[h][pos], scales[h][pos];
 *   2. out[h][t] = inverse step of cache row t for t < pos, and
 *      out[h][pos] = inverse step of the fresh codes of x_new[h].
 * K and V of a layer are passed either as two calls or as 2*n_heads heads of
 * one buffer.
 *
 *   x_new   [n_heads][d] fp16, 16-byte aligned (read)
 *   packed  [n_heads][cap][d/2] uint8, 16-byte aligned (row pos written,
 *           rows < pos read)
 *   scales  [n_heads][cap][d/g] fp32, 4-byte aligned (same)
 *   n_heads >= 0 (0: no-op); cap >= 1; 0 <= pos < cap
 *   out     [n_heads][pos+1][d] fp16, 16-byte aligned (written)
 *   other arguments as in kvq_rot_quant_fwd.
 */
KVQ_API kvq_status kvq_decode_step(const uint16_t *x_new, uint8_t *packed,
                                   float *scales, int64_t n_heads, int64_t cap,
                                   int64_t pos, int32_t d, int32_t group,
                                   const int8_t *signs, kvq_rot rot, uint16_t *out,
                                   kvq_stream stream);

/*
 * Decode step with a dequantized-prefix cache and an fp16 tail ("Quantization
 * Speed Is Often a Kernel Problem", section "Before you celebrate...", second
 * condition: the dequantized prefix is kept between steps instead of being
 * recomputed, the last tokens stay in fp16, and the cache is refreshed when
 * that window fills).  `kv` is the attention view the caller keeps across
 * the steps of one sequence; a step touches O(window) rows, not O(pos).
 *
 * For every head h < n_heads:
 *   - kv[h][pos] = x_new[h] exactly (fp16 tail);
 *   - if (pos + 1) % window == 0, the window rows r in
 *     [pos + 1 - window, pos] (kv rows, and x_new for r = pos) go through the
 *     forward step into packed[h][r], scales[h][r], and kv[h][r] is replaced
 *     by the inverse step of those codes.
 * So after the call, kv rows of completed windows hold the dequantized
 * values (identical to kvq_decode_step's output rows) and the rows of the
 * open window hold the tokens themselves; packed/scales rows of the open
 * window are not written.
 *
 *   x_new   [n_heads][d] fp16, 16-byte aligned (read)
 *   packed  [n_heads][cap][d/2] uint8, 16-byte aligned (window rows written)
 *   scales  [n_heads][cap][d/g] fp32, 4-byte aligned (window rows written)
 *   kv      [n_heads][cap][d] fp16, 16-byte aligned (row pos written; on a
 *           flush the window rows are read and rewritten)
 *   n_heads >= 0 (0: no-op); cap >= 1; 0 <= pos < cap
 *   window  1 <= window <= 4096 (16 in the pages' design)
 *   other arguments as in kvq_rot_quant_fwd.
 */
KVQ_API kvq_status kvq_decode_step_windowed(const uint16_t *x_new, uint8_t *packed,
                                            float *scales, uint16_t *kv,
                                            int64_t n_heads, int64_t cap, int64_t pos,
                                            int32_t window, int32_t d, int32_t group,
                                            const int8_t *signs, kvq_rot rot,
                                            kvq_stream stream);

/*
 * Decode attention that reads the int4 cache directly ("Day 9 -
 * Quantization: Shrink the Bytes Themselves", section "Decode into HBM, or
 * Decode into Registers": the dequantization happens inside the consuming
 * kernel; "Quantization Speed Is Often a Kernel Problem", "First, the 17%":
 * K and V are dequantized and rotated back when attention reads them).
 *
 * For every KV head h < n_kv_heads and query i < n_q, with
 * K_t = D R^T (s q)_K[h][t] and V_t likewise for t < len (exact, not
 * rounded to fp16):
 *   s_t = sm_scale <q[h][i], K_t>,  p = softmax(s),
 *   out[h][i] = sum_t p_t V_t, rounded to fp16.
 * Only codes and scales are read from memory: the kernel rotates each query
 * once (R orthonormal: <q, D R^T y> = <R D q, y>), accumulates
 * sum_t p_t y_V,t in the rotated domain and rotates back once per query.
 * Arithmetic is fp32.  With one scale per token (group == d) the products
 * run on the tensor cores, up to 4 queries per thread block (except d = 64
 * with one query, and more than 4 queries over more than 32,767 KV heads):
 * scores as exact integer products of the codes with each query in 27-bit
 * fixed point (error at most 2^-27 of the query's largest coordinate), the
 * weighted sum of V with each weight split into bf16 high and low parts
 * (about 2^-17 relative); both below the fp16 rounding of the output.
 *
 *   q         [n_kv_heads][n_q][d] fp16, 16-byte aligned (read)
 *   k_packed, v_packed  [n_kv_heads][cap][d/2] uint8, 16-byte aligned (read)
 *   k_scales, v_scales  [n_kv_heads][cap][d/g] fp32, 4-byte aligned (read)
 *   n_kv_heads 0..65535 (0: no-op); n_q 1..8 queries per KV head (GQA)
 *   cap >= 1; 1 <= len <= cap (rows [0, len) are attended)
 *   sm_scale  finite softmax scale (e.g. 1/sqrt(d))
 *   out       [n_kv_heads][n_q][d] fp16, 16-byte aligned (written)
 *   signs, rot, d, group as in kvq_rot_quant_fwd (the D and R the cache
 *   was written with).
 */
KVQ_API kvq_status kvq_attend_decode(const uint16_t *q, const uint8_t *k_packed,
                                     const float *k_scales, const uint8_t *v_packed,
                                     const float *v_scales, int64_t n_kv_heads,
                                     int32_t n_q, int64_t cap, int64_t len, int32_t d,
                                     int32_t group, const int8_t *signs, kvq_rot rot,
                                     float sm_scale, uint16_t *out, kvq_stream stream);

/* Static, NUL-terminated description of a status code (never NULL). */
KVQ_API const char *kvq_status_string(kvq_status s);

/*
 * Device-side error word of the current device.  The kernels bound every
 * wait on their own asynchronous copies; a wait that runs out records
 * KVQ_ERR_DEVICE_TIMEOUT here and the kernel returns early.  This call
 * synchronizes the device, returns KVQ_OK or the recorded status, and clears
 * the word when `clear` is non-zero.
 */
KVQ_API kvq_status kvq_device_status(int32_t clear);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
KVQ_API int32_t kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
