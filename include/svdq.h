/*
 * svdq.h — C ABI of the B200 (sm_100a) SVDQuant W4A4 and AWQ W4A16 linear
 * layers.
 *
 * The layer (blog "Introducing Nunchaku 4-bit inference in Diffusers",
 * section "Background: SVDQuant and Nunchaku"): SVDQuant migrates activation
 * outliers into the weights with a per-input-channel smoothing vector lambda,
 * keeps the hardest part of each weight as a small 16-bit low-rank branch
 * L1 [K,r] L2 [r,N], and quantises the residual R = diag(lambda) W - L1 L2 to
 * 4 bits. The layer output is
 *     y = Q4(x_hat) . Q4(R) + (x_hat L1) L2 + b,   x_hat = bf16(x * (1/lambda)).
 * The low-rank down-projection runs inside the activation-quantisation pass and
 * the up-projection inside the 4-bit GEMM (same section, figure caption).
 * Formats (Diffusers "Nunchaku Lite" page, table "Supported quantization
 * types"): svdq_w4a4/nvfp4 group 16, svdq_w4a4/int4 group 64, awq_w4a16/int4
 * group 64; compute dtype bf16 (section "NunchakuLiteQuantizationConfig").
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call is
 *     asynchronous on it; results are valid after the stream reaches them.
 *   - Arguments are validated on the host before anything is launched:
 *     a bad argument returns an error status and launches nothing.
 *   - The device must be compute capability 10.0 (B200); any other device
 *     returns SVDQ_ERR_UNSUPPORTED_ARCH and launches nothing (the pages'
 *     loader likewise refuses an unsupported GPU with a clear error instead of
 *     producing wrong output: blog, section "Hardware support").
 *   - SVDQ_ERR_CUDA reports a failed launch (cudaGetLastError after launch).
 *   - Kernels bound every wait on another warp or on the copy engine; a wait
 *     that runs out sets the device error word (svdq_device_error) instead of
 *     hanging. There is ONE error word per device, shared by every stream and
 *     every call on that device: after concurrent calls on several streams a
 *     set bit cannot be attributed to one of them.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Packed 4-bit codes: element 2j of a row in the low nibble of byte j.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,      /* null pointer, bad enum, negative size */
  SVDQ_ERR_SHAPE = 2,            /* a size violates the shape rules below */
  SVDQ_ERR_ALIGN = 3,            /* a pointer is not 16-byte aligned */
  SVDQ_ERR_UNSUPPORTED_ARCH = 4, /* device is not compute capability 10.x */
  SVDQ_ERR_CUDA = 5,             /* CUDA runtime error (launch or query) */
  SVDQ_ERR_TIMEOUT = 6           /* a device-side bounded wait ran out */
} svdq_status;

typedef enum {
  SVDQ_NVFP4 = 0, /* E2M1 codes, UE4M3 scale per 16 along K, fp32 tensor scale */
  SVDQ_INT4 = 1   /* symmetric INT4 codes, bf16 scale per 64 along K */
} svdq_precision;

typedef enum {
  SVDQ_OUT_BF16 = 0,      /* y as bf16 [M, N] (the layer output) */
  SVDQ_OUT_F32 = 1,       /* y as fp32 [M, N] before the final bf16 rounding */
  SVDQ_OUT_I32_GROUPS = 2, /* INT4 only: raw int32 group dot products [M, N, K/64] */
  SVDQ_OUT_BF16_GELU = 3   /* NVFP4 only: bf16 of GELU(y), erf form, of the unrounded
                              output: the up-projection of the fused GELU-MLP
                              (Diffusers "Nunchaku Lite" page, section on fused
                              kernels), whose output feeds svdq_quantize_act of the
                              down-projection directly */
} svdq_out_dtype;

/* Human-readable name of a status. Never NULL. */
const char* svdq_status_str(svdq_status s);

/* Bytes of a scale buffer for a [rows, K] operand.
 * NVFP4: scales use the tiled layout read directly by the tensor-core GEMM:
 *   512-byte atoms of 128 rows x 4 scales (64 K elements). Atom (rb, ka)
 *   starts at byte ((rb * (K/64)) + ka) * 512; inside it, the scale of row
 *   rb*128 + 32*i + j (i < 4, j < 32) for K block 4*ka + c (c < 4) is at byte
 *   16*j + 4*i + c. rows are padded up to a multiple of 128 (padding scales 0).
 *   Size = ceil(rows/128) * 128 * K/16.
 * INT4: bf16, one per (row, 64-block): activations row-major [M, K/64] with
 *   the row pitch padded to pitch = 8 * ceil(K/512) scales (every row starts on
 *   a 16-byte boundary; the padding is never read); weights group-major
 *   [K/64, N] (one group's column scales contiguous for the GEMM epilogue).
 *   Size = rows * pitch * 2 (also enough for the weights' K/64 * N * 2).
 * Returns 0 for invalid arguments. */
size_t svdq_scale_bytes(svdq_precision p, int rows, int K);

/* Elements (bf16) of the prepared low-rank up-projection buffer `lr_up`:
 * NVFP4: N * 2r (see svdq_pack_weight); INT4: N * r. */
size_t svdq_lr_up_elems(svdq_precision p, int N, int r);

/* svdq_pack_weight — offline pack of one layer's weight (not on the timed path).
 * Defines (the blog's "Background" section; the readings of the open steps are
 * in the repository's design notes):
 *   inv_lambda[k] = 1/lambda[k]                 (fp32 division)
 *   R[k,n] = fp32( fp32(lambda[k]*W[k,n]) - sum_j L1[k,j] L2[j,n] ), sum in fp64
 *   NVFP4: s_tw = amax|R| / (6*448) (1 if 0); per (n, 16-block of k):
 *          sf = e4m3(amax/(6*s_tw)), code = e2m1(R * (1/(float(sf)*s_tw)))
 *   INT4:  per (n, 64-block of k): s = bf16(amax/7), q = clamp(rne(R/s), -8, 7)
 * In:  W fp32 [K, N] row-major (y = x W); lambda fp32 [K]; L1 bf16 [K, r];
 *      L2 bf16 [r, N]; act_tensor_scale = the static NVFP4 activation tensor
 *      scale s_tx the layer will be run with (ignored for INT4).
 * Out: w_codes u8 [N, K/2]; w_scales (svdq_scale_bytes(p, N, K) bytes);
 *      w_tensor_scale fp32 [2] = {s_tw, s_tx} ({1, 1} for INT4);
 *      inv_lambda fp32 [K];
 *      lr_up bf16 [N, rr] (K-major for the GEMM): NVFP4 rr = 2r holds the
 *      bf16 split hi + lo of L2[j,n] / (s_tw*s_tx) (hi in columns 0..r-1, lo
 *      in r..2r-1), so that the up-projection can share the 4-bit GEMM's
 *      accumulator; INT4 rr = r holds L2 transposed.
 * Shapes: K % 64 == 0; N % 8 == 0; N, K >= 1; r % 16 == 0 with 0 <= r <= 32
 *      (NVFP4) or 0 <= r <= 64 (INT4). r = 0 allows NULL L1/L2/lr_up/P.
 * Pointers 16-byte aligned. */
svdq_status svdq_pack_weight(svdq_precision p, int K, int N, int r, const float* W,
                             const float* lambda, const uint16_t* L1, const uint16_t* L2,
                             float act_tensor_scale, uint8_t* w_codes, void* w_scales,
                             float* w_tensor_scale, float* inv_lambda, uint16_t* lr_up,
                             void* stream);

/* svdq_quantize_act — the fused activation pass (smoothing, 4-bit group
 * quantisation and low-rank down-projection in one pass over x; blog,
 * "Background" section, figure caption).
 *   x_hat[m,k] = bf16(x[m,k] * inv_lambda[k])
 *   NVFP4: per 16-block: sf = e4m3(amax/(6*s_tx)), code = e2m1(x_hat * (1/(float(sf)*s_tx)))
 *   INT4:  per 64-block: s = bf16(amax/7), q = clamp(rne(x_hat/s), -8, 7)
 *   P[m,j] = bf16(sum_k x_hat[m,k] L1[k,j])      (fp32 accumulation)
 * In:  x bf16 [M, K]; inv_lambda fp32 [K] and w_tensor_scale fp32 [2] (both
 *      from svdq_pack_weight of the layer); L1 bf16 [K, r].
 *      The activation tensor scale s_tx is read from w_tensor_scale[1] on the
 *      device, so the activation pass and the GEMM (which folds s_tx into its
 *      output scale and into lr_up) always use the one value given to
 *      svdq_pack_weight. INT4 ignores w_tensor_scale (it may be NULL).
 * Out: x_codes u8 [M, K/2]; x_scales (svdq_scale_bytes(p, M, K) bytes);
 *      P bf16 [M, r].
 * Shapes: as svdq_pack_weight; M >= 0 (M = 0 is a no-op). */
svdq_status svdq_quantize_act(svdq_precision p, int M, int K, int r, const uint16_t* x,
                              const float* inv_lambda, const float* w_tensor_scale, const uint16_t* L1,
                              uint8_t* x_codes, void* x_scales, uint16_t* P, void* stream);

/* svdq_w4a4_linear — the 4-bit GEMM with the low-rank up-projection and the
 * bias fused in (blog, "Background" section, figure caption):
 *   NVFP4: y = s_tx*s_tw * sum_b sx[m,b] sw[n,b] sum_{k in b} qx qw + P L2 + bias
 *   INT4:  y = sum_g sx[m,g] sw[n,g] sum_{k in g} qx qw + P L2 + bias
 * In:  the outputs of svdq_quantize_act (x_codes, x_scales, P) and of
 *      svdq_pack_weight (w_codes, w_scales, w_tensor_scale, lr_up);
 *      bias bf16 [N] or NULL.
 * Out: y [M, N] row-major in the dtype selected by `out`
 *      (SVDQ_OUT_I32_GROUPS: int32 [M, N, K/64], INT4 only, ignores P/bias).
 * Shapes: as svdq_pack_weight; M >= 0. */
svdq_status svdq_w4a4_linear(svdq_precision p, int M, int K, int N, int r, const uint8_t* x_codes,
                             const void* x_scales, const uint16_t* P, const uint8_t* w_codes,
                             const void* w_scales, const float* w_tensor_scale,
                             const uint16_t* lr_up, const uint16_t* bias, void* y,
                             svdq_out_dtype out, void* stream);

/* svdq_rope_packed_bytes — bytes of the packed rotary table that
 * svdq_rope_pack writes for M rows: 16384 * ceil(M / 32). 0 for M < 0. */
size_t svdq_rope_packed_bytes(int M);

/* svdq_rope_pack — the rotary embedding's cos/sin tables in the layout the
 * fused QKV epilogue reads (a change of layout only: no arithmetic and no
 * step of the method itself). The tables depend only on the tokens'
 * positions, so one pack serves every attention layer of a forward pass.
 * In:  cos_t, sin_t fp32 [M, 64] (row m = the token's angles for the rotary
 *      pairs i = 0..63).
 * Out: rope fp32, svdq_rope_packed_bytes(M) bytes: blocks of 32 rows, each
 *      block 16 groups of 4 pairs, each group the cos part then the sin part,
 *      each part [32 rows][4 pairs]:
 *        cos[m, i] at float offset ((m/32 * 16 + i/4) * 2 + 0) * 128 + (m%32) * 4 + i%4
 *        sin[m, i] at the same offset + 128.
 *      Rows past M in the last block are written as zero.
 *      A warp whose lanes hold 32 consecutive rows reads one group of a table
 *      as 512 contiguous bytes (the plain [M, 64] rows would be 32 strided
 *      pieces).
 * The caller allocates rope. Pointers 16-byte aligned (else SVDQ_ERR_ALIGN);
 * M < 0, a NULL pointer, or rope overlapping cos_t or sin_t give
 * SVDQ_ERR_INVALID_ARG; M = 0 is a no-op. */
svdq_status svdq_rope_pack(int M, const float* cos_t, const float* sin_t, float* rope, void* stream);

/* svdq_w4a4_linear_qkv — the NVFP4 layer as a grouped Q/K/V projection with
 * the per-head RMSNorm of Q and K and the rotary embedding fused into the
 * GEMM's epilogue (Diffusers "Nunchaku Lite" page, section on fused kernels:
 * the QKV projection, RMSNorm and RoPE in one operator, and the grouped
 * to_qkv linear with Q, K and V concatenated along the output dimension).
 *   y_l = alpha * acc + P L2 + bias                      (as svdq_w4a4_linear, unrounded)
 *   for each row m and each head of Q (weight norm_q) and of K (norm_k), head
 *   columns d = 0..127:
 *     u[d] = y_l[d] / sqrt(mean_d(y_l[d]^2) + eps) * w[d]
 *     y[2i] = u[2i] cos[m,i] - u[2i+1] sin[m,i]; y[2i+1] = u[2i] sin[m,i] + u[2i+1] cos[m,i]
 *   V heads: y = y_l. Output rounded to bf16 once.
 * In:  as svdq_w4a4_linear (NVFP4); heads = heads per section (head_dim 128,
 *      N = 3 * heads * 128); norm_q, norm_k bf16 [128]; eps >= 0; rope = the
 *      M rows' cos/sin tables packed by svdq_rope_pack (for the same M).
 * Out: y bf16 [M, N].
 * Pointers 16-byte aligned (bias 4-byte). */
svdq_status svdq_w4a4_linear_qkv(int M, int K, int heads, int r, const uint8_t* x_codes, const void* x_scales,
                                 const uint16_t* P, const uint8_t* w_codes, const void* w_scales,
                                 const float* w_tensor_scale, const uint16_t* lr_up, const uint16_t* bias,
                                 const uint16_t* norm_q, const uint16_t* norm_k, float eps, const float* rope,
                                 uint16_t* y, void* stream);

/* svdq_qkv_norm_rope — the same per-head RMSNorm and rotary embedding as
 * svdq_w4a4_linear_qkv, as a separate pass over a grouped Q/K/V projection's
 * bf16 output y [M, 3 * heads * 128] (Q and K sections updated in place, V
 * untouched). It reads the rounded output, so it is the unfused form of the
 * operator that svdq_w4a4_linear_qkv computes on the unrounded accumulator.
 * Arguments as svdq_w4a4_linear_qkv, but with the plain tables: cos_t, sin_t
 * fp32 [M, 64]; pointers 16-byte aligned. */
svdq_status svdq_qkv_norm_rope(int M, int heads, const uint16_t* norm_q, const uint16_t* norm_k, float eps,
                               const float* cos_t, const float* sin_t, uint16_t* y, void* stream);

/* awq_pack_weight — round-to-nearest asymmetric INT4 pack of W [K, N] with one
 * bf16 (scale, zero point) per output column and 64-block of K (Diffusers
 * "Nunchaku Lite" page, table "Supported quantization types", awq_w4a16):
 *   s = bf16((max-min)/15) (1 if 0); z = clamp(rne(-min/s), 0, 15);
 *   q = clamp(rne(w/s) + z, 0, 15)
 * Out: q u8 [N, K/2] (unsigned nibbles); scales bf16 [N, K/64];
 *      zeros bf16 [N, K/64] (integers 0..15).
 * Shapes: K % 64 == 0, N % 8 == 0. */
svdq_status awq_pack_weight(int K, int N, const float* W, uint8_t* q, uint16_t* scales,
                            uint16_t* zeros, void* stream);

/* awq_w4a16_linear — INT4 weight x bf16 activation linear for the memory-bound
 * modulation projections (blog, section "Introducing Nunchaku Lite"):
 *   y[m,n] = bf16( sum_g s[n,g] sum_{k in g} x[m,k] (q[n,k] - z[n,g]) + bias[n] )
 * In:  x bf16 [M, K]; q, scales, zeros from awq_pack_weight; bias bf16 [N] or NULL.
 * Out: y bf16 [M, N].
 * Shapes: K % 64 == 0, K <= 16384 (the activations of a block of rows are
 * held in shared memory), N % 8 == 0, M >= 0.
 * M = 1..4 runs the GEMV kernel (M = 3, 4 only while its shared-memory plan
 * fits K; otherwise the batched kernel): each group's dot product is formed with
 * exact products in fp32 (the activations scaled into fp16 by a power of two
 * per group and row, the weight nibbles as exact fp16 values) and the zero
 * point applied once per group through the activation group sum; larger M runs
 * the batched kernel, which subtracts the zero point before its MMAs. Both
 * meet the same output tolerance; they may differ from each other in the
 * last bits of the fp32 sums (summation order).
 * Launched with programmatic dependent launch: the kernel may be scheduled
 * while the previous kernel in the stream finishes, but it reads none of its
 * inputs (x, q, scales, zeros, bias) before that kernel has completed, so any
 * of them may be that kernel's output (e.g. awq_pack_weight into the same
 * buffers just before). */
svdq_status awq_w4a16_linear(int M, int K, int N, const uint16_t* x, const uint8_t* q,
                             const uint16_t* scales, const uint16_t* zeros, const uint16_t* bias,
                             uint16_t* y, void* stream);

/* Reads and clears the device error word of the current device: bit 0 = a
 * bounded wait ran out, bit 1 = a kernel saw an inconsistent launch. The
 * caller synchronises the stream first. Returns SVDQ_ERR_TIMEOUT if bit 0 was
 * set, SVDQ_ERR_CUDA if bit 1 was set or the read failed, else SVDQ_OK;
 * `bits` (nullable) receives the raw word. */
svdq_status svdq_device_error(unsigned* bits);

/* Limit, in nanoseconds, of every bounded device-side wait (default 2e9). */
void svdq_set_wait_limit_ns(unsigned long long ns);

/* Diagnostics ------------------------------------------------------------- */

/* Applies the device conversions the kernels use to n fp32 values:
 * e2m1[i] = E2M1 code of in[i] (round to nearest even, saturating; low nibble),
 * e4m3[i] = E4M3 code (round to nearest even, saturating),
 * bf16[i] = bf16 bits (round to nearest even). Any output may be NULL.
 * Used to pin the device conversions against the CPU oracle on every fp32 value. */
svdq_status svdq_probe_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3,
                               uint16_t* bf16, void* stream);

/* Launches one CTA that waits on a barrier nothing arrives at, for at most
 * `limit_ns`; it must set the timeout bit of the device error word and exit.
 * Exercises the bounded-wait path without hanging the GPU. */
svdq_status svdq_probe_wait_timeout(unsigned long long limit_ns, void* stream);

/* Tensor-core rate probe (the measured denominator of the GEMM's roofline):
 * every CTA pair of the device (one pair per two SMs) issues `iters` K stages
 * of 4 block-scaled NVFP4 MMAs (tcgen05.mma.cta_group::2.kind::mxf4nvf4,
 * 256 x 256 x 64 each, the GEMM's instruction) on operands that stay in
 * shared memory: no loads, no epilogue. mode 1 also issues 12 scale copies
 * (tcgen05.cp) per stage; modes 2 and 3 issue the same work as N = 128 or
 * N = 64 MMAs (mode 4: the N = 128 MMAs of each half back to back into one
 * accumulator). The caller times the launch; the work is
 * (SMs/2) * iters * 4 * 2*256*256*64 FLOP. 1 <= iters <= 2^20, 0 <= mode <= 4. */
svdq_status svdq_probe_mma_peak(int iters, int mode, void* stream);

/* Test hook: pretend the device has compute capability major.minor (0, 0
 * restores the real query), to exercise SVDQ_ERR_UNSUPPORTED_ARCH. */
void svdq_debug_force_arch(int major, int minor);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
