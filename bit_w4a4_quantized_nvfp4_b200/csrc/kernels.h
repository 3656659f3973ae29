// Launch interfaces of the library's kernels (host side of csrc/*.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace svdq {

struct QuantActArgs {
  const uint16_t* x;          // bf16 [M, K]
  const float* inv_lambda;    // [K]
  const uint16_t* L1;         // bf16 [K, r]
  uint8_t* codes;             // [M, K/2]
  void* scales;               // NVFP4 tiled e4m3 / INT4 bf16 [M, K/64]
  uint16_t* P;                // bf16 [M, r]
  int M, K, r;
  const float* tensor_scale;  // NVFP4: [2] = {s_tw, s_tx} (s_tx read on the device); INT4: unused
};
cudaError_t launch_quant_act(int prec, const QuantActArgs& a, unsigned* err, unsigned long long wait_ns,
                             cudaStream_t s);

struct PackArgs {
  const float* W;             // [K, N]
  const float* lambda;        // [K]
  const uint16_t* L1;         // [K, r]
  const uint16_t* L2;         // [r, N]
  uint8_t* codes;             // [N, K/2]
  void* scales;
  float* tensor_scale;        // [2]
  float* inv_lambda;          // [K]
  uint16_t* lr_up;            // [N, rr]
  int K, N, r;
  float s_tx;
};
cudaError_t launch_pack(int prec, const PackArgs& a, size_t scale_bytes, cudaStream_t s);

struct AwqPackArgs {
  const float* W;
  uint8_t* q;
  uint16_t* s;
  uint16_t* z;
  int K, N;
};
cudaError_t launch_awq_pack(const AwqPackArgs& a, cudaStream_t s);

struct AwqArgs {
  const uint16_t* x;
  const uint8_t* q;
  const uint16_t* s;
  const uint16_t* z;
  const uint16_t* bias;
  uint16_t* y;
  int M, K, N;
};
cudaError_t launch_awq(const AwqArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s);
// M = 1..4: the GEMV kernel (awq_gemv.cu), when awq_gemv_fits(M, K);
// launch_awq dispatches to it
bool awq_gemv_fits(int M, int K);
cudaError_t launch_awq_gemv(const AwqArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s);

// Row pitch, in scales, of the INT4 activation scales [M, K/64]: padded to a
// multiple of 8 so that every row starts on a 16-byte boundary (the GEMM
// reads them with TMA).
__host__ __device__ inline int int4_act_scale_pitch(int K) { return ((K / 64 + 7) / 8) * 8; }

struct GemmArgs {
  const uint8_t* x_codes;
  const void* x_scales;
  const uint16_t* P;
  const uint8_t* w_codes;
  const void* w_scales;
  const float* tensor_scale;  // [2] = {s_tw, s_tx}
  const uint16_t* lr_up;
  const uint16_t* bias;
  void* y;
  int M, K, N, r;
  int out;                    // svdq_out_dtype
  unsigned* err;
  unsigned long long wait_ns;
  int num_sms;
  // NVFP4 only: fused QKV epilogue when qkv_heads > 0 (head_dim 128)
  int qkv_heads = 0;
  const uint16_t* norm_q = nullptr;
  const uint16_t* norm_k = nullptr;
  float eps = 0.f;
  const float* rope = nullptr;  // cos/sin packed by svdq_rope_pack
};
cudaError_t launch_gemm_nvfp4(const GemmArgs& a, cudaStream_t s);
cudaError_t launch_gemm_int4(const GemmArgs& a, cudaStream_t s);

struct NormRopeArgs {
  uint16_t* y;                // bf16 [M, 3 * heads * 128], Q and K sections updated in place
  const uint16_t* norm_q;     // bf16 [128]
  const uint16_t* norm_k;     // bf16 [128]
  const float* cos_t;         // [M, 64]
  const float* sin_t;         // [M, 64]
  int M, heads;
  float eps;
};
cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s);

// cos/sin [M, 64] -> the packed rotary table (16384 * ceil(M / 32) bytes)
cudaError_t launch_rope_pack(int M, const float* cos_t, const float* sin_t, float* rope, cudaStream_t s);

cudaError_t launch_probe_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3,
                                 uint16_t* bf16, cudaStream_t s);
cudaError_t launch_probe_wait(unsigned* err, unsigned long long limit_ns, cudaStream_t s);
cudaError_t launch_probe_mma(int iters, int mode, int num_sms, unsigned* err, unsigned long long wait_ns,
                             cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device. The attribute is set once per (kernel, device, size): the
// calls on the hot path then cost a table lookup.
cudaError_t ensure_smem(const void* func, int bytes);

// Host helper: encode a 2-D tiled tensor map (driver entry point looked up at
// run time; no link-time dependency on libcuda). Encodings are cached by
// their full argument list, so a layer called again on the same buffers
// reuses its maps.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swz);
// 3-D tiled tensor map without swizzle: dims {d0, d1, d2}, byte strides of
// dims 1 and 2, box {b0, b1, b2}.
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2);

}  // namespace svdq
