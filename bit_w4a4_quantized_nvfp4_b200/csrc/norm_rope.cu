// Per-head RMSNorm and rotary embedding of the Q and K sections of a grouped
// Q/K/V projection's bf16 output, in place (Diffusers "Nunchaku Lite" page,
// section on fused kernels: the RMSNorm and RoPE that follow the QKV
// projection). This is the separate pass that svdq_w4a4_linear_qkv fuses into
// the GEMM's epilogue; it reads the layer's rounded bf16 output.
//
// One warp per (row, head) of 128 columns: each lane holds 4 consecutive
// columns (two rotary pairs), the sum of squares is a warp-shuffle reduction,
// and the row's cos/sin values of the lane's two pairs are one 8-byte load
// each. Bound by HBM: the Q and K sections are read and written once.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kWarpsNR = 8;

__global__ void __launch_bounds__(kWarpsNR * 32)
norm_rope_kernel(NormRopeArgs a) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * kWarpsNR + (threadIdx.x >> 5);  // (row, head of Q or K)
  const int hq = 2 * a.heads;
  if (task >= (long long)a.M * hq) return;
  const int m = (int)(task / hq), hd = (int)(task % hq);
  const uint16_t* w = hd < a.heads ? a.norm_q : a.norm_k;
  uint16_t* row = a.y + (size_t)m * (size_t)(3 * a.heads * 128) + (size_t)hd * 128 + 4 * lane;
  const uint2 raw = *reinterpret_cast<const uint2*>(row);
  float v[4] = {bf16_bits_to_f32(raw.x & 0xFFFFu), bf16_bits_to_f32(raw.x >> 16), bf16_bits_to_f32(raw.y & 0xFFFFu),
                bf16_bits_to_f32(raw.y >> 16)};
  float ss = v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3];
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(fmaf(ss, 1.0f / 128.0f, a.eps));
  const uint2 wr = __ldg(reinterpret_cast<const uint2*>(w + 4 * lane));
  const float wv[4] = {bf16_bits_to_f32(wr.x & 0xFFFFu), bf16_bits_to_f32(wr.x >> 16), bf16_bits_to_f32(wr.y & 0xFFFFu),
                       bf16_bits_to_f32(wr.y >> 16)};
  const float2 cs = __ldg(reinterpret_cast<const float2*>(a.cos_t + (size_t)m * 64 + 2 * lane));
  const float2 sn = __ldg(reinterpret_cast<const float2*>(a.sin_t + (size_t)m * 64 + 2 * lane));
  float u[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) u[k] = v[k] * inv * wv[k];
  const float o0 = fmaf(u[0], cs.x, -u[1] * sn.x), o1 = fmaf(u[0], sn.x, u[1] * cs.x);
  const float o2 = fmaf(u[2], cs.y, -u[3] * sn.y), o3 = fmaf(u[2], sn.y, u[3] * cs.y);
  *reinterpret_cast<uint2*>(row) = make_uint2(f32_to_bf16_bits(o0) | (f32_to_bf16_bits(o1) << 16),
                                              f32_to_bf16_bits(o2) | (f32_to_bf16_bits(o3) << 16));
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s) {
  const long long tasks = (long long)a.M * 2 * a.heads;
  const long long blocks = (tasks + kWarpsNR - 1) / kWarpsNR;
  norm_rope_kernel<<<(unsigned)blocks, kWarpsNR * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace svdq
