// Per-head RMSNorm and rotary embedding of the Q and K sections of a grouped
// Q/K/V projection's bf16 output, in place (Diffusers "Nunchaku Lite" page,
// section on fused kernels: the RMSNorm and RoPE that follow the QKV
// projection). This is the separate pass that svdq_w4a4_linear_qkv fuses into
// the GEMM's epilogue; it reads the layer's rounded bf16 output.
//
// One CTA of 8 warps per row. A lane holds 4 consecutive columns of a head
// (two rotary pairs): the same pair positions in every head, so each warp
// loads the row's cos/sin for its lane's two pairs and the lane's norm
// weights once, then takes the heads warp, warp + 8, ... (all their loads in
// flight at once). The sum of squares is a warp-shuffle reduction. Bound by
// HBM: the Q and K sections are read and written once.
//
// Also here: the pack of the cos/sin tables into the 32-row-block layout that
// the fused epilogue reads (svdq_rope_pack).
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kWarpsNR = 8;
constexpr int kHPW = 6;  // heads per warp in flight (48 Q/K heads per row at 24 heads per section)

__global__ void __launch_bounds__(kWarpsNR * 32)
norm_rope_kernel(NormRopeArgs a) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int m = blockIdx.x;
  const int hq = 2 * a.heads;  // Q and K heads of the row
  uint16_t* rowp = a.y + (size_t)m * (size_t)(3 * a.heads * 128) + 4 * lane;
  const float2 cs = __ldg(reinterpret_cast<const float2*>(a.cos_t + (size_t)m * 64 + 2 * lane));
  const float2 sn = __ldg(reinterpret_cast<const float2*>(a.sin_t + (size_t)m * 64 + 2 * lane));
  const uint2 wq = __ldg(reinterpret_cast<const uint2*>(a.norm_q + 4 * lane));
  const uint2 wk = __ldg(reinterpret_cast<const uint2*>(a.norm_k + 4 * lane));
  for (int h0 = warp; h0 < hq; h0 += kWarpsNR * kHPW) {
    uint2 raw[kHPW];
#pragma unroll
    for (int k = 0; k < kHPW; ++k) {
      const int hd = h0 + kWarpsNR * k;
      raw[k] = hd < hq ? *reinterpret_cast<const uint2*>(rowp + (size_t)hd * 128) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kHPW; ++k) {
      const int hd = h0 + kWarpsNR * k;
      const float v0 = bf16_bits_to_f32(raw[k].x & 0xFFFFu), v1 = bf16_bits_to_f32(raw[k].x >> 16);
      const float v2 = bf16_bits_to_f32(raw[k].y & 0xFFFFu), v3 = bf16_bits_to_f32(raw[k].y >> 16);
      float ss = v0 * v0 + v1 * v1 + v2 * v2 + v3 * v3;
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (hd >= hq) continue;
      const float inv = rsqrtf(fmaf(ss, 1.0f / 128.0f, a.eps));
      const uint2 wr = hd < a.heads ? wq : wk;
      const float u0 = v0 * inv * bf16_bits_to_f32(wr.x & 0xFFFFu), u1 = v1 * inv * bf16_bits_to_f32(wr.x >> 16);
      const float u2 = v2 * inv * bf16_bits_to_f32(wr.y & 0xFFFFu), u3 = v3 * inv * bf16_bits_to_f32(wr.y >> 16);
      const float o0 = fmaf(u0, cs.x, -u1 * sn.x), o1 = fmaf(u0, sn.x, u1 * cs.x);
      const float o2 = fmaf(u2, cs.y, -u3 * sn.y), o3 = fmaf(u2, sn.y, u3 * cs.y);
      *reinterpret_cast<uint2*>(rowp + (size_t)hd * 128) =
          make_uint2(f32_to_bf16_bits(o0) | (f32_to_bf16_bits(o1) << 16),
                     f32_to_bf16_bits(o2) | (f32_to_bf16_bits(o3) << 16));
    }
  }
}

// The packed rotary table: one CTA per 32-row block, thread (row lane,
// group g) moves the cos and sin of pairs 4g .. 4g + 3 of its row (zero for
// rows past M). The writes of a group are 512 contiguous bytes per table.
__global__ void __launch_bounds__(512) rope_pack_kernel(int M, const float* __restrict__ cos_t,
                                                        const float* __restrict__ sin_t, float* __restrict__ rope) {
  const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int blk = blockIdx.x, m = blk * 32 + lane;
  float4 c = make_float4(0.f, 0.f, 0.f, 0.f), sn = c;
  if (m < M) {
    c = __ldg(reinterpret_cast<const float4*>(cos_t + (size_t)m * 64 + 4 * g));
    sn = __ldg(reinterpret_cast<const float4*>(sin_t + (size_t)m * 64 + 4 * g));
  }
  float* dst = rope + ((size_t)blk * 16 + g) * 256 + 4 * lane;
  *reinterpret_cast<float4*>(dst) = c;
  *reinterpret_cast<float4*>(dst + 128) = sn;
}

}  // namespace

cudaError_t launch_norm_rope(const NormRopeArgs& a, cudaStream_t s) {
  norm_rope_kernel<<<(unsigned)a.M, kWarpsNR * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rope_pack(int M, const float* cos_t, const float* sin_t, float* rope, cudaStream_t s) {
  rope_pack_kernel<<<(unsigned)((M + 31) / 32), 512, 0, s>>>(M, cos_t, sin_t, rope);
  return cudaGetLastError();
}

}  // namespace svdq
