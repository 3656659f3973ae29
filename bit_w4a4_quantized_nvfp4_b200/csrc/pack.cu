// Offline weight packing: svdq_pack_weight (NVFP4 / INT4 residual with the
// low-rank branch removed) and awq_pack_weight (asymmetric INT4, g64).
//
// svdq residual (blog "Introducing Nunchaku 4-bit inference in Diffusers",
// section "Background: SVDQuant and Nunchaku"): the smoothed weight
// lambda*W keeps its dominant part as the 16-bit low-rank branch L1 L2; the
// residual R = lambda*W - L1 L2 is what gets 4 bits. R is recomputed where it
// is needed (amax pass, quantise pass) instead of being stored, so packing
// needs no buffer beyond its outputs.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

// R[k,n] = fp32( fp32(lambda[k]*W[k,n]) - sum_j L1[k,j] L2[j,n] ), the sum in
// fp64 with j ascending (each product of two bf16 values is exact).
__device__ __forceinline__ float residual(const PackArgs& a, int k, int n) {
  const float what = __fmul_rn(a.lambda[k], a.W[(size_t)k * a.N + n]);
  double lr = 0.0;
  for (int j = 0; j < a.r; ++j)
    lr = fma((double)bf16_bits_to_f32(a.L1[(size_t)k * a.r + j]),
             (double)bf16_bits_to_f32(a.L2[(size_t)j * a.N + n]), lr);
  return __double2float_rn((double)what - lr);
}

__global__ void residual_amax_kernel(PackArgs a) {
  const size_t total = (size_t)a.K * a.N;
  float m = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(i / a.N), n = (int)(i % a.N);
    m = fmaxf(m, fabsf(residual(a, k, n)));
    if (n == 0) a.inv_lambda[k] = __frcp_rn(a.lambda[k]);
  }
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned*>(a.tensor_scale), __float_as_uint(m));
}

__global__ void finalize_kernel(PackArgs a, int prec) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (prec == 0) {
    const float amax = a.tensor_scale[0];
    const float t = __fdiv_rn(amax, 2688.0f);  // 6 * 448
    a.tensor_scale[0] = (t == 0.f) ? 1.0f : t;
    a.tensor_scale[1] = a.s_tx;
  } else {
    a.tensor_scale[0] = 1.0f;
    a.tensor_scale[1] = 1.0f;
  }
}

// One thread per (n, 16-block of k).
__global__ void quant_w_nvfp4_kernel(PackArgs a) {
  const int nb = a.K / 16;
  const size_t total = (size_t)a.N * nb;
  const float t = a.tensor_scale[0];
  const float six_t = __fmul_rn(6.0f, t);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % a.N), b = (int)(i / a.N);
    float v[16];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      v[e] = residual(a, b * 16 + e, n);
      amax = fmaxf(amax, fabsf(v[e]));
    }
    const uint32_t sf = cvt_e4m3(__fdiv_rn(amax, six_t));
    const float d = __fmul_rn(e4m3_to_f32(sf), t);
    uint32_t c0 = 0, c1 = 0;
    if (d != 0.f) {
      const float inv = __frcp_rn(d);
      float q0[8], q1[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        q0[e] = __fmul_rn(v[e], inv);
        q1[e] = __fmul_rn(v[8 + e], inv);
      }
      c0 = cvt_e2m1x8(q0);
      c1 = cvt_e2m1x8(q1);
    }
    *reinterpret_cast<uint2*>(a.codes + (size_t)n * (a.K / 2) + b * 8) = make_uint2(c0, c1);
    const size_t atom = ((size_t)(n / 128) * (a.K / 64) + b / 4) * 512;
    static_cast<uint8_t*>(a.scales)[atom + 16 * (n % 32) + 4 * ((n % 128) / 32) + (b % 4)] = (uint8_t)sf;
  }
}

// One thread per (n, 64-block of k).
__global__ void quant_w_int4_kernel(PackArgs a) {
  const int nb = a.K / 64;
  const size_t total = (size_t)a.N * nb;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % a.N), b = (int)(i / a.N);
    float v[64];
    float amax = 0.f;
    for (int e = 0; e < 64; ++e) {
      v[e] = residual(a, b * 64 + e, n);
      amax = fmaxf(amax, fabsf(v[e]));
    }
    const uint32_t sb = f32_to_bf16_bits(__fdiv_rn(amax, 7.0f));
    const float sfv = bf16_bits_to_f32(sb);
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (sfv != 0.f) {
      const float inv = __frcp_rn(sfv);
      for (int e = 0; e < 64; ++e) {
        int q = __float2int_rn(__fmul_rn(v[e], inv));
        q = max(-8, min(7, q));
        w[e / 8] |= ((uint32_t)q & 0xFu) << (4 * (e % 8));
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(a.codes + (size_t)n * (a.K / 2) + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    static_cast<uint16_t*>(a.scales)[(size_t)b * a.N + n] = (uint16_t)sb;  // group-major [K/64, N]
  }
}

// lr_up: NVFP4 -> bf16 hi/lo split of L2 / (s_tw * s_tx), K-major [N, 2r];
//        INT4  -> L2 transposed [N, r].
__global__ void lr_up_kernel(PackArgs a, int prec) {
  const size_t total = (size_t)a.N * a.r;
  const float alpha = __fmul_rn(a.tensor_scale[0], a.tensor_scale[1]);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % a.N), j = (int)(i / a.N);
    const uint16_t l2 = a.L2[(size_t)j * a.N + n];
    if (prec == 0) {
      const float v = __fdiv_rn(bf16_bits_to_f32(l2), alpha);
      const uint32_t hi = f32_to_bf16_bits(v);
      const uint32_t lo = f32_to_bf16_bits(__fsub_rn(v, bf16_bits_to_f32(hi)));
      a.lr_up[(size_t)n * 2 * a.r + j] = (uint16_t)hi;
      a.lr_up[(size_t)n * 2 * a.r + a.r + j] = (uint16_t)lo;
    } else {
      a.lr_up[(size_t)n * a.r + j] = l2;
    }
  }
}

// AWQ: one thread per (n, 64-group).
__global__ void awq_pack_kernel(AwqPackArgs a) {
  const int ng = a.K / 64;
  const size_t total = (size_t)a.N * ng;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % a.N), g = (int)(i / a.N);
    const float* col = a.W + (size_t)(g * 64) * a.N + n;
    float mn = col[0], mx = col[0];
    for (int e = 1; e < 64; ++e) {
      const float w = col[(size_t)e * a.N];
      mn = fminf(mn, w);
      mx = fmaxf(mx, w);
    }
    uint32_t sb = f32_to_bf16_bits(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
    if (bf16_bits_to_f32(sb) == 0.f) sb = 0x3F80u;
    const float inv = __frcp_rn(bf16_bits_to_f32(sb));
    int z = __float2int_rn(__fmul_rn(-mn, inv));
    z = max(0, min(15, z));
    uint32_t w8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int e = 0; e < 64; ++e) {
      int q = __float2int_rn(__fmul_rn(col[(size_t)e * a.N], inv)) + z;
      q = max(0, min(15, q));
      w8[e / 8] |= (uint32_t)q << (4 * (e % 8));
    }
    uint4* dst = reinterpret_cast<uint4*>(a.q + (size_t)n * (a.K / 2) + g * 32);
    dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
    dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
    a.s[(size_t)n * ng + g] = (uint16_t)sb;
    a.z[(size_t)n * ng + g] = (uint16_t)f32_to_bf16_bits((float)z);
  }
}

int grid_for(size_t total, int block) {
  size_t g = (total + block - 1) / block;
  if (g > 148 * 32) g = 148 * 32;
  return (int)(g ? g : 1);
}

}  // namespace

cudaError_t launch_pack(int prec, const PackArgs& a, size_t scale_bytes, cudaStream_t s) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.tensor_scale, 0, 2 * sizeof(float), s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.scales, 0, scale_bytes, s)) != cudaSuccess) return e;
  const size_t kn = (size_t)a.K * a.N;
  residual_amax_kernel<<<grid_for(kn, 256), 256, 0, s>>>(a);
  finalize_kernel<<<1, 32, 0, s>>>(a, prec);
  if (prec == 0)
    quant_w_nvfp4_kernel<<<grid_for((size_t)a.N * (a.K / 16), 128), 128, 0, s>>>(a);
  else
    quant_w_int4_kernel<<<grid_for((size_t)a.N * (a.K / 64), 128), 128, 0, s>>>(a);
  if (a.r > 0) lr_up_kernel<<<grid_for((size_t)a.N * a.r, 256), 256, 0, s>>>(a, prec);
  return cudaGetLastError();
}

cudaError_t launch_awq_pack(const AwqPackArgs& a, cudaStream_t s) {
  awq_pack_kernel<<<grid_for((size_t)a.N * (a.K / 64), 128), 128, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace svdq
