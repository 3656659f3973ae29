// K1 — the fused activation pass of the SVDQuant W4A4 layer.
//
// One coalesced, vectorised pass over x computes, for every row:
//   x_hat = bf16(x * inv_lambda)                       (smoothing)
//   4-bit codes and group scales of x_hat              (NVFP4 g16 / INT4 g64)
//   P = bf16(x_hat L1)                                  (low-rank down-projection)
// so that the 16-bit branch costs no extra pass over the activations
// (blog "Introducing Nunchaku 4-bit inference in Diffusers", section
// "Background: SVDQuant and Nunchaku", figure caption).
//
// Work split: a CTA owns 32 rows and walks K in chunks of 256 columns. Each of
// its 8 warps quantises 4 rows; lane l handles 8 consecutive columns of a row
// (one 16-byte load), so a warp reads a 512-byte row segment per load and
// writes 128 contiguous bytes of codes. x_hat is staged in shared memory and
// multiplied by the L1 chunk on tensor cores (mma.sync bf16, fp32 accumulate);
// the 8 warps split the chunk 2 (row tiles) x 4 (K quarters) and the K
// quarters are summed in a fixed order at the end.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRows = 32;     // rows per CTA
constexpr int kChunk = 256;   // K columns per step
constexpr int kXhStride = kChunk + 8;  // bf16 elements per staged row (bank spread)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// PREC 0 = NVFP4 (group 16, E4M3 scales in the tiled layout), 1 = INT4
// (group 64, bf16 scales row-major). NT = r / 8 tiles of the P output.
template <int PREC, int NT>
__global__ void __launch_bounds__(256) quant_act_kernel(QuantActArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* xh = reinterpret_cast<__nv_bfloat16*>(smem);                 // [32][264]
  constexpr int kR = NT * 8;
  constexpr int kL1Stride = kR + 8;
  __nv_bfloat16* l1s = xh + kRows * kXhStride;                                // [256][r+8]
  float* red = reinterpret_cast<float*>(l1s + (NT ? kChunk * kL1Stride : 0));  // [4][32][r]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int M = a.M, K = a.K;
  const int nchunks = (K + kChunk - 1) / kChunk;
  const float s_tx = a.s_tx;
  const float six_t = __fmul_rn(6.0f, s_tx);

  float acc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int t = 0; t < (NT > 0 ? NT : 1); ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  // prefetch chunk 0
  uint4 xv[4];
  auto load_chunk = [&](int c, uint4 (&v)[4]) {
    const int col = c * kChunk + lane * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = row0 + warp + 8 * i;
      if (m < M && col < K)
        v[i] = ldg_stream(a.x + (size_t)m * K + col);
      else
        v[i] = make_uint4(0, 0, 0, 0);
    }
  };
  load_chunk(0, xv);

  for (int c = 0; c < nchunks; ++c) {
    const int col = c * kChunk + lane * 8;
    const bool col_ok = col < K;
    uint4 cur[4] = {xv[0], xv[1], xv[2], xv[3]};
    if (c + 1 < nchunks) load_chunk(c + 1, xv);

    // stage the L1 chunk [256 x r] (rows beyond K are zero)
    if constexpr (NT > 0) {
      constexpr int kVecPerRow = kR / 8;  // 16-byte vectors per L1 row
      for (int v = threadIdx.x; v < kChunk * kVecPerRow; v += blockDim.x) {
        const int kr = v / kVecPerRow, cv = v % kVecPerRow;
        const int kg = c * kChunk + kr;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (kg < K) val = *reinterpret_cast<const uint4*>(a.L1 + (size_t)kg * kR + cv * 8);
        *reinterpret_cast<uint4*>(l1s + kr * kL1Stride + cv * 8) = val;
      }
    }

    float il[8];
    if (col_ok) {
      const float4 i0 = *reinterpret_cast<const float4*>(a.inv_lambda + col);
      const float4 i1 = *reinterpret_cast<const float4*>(a.inv_lambda + col + 4);
      il[0] = i0.x; il[1] = i0.y; il[2] = i0.z; il[3] = i0.w;
      il[4] = i1.x; il[5] = i1.y; il[6] = i1.z; il[7] = i1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) il[j] = 0.f;
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int lr = warp + 8 * i;  // local row
      const int m = row0 + lr;
      const uint32_t w[4] = {cur[i].x, cur[i].y, cur[i].z, cur[i].w};
      float xf[8];
      uint32_t hb[4];
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float x0 = bf16_bits_to_f32(w[j] & 0xFFFFu), x1 = bf16_bits_to_f32(w[j] >> 16);
        const uint32_t h0 = f32_to_bf16_bits(__fmul_rn(x0, il[2 * j]));
        const uint32_t h1 = f32_to_bf16_bits(__fmul_rn(x1, il[2 * j + 1]));
        hb[j] = h0 | (h1 << 16);
        xf[2 * j] = bf16_bits_to_f32(h0);
        xf[2 * j + 1] = bf16_bits_to_f32(h1);
        amax = fmaxf(amax, fmaxf(fabsf(xf[2 * j]), fabsf(xf[2 * j + 1])));
      }
      *reinterpret_cast<uint4*>(xh + lr * kXhStride + lane * 8) = make_uint4(hb[0], hb[1], hb[2], hb[3]);

      if (PREC == 0) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        const uint32_t sf = cvt_e4m3(__fdiv_rn(amax, six_t));
        const float d = __fmul_rn(e4m3_to_f32(sf), s_tx);
        uint32_t code = 0;
        if (d != 0.f) {
          const float inv = __frcp_rn(d);
          float q[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) q[j] = __fmul_rn(xf[j], inv);
          code = cvt_e2m1x8(q);
        }
        // gather the 4 scales of one 64-column atom (lanes 8a, 8a+2, 8a+4, 8a+6)
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, sf, 2);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, sf, 4);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, sf, 6);
        if (m < M && col_ok) {
          *reinterpret_cast<uint32_t*>(a.codes + (size_t)m * (K / 2) + col / 2) = code;
          if ((lane & 7) == 0) {
            const int ka = (c * kChunk + lane * 8) / 64;  // atom index along K
            const size_t atom = ((size_t)(m / 128) * (K / 64) + ka) * 512;
            const uint32_t word = sf | (s1 << 8) | (s2 << 16) | (s3 << 24);
            *reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.scales) + atom + 16 * (m % 32) +
                                         4 * ((m % 128) / 32)) = word;
          }
        }
      } else {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const uint32_t sb = f32_to_bf16_bits(__fdiv_rn(amax, 7.0f));
        const float sfv = bf16_bits_to_f32(sb);
        uint32_t code = 0;
        if (sfv != 0.f) {
          const float inv = __frcp_rn(sfv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            int q = __float2int_rn(__fmul_rn(xf[j], inv));
            q = max(-8, min(7, q));
            code |= ((uint32_t)q & 0xFu) << (4 * j);
          }
        }
        if (m < M && col_ok) {
          *reinterpret_cast<uint32_t*>(a.codes + (size_t)m * (K / 2) + col / 2) = code;
          if ((lane & 7) == 0)
            static_cast<uint16_t*>(a.scales)[(size_t)m * (K / 64) + col / 64] = (uint16_t)sb;
        }
      }
    }
    __syncthreads();

    if constexpr (NT > 0) {
      // tensor-core partial products: warp -> (row tile, K quarter)
      const int mt = warp & 1, kq = warp >> 1;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int k0 = (kq * 4 + s) * 16;
        uint32_t a0, a1, a2, a3;
        const int ar = mt * 16 + (lane & 15), ac = k0 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(xh + ar * kXhStride + ac), a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < NT; t += 2) {
          uint32_t b0, b1, b2, b3;
          const int br = k0 + (lane & 7) + ((lane >> 3) & 1) * 8, bc = t * 8 + (lane >> 4) * 8;
          ldsm_x4_t(smem_u32(l1s + br * kL1Stride + bc), b0, b1, b2, b3);
          mma_16816(acc[t], a0, a1, a2, a3, b0, b1);
          mma_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();
  }

  if constexpr (NT > 0) {
    // fixed-order reduction of the four K quarters, then one bf16 rounding
    const int mt = warp & 1, kq = warp >> 1;
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int j = t * 8 + 2 * t4;
      float* base = red + (size_t)kq * kRows * kR;
      base[(mt * 16 + g) * kR + j] = acc[t][0];
      base[(mt * 16 + g) * kR + j + 1] = acc[t][1];
      base[(mt * 16 + g + 8) * kR + j] = acc[t][2];
      base[(mt * 16 + g + 8) * kR + j + 1] = acc[t][3];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kRows * kR; e += blockDim.x) {
      const int lr = e / kR, j = e % kR;
      const int m = row0 + lr;
      if (m >= M) continue;
      float v = red[e];
      v += red[kRows * kR + e];
      v += red[2 * kRows * kR + e];
      v += red[3 * kRows * kR + e];
      a.P[(size_t)m * kR + j] = (uint16_t)f32_to_bf16_bits(v);
    }
  }
}

template <int PREC, int NT>
cudaError_t launch_t(const QuantActArgs& a, cudaStream_t s) {
  constexpr int kR = NT * 8;
  const size_t smem = (size_t)kRows * kXhStride * 2 + (NT ? (size_t)kChunk * (kR + 8) * 2 : 0) +
                      (size_t)4 * kRows * kR * 4;
  auto k = quant_act_kernel<PREC, NT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (a.M + kRows - 1) / kRows;
  k<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_act(int prec, const QuantActArgs& a, cudaStream_t s) {
  const int nt = a.r / 8;
  if (prec == 0) {
    switch (nt) {
      case 0: return launch_t<0, 0>(a, s);
      case 2: return launch_t<0, 2>(a, s);
      case 4: return launch_t<0, 4>(a, s);
    }
  } else {
    switch (nt) {
      case 0: return launch_t<1, 0>(a, s);
      case 2: return launch_t<1, 2>(a, s);
      case 4: return launch_t<1, 4>(a, s);
      case 6: return launch_t<1, 6>(a, s);
      case 8: return launch_t<1, 8>(a, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace svdq
