// K1 — the fused activation pass of the SVDQuant W4A4 layer.
//
// One coalesced pass over x computes, for every row:
//   x_hat = bf16(x * inv_lambda)                       (smoothing)
//   4-bit codes and group scales of x_hat              (NVFP4 g16 / INT4 g64)
//   P = bf16(x_hat L1)                                  (low-rank down-projection)
// so that the 16-bit branch costs no extra pass over the activations
// (blog "Introducing Nunchaku 4-bit inference in Diffusers", section
// "Background: SVDQuant and Nunchaku", figure caption).
//
// Work split: a CTA owns 32 rows and walks K in chunks of 256 columns through
// a multi-stage TMA pipeline (each stage: the 32 x 256 x tile and the matching
// 256 x r L1 tile, the latter with the TMA swizzle that makes the ldmatrix
// reads below bank-conflict free), so that several chunks are in flight per SM.
// Each of the 16 warps quantises 2 rows; lane l handles 8 consecutive columns
// of a row, so a warp writes 128 contiguous bytes of codes per row. x_hat is
// staged in shared memory and multiplied by the L1 tile on tensor cores
// (mma.sync bf16, fp32 accumulate); the warps split each chunk 2 (row tiles) x
// 8 (K eighths) and the eighths are summed in a fixed order at the end.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRows = 32;              // rows per CTA
constexpr int kChunk = 256;            // K columns per stage
constexpr int kXhStride = kChunk + 8;  // bf16 elements per staged x_hat row (bank spread)
constexpr int kXBytes = kRows * kChunk * 2;
constexpr int kThreadsQA = 512;
constexpr int kWarpsQA = kThreadsQA / 32;
constexpr int kRowsPerWarp = kRows / kWarpsQA;    // 2
constexpr int kKParts = kWarpsQA / 2;             // K splits of a chunk for the P product

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

// two fp32 -> bf16x2 (round to nearest even); `lo` in bits 0..15
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int NT>
struct StageLayout {
  static constexpr int kR = NT * 8;
  static constexpr int kL1Bytes = NT ? kChunk * kR * 2 : 0;
  static constexpr int kIlBytes = kChunk * 4;  // the chunk's inv_lambda
  static constexpr int kStageBytes = ((kXBytes + kL1Bytes + kIlBytes + 1023) / 1024) * 1024;
  static constexpr int kStages = (kR <= 32) ? 4 : 3;
  // L1 tile rows are 2r bytes; the TMA swizzle span equals the row (32/64/128 B)
  static constexpr uint32_t kSwzMask = kR <= 16 ? 1u : (kR == 32 ? 3u : 7u);
};

// PREC 0 = NVFP4 (group 16, E4M3 scales in the tiled layout), 1 = INT4
// (group 64, bf16 scales row-major). NT = r / 8 tiles of the P output.
template <int PREC, int NT>
__global__ void __launch_bounds__(kThreadsQA, 1)
quant_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
                 QuantActArgs a, unsigned* err, unsigned long long wait_ns) {
  using L = StageLayout<NT>;
  constexpr int kR = L::kR;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = base;                                                      // S x kStageBytes
  __nv_bfloat16* xh = reinterpret_cast<__nv_bfloat16*>(base + S * L::kStageBytes);  // [32][264]
  // [kKParts][32][r] partial P sums, written after the K loop when the stage
  // buffers are idle (every issued stage has been consumed by then)
  float* red = reinterpret_cast<float*>(stages);
  uint64_t* full = reinterpret_cast<uint64_t*>(xh + kRows * kXhStride);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int M = a.M, K = a.K;
  const int nchunks = (K + kChunk - 1) / kChunk;
  const float s_tx = a.s_tx;
  const float six_t = __fmul_rn(6.0f, s_tx);
  auto issue_stage = [&](int c, uint8_t* st, uint64_t* bar) {
    const int kcols = min(kChunk, K - c * kChunk);
    mbar_expect_tx(bar, kXBytes + L::kL1Bytes + kcols * 4);
    tma_load_2d(st, &tm_x, bar, c * kChunk, row0);
    if (NT) tma_load_2d(st + kXBytes, &tm_l1, bar, 0, c * kChunk);
    bulk_load(st + kXBytes + L::kL1Bytes, a.inv_lambda + (size_t)c * kChunk, (uint32_t)kcols * 4, bar);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    if (NT) tma_prefetch_desc(&tm_l1);
    for (int c = 0; c < S && c < nchunks; ++c) issue_stage(c, stages + c * L::kStageBytes, &full[c]);
  }
  __syncthreads();

  float acc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int t = 0; t < (NT > 0 ? NT : 1); ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  bool ok = true;
  int first_bad = nchunks;
  for (int c = 0; c < nchunks; ++c) {
    const int s = c % S;
    uint8_t* st = stages + s * L::kStageBytes;
    if (ok && !mbar_wait(&full[s], (c / S) & 1, wait_ns, err)) {
      ok = false;
      first_bad = c;
    }
    // every thread reaches the barriers below whatever happened, so that no
    // thread waits on one that others skipped
    const int col = c * kChunk + lane * 8;
    const bool col_ok = ok && col < K;

    float il[8];
    if (col_ok) {
      const float* ils = reinterpret_cast<const float*>(st + kXBytes + L::kL1Bytes);
      const float4 i0 = *reinterpret_cast<const float4*>(ils + lane * 8);
      const float4 i1 = *reinterpret_cast<const float4*>(ils + lane * 8 + 4);
      il[0] = i0.x; il[1] = i0.y; il[2] = i0.z; il[3] = i0.w;
      il[4] = i1.x; il[5] = i1.y; il[6] = i1.z; il[7] = i1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) il[j] = 0.f;
    }

#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int lr = warp + kWarpsQA * i;  // local row
      const int m = row0 + lr;
      const uint4 xv = *reinterpret_cast<const uint4*>(st + lr * (kChunk * 2) + lane * 16);
      const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
      float xf[8];
      uint32_t hb[4];
      __nv_bfloat162 amax2 = __float2bfloat162_rn(0.f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float x0 = __uint_as_float(w[j] << 16), x1 = __uint_as_float(w[j] & 0xFFFF0000u);
        hb[j] = pack_bf16x2(__fmul_rn(x0, il[2 * j]), __fmul_rn(x1, il[2 * j + 1]));
        xf[2 * j] = __uint_as_float(hb[j] << 16);
        xf[2 * j + 1] = __uint_as_float(hb[j] & 0xFFFF0000u);
        amax2 = __hmax2(amax2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&hb[j])));
      }
      float amax = fmaxf(__low2float(amax2), __high2float(amax2));
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
            const int ka = col / 64;  // atom index along K
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
      // tensor-core partial products: warp -> (row tile, K eighth)
      const int mt = warp & 1, kq = warp >> 1;
      const uint32_t l1base = smem_u32(st + kXBytes);
      constexpr int kSteps = kChunk / 16 / kKParts;  // k16 steps per warp and chunk
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        const int k0 = (kq * kSteps + ks) * 16;
        uint32_t a0, a1, a2, a3;
        const int ar = mt * 16 + (lane & 15), ac = k0 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(xh + ar * kXhStride + ac), a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < NT; t += 2) {
          uint32_t b0, b1, b2, b3;
          const int br = k0 + (lane & 7) + ((lane >> 3) & 1) * 8, bc = t + (lane >> 4);  // bc in 16-byte chunks
          const uint32_t off = (uint32_t)(br * (2 * kR) + 16 * bc);
          ldsm_x4_t(l1base + (off ^ (((off >> 7) & L::kSwzMask) << 4)), b0, b1, b2, b3);
          mma_16816(acc[t], a0, a1, a2, a3, b0, b1);
          mma_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();
    // stage s is free: refill it with chunk c + S
    if (threadIdx.x == 0 && ok && c + S < nchunks) issue_stage(c + S, st, &full[s]);
  }

  if (!ok) {
    // a stage never completed: let the copies already issued land before the
    // CTA exits (bounded), and write nothing more
    if (threadIdx.x == 0)
      for (int c = first_bad; c < nchunks && c < first_bad + S; ++c)
        (void)mbar_wait(&full[c % S], (c / S) & 1, wait_ns, nullptr);
    return;
  }
  if constexpr (NT > 0) {
    // fixed-order reduction of the K parts, then one bf16 rounding
    const int mt = warp & 1, kq = warp >> 1;
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int j = t * 8 + 2 * t4;
      float* rb = red + (size_t)kq * kRows * kR;
      rb[(mt * 16 + g) * kR + j] = acc[t][0];
      rb[(mt * 16 + g) * kR + j + 1] = acc[t][1];
      rb[(mt * 16 + g + 8) * kR + j] = acc[t][2];
      rb[(mt * 16 + g + 8) * kR + j + 1] = acc[t][3];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kRows * kR; e += blockDim.x) {
      const int lr = e / kR, j = e % kR;
      const int m = row0 + lr;
      if (m >= M || !ok) continue;
      float v = red[e];
#pragma unroll
      for (int part = 1; part < kKParts; ++part) v += red[part * kRows * kR + e];
      a.P[(size_t)m * kR + j] = (uint16_t)f32_to_bf16_bits(v);
    }
  }
}

template <int PREC, int NT>
cudaError_t launch_t(const QuantActArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  using L = StageLayout<NT>;
  constexpr int kR = L::kR;
  CUtensorMap tm_x, tm_l1;
  if (!make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, a.K, a.M, (uint64_t)a.K * 2, kChunk, kRows,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (NT) {
    const CUtensorMapSwizzle swz = kR == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : (kR == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    if (!make_tmap_2d(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L1, kR, a.K, (uint64_t)kR * 2, kR, kChunk, swz))
      return cudaErrorInvalidValue;
  } else {
    tm_l1 = tm_x;
  }
  static_assert((size_t)kKParts * kRows * kR * 4 <= (size_t)L::kStages * L::kStageBytes, "reduction fits the stages");
  const size_t smem = 1024 + (size_t)L::kStages * L::kStageBytes + (size_t)kRows * kXhStride * 2 + 64;
  auto k = quant_act_kernel<PREC, NT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (a.M + kRows - 1) / kRows;
  k<<<grid, kThreadsQA, smem, s>>>(tm_x, tm_l1, a, err, wait_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant_act(int prec, const QuantActArgs& a, unsigned* err, unsigned long long wait_ns,
                             cudaStream_t s) {
  const int nt = a.r / 8;
  if (prec == 0) {
    switch (nt) {
      case 0: return launch_t<0, 0>(a, err, wait_ns, s);
      case 2: return launch_t<0, 2>(a, err, wait_ns, s);
      case 4: return launch_t<0, 4>(a, err, wait_ns, s);
    }
  } else {
    switch (nt) {
      case 0: return launch_t<1, 0>(a, err, wait_ns, s);
      case 2: return launch_t<1, 2>(a, err, wait_ns, s);
      case 4: return launch_t<1, 4>(a, err, wait_ns, s);
      case 6: return launch_t<1, 6>(a, err, wait_ns, s);
      case 8: return launch_t<1, 8>(a, err, wait_ns, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace svdq
