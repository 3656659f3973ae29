// K3 — AWQ W4A16 linear: INT4 weights (asymmetric, bf16 scale/zero per 64
// along K) times bf16 activations, for the memory-bound modulation /
// adaptive-norm projections (blog "Introducing Nunchaku 4-bit inference in
// Diffusers", section "Introducing Nunchaku Lite").
//
// The weight stream is the whole cost at small M, so the kernel reads every
// weight byte once with 8-byte loads, unpacks nibbles to bf16 with bit
// operations ((128 + q) has an exact bf16 encoding; subtracting 128 + z gives
// q - z exactly) and lets the tensor cores (mma.sync m16n8k16, fp32
// accumulate) form the dot products, so that the CUDA cores only unpack.
//
// Work split: a CTA of 4 warps owns 64 output columns (16 per warp, the MMA's
// 16-row operand) and walks K in chunks of 16 groups. Activations of up to 16
// rows are staged per chunk in shared memory in MMA-fragment order. Each
// group's partial dot products are scaled by the group scale in fp32.
//
// K order inside a group: lane t of a row quad owns k = 16t .. 16t+15 (one
// 8-byte load). Its nibbles are unpacked in pairs (k, k+4) and fed to the MMA
// K slots in the order (0,4),(1,5) | (2,6),(3,7) | (8,12),(9,13) | (10,14),(11,15)
// for the four k16 steps; the activation fragments use the same order, so the
// dot product is unchanged.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kCols = 64;          // output columns per CTA
constexpr int kChunkGroups = 16;   // groups of 64 per K chunk
constexpr int kMaxMT = 2;          // m-tiles of 8 rows per pass

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// nibbles k and k+4 of `w` (k = sh/4) -> bf16x2 of (q - z)
__device__ __forceinline__ uint32_t deq_pair(uint32_t w, int sh, uint32_t zz) {
  const uint32_t v = ((w >> sh) & 0x000F000Fu) | 0x43004300u;
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(zz));
  return r;
}

// x fragment store layout per chunk: [group][step][t][m (8)][2 words], one
// m-tile after another.
__global__ void __launch_bounds__(128) awq_kernel(AwqArgs a) {
  extern __shared__ __align__(16) uint32_t xs[];  // kMaxMT * kChunkGroups * 4 * 4 * 8 * 2 words
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, t = lane & 3;
  const int K = a.K, N = a.N, M = a.M;
  const int ng = K / 64;
  const int n_lo = blockIdx.x * kCols + warp * 16 + gid;   // row gid of the warp's A tile
  const int n_hi = n_lo + 8;
  const bool ok_lo = n_lo < N, ok_hi = n_hi < N;
  const uint8_t* q_lo = a.q + (size_t)n_lo * (K / 2);
  const uint8_t* q_hi = a.q + (size_t)n_hi * (K / 2);

  for (int m0 = 0; m0 < M; m0 += 8 * kMaxMT) {
    const int mt_count = min(kMaxMT, (M - m0 + 7) / 8);
    float tot[kMaxMT][4];
#pragma unroll
    for (int i = 0; i < kMaxMT; ++i) tot[i][0] = tot[i][1] = tot[i][2] = tot[i][3] = 0.f;

    for (int g0 = 0; g0 < ng; g0 += kChunkGroups) {
      const int gcount = min(kChunkGroups, ng - g0);
      // weights of this chunk: issue all loads first
      uint2 wl[kChunkGroups], wh[kChunkGroups];
      uint32_t sl[kChunkGroups], sh[kChunkGroups];
#pragma unroll
      for (int j = 0; j < kChunkGroups; ++j) {
        const int g = g0 + j;
        wl[j] = wh[j] = make_uint2(0, 0);
        sl[j] = sh[j] = 0;
        if (j < gcount) {
          if (ok_lo) {
            wl[j] = *reinterpret_cast<const uint2*>(q_lo + g * 32 + t * 8);
            sl[j] = (uint32_t)a.s[(size_t)n_lo * ng + g] | ((uint32_t)a.z[(size_t)n_lo * ng + g] << 16);
          }
          if (ok_hi) {
            wh[j] = *reinterpret_cast<const uint2*>(q_hi + g * 32 + t * 8);
            sh[j] = (uint32_t)a.s[(size_t)n_hi * ng + g] | ((uint32_t)a.z[(size_t)n_hi * ng + g] << 16);
          }
        }
      }

      // stage activations of this chunk in fragment order: one 16-byte load
      // holds x[m, 64g + 16t + 8h .. +7], i.e. the pairs (e, e+4) of steps
      // 2h (e = 8h, 8h+1) and 2h+1 (e = 8h+2, 8h+3)
      __syncthreads();
      const int loads = mt_count * 8 * kChunkGroups * 8;  // (m, group, t, h)
      for (int li = threadIdx.x; li < loads; li += blockDim.x) {
        int r = li;
        const int h = r & 1; r >>= 1;
        const int tt = r & 3; r >>= 2;
        const int gg = r % kChunkGroups; r /= kChunkGroups;
        const int mm = r & 7;
        const int mt = r >> 3;
        const int m = m0 + mt * 8 + mm;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M && gg < gcount)
          v = *reinterpret_cast<const uint4*>(a.x + (size_t)m * K + (g0 + gg) * 64 + tt * 16 + h * 8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        // element e' (0..7) of the load: bf16 halves of w[e'/2]
#pragma unroll
        for (int q = 0; q < 4; ++q) {          // pair (q, q+4) of the load
          const uint32_t lo = (q & 1) ? (w[q >> 1] >> 16) : (w[q >> 1] & 0xFFFFu);
          const uint32_t hi = (q & 1) ? (w[2 + (q >> 1)] >> 16) : (w[2 + (q >> 1)] & 0xFFFFu);
          const int st = 2 * h + (q >> 1), half = q & 1;
          xs[((((mt * kChunkGroups + gg) * 4 + st) * 4 + tt) * 8 + mm) * 2 + half] = lo | (hi << 16);
        }
      }
      __syncthreads();

#pragma unroll
      for (int j = 0; j < kChunkGroups; ++j) {
        if (j < gcount) {
          const uint32_t zl = (sl[j] >> 16) & 0xFFFFu, zh = (sh[j] >> 16) & 0xFFFFu;
          // bf16(128 + z) for both halves
          const uint32_t zzl = f32_to_bf16_bits(128.0f + bf16_bits_to_f32(zl)) * 0x10001u;
          const uint32_t zzh = f32_to_bf16_bits(128.0f + bf16_bits_to_f32(zh)) * 0x10001u;
          uint32_t A[4][4];
          // step 0: (0,4),(1,5) from word 0; step 1: (2,6),(3,7); step 2/3 from word 1
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint32_t wlo = (s < 2) ? wl[j].x : wl[j].y;
            const uint32_t whi = (s < 2) ? wh[j].x : wh[j].y;
            const int sh0 = (s & 1) * 8;
            A[s][0] = deq_pair(wlo, sh0, zzl);
            A[s][1] = deq_pair(whi, sh0, zzh);
            A[s][2] = deq_pair(wlo, sh0 + 4, zzl);
            A[s][3] = deq_pair(whi, sh0 + 4, zzh);
          }
          const float s_lo = bf16_bits_to_f32(sl[j] & 0xFFFFu), s_hi = bf16_bits_to_f32(sh[j] & 0xFFFFu);
#pragma unroll
          for (int mt = 0; mt < kMaxMT; ++mt) {
            if (mt < mt_count) {
              float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int s = 0; s < 4; ++s) {
                const uint32_t* bp = xs + ((((mt * kChunkGroups + j) * 4 + s) * 4 + t) * 8 + gid) * 2;
                mma_16816(c, A[s], bp[0], bp[1]);
              }
              tot[mt][0] = fmaf(s_lo, c[0], tot[mt][0]);
              tot[mt][1] = fmaf(s_lo, c[1], tot[mt][1]);
              tot[mt][2] = fmaf(s_hi, c[2], tot[mt][2]);
              tot[mt][3] = fmaf(s_hi, c[3], tot[mt][3]);
            }
          }
        }
      }
    }

    // write y: c0/c1 -> (n_lo, m = 2t, 2t+1), c2/c3 -> (n_hi, ...)
    const float b_lo = (a.bias && ok_lo) ? bf16_bits_to_f32(a.bias[n_lo]) : 0.f;
    const float b_hi = (a.bias && ok_hi) ? bf16_bits_to_f32(a.bias[n_hi]) : 0.f;
#pragma unroll
    for (int mt = 0; mt < kMaxMT; ++mt) {
      if (mt >= mt_count) continue;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int m = m0 + mt * 8 + 2 * t + i;
        if (m >= M) continue;
        if (ok_lo) a.y[(size_t)m * N + n_lo] = (uint16_t)f32_to_bf16_bits(__fadd_rn(tot[mt][i], b_lo));
        if (ok_hi) a.y[(size_t)m * N + n_hi] = (uint16_t)f32_to_bf16_bits(__fadd_rn(tot[mt][2 + i], b_hi));
      }
    }
  }
}

}  // namespace

cudaError_t launch_awq(const AwqArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)kMaxMT * kChunkGroups * 4 * 4 * 8 * 2 * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(awq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (a.N + kCols - 1) / kCols;
  awq_kernel<<<grid, 128, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace svdq
