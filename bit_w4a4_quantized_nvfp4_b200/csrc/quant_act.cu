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
// Work split: a CTA owns 32 rows (two 16-row MMA tiles) and walks K in chunks
// of 256 columns. A producer warp streams each chunk through a multi-stage
// TMA pipeline (the 32 x 256 x tile as four 128-byte-swizzled boxes, the
// matching 256 x r L1 tile and the chunk's inv_lambda); full/empty mbarriers
// let every consumer warp run at its own pace, with no CTA-wide barrier
// inside the K loop.
//
// Each of the 16 consumer warps owns one (row tile, K slice) block of 16 rows
// x 64 columns in every other chunk (eight warps per chunk, two chunks in
// work at a time). A lane holds 32 columns of one row: two NVFP4 groups,
// whose independent dependency chains interleave, or half an INT4 group. The
// warp quantises its block, writes x_hat back over its x block in the stage
// and multiplies it by its K slice of the L1 tile on tensor cores (mma.sync
// bf16, fp32 accumulate), so P needs no cross-warp exchange until the end,
// where the eight partial sums of each row tile are added in a fixed order
// and rounded to bf16 once.
//
// Stage reuse: chunk c lives in stage c % S and the two warp groups take
// alternate chunks, so S is kept even. A stage is then always refilled for
// the group that released it, and no warp can wait on a full barrier more
// than one phase ahead of it (with S odd, the previous user of a stage is
// the other group, and a parity wait could pass on the wrong phase). The NVFP4 dequantisation step d = e4m3(s) * s_tx and
// its reciprocal depend only on the 8-bit scale code, so each CTA tabulates
// them once for all 256 codes.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRows = 32;                   // rows per CTA
constexpr int kChunk = 256;                 // K columns per stage
constexpr int kXBytes = kRows * kChunk * 2;
constexpr int kXBoxBytes = kRows * 64 * 2;  // one [32 rows][64 cols] box, 128-byte swizzle
constexpr int kConsumerWarps = 16;
constexpr int kThreadsQA = (kConsumerWarps + 1) * 32;
constexpr int kParts = 8;                   // partial P sums per row tile
constexpr int kSmemLimit = 232448;          // dynamic shared memory per CTA on sm_100

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

// (a0 * b0, a1 * b1), each rounded to nearest like two fp32 multiplies
__device__ __forceinline__ void mul2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  unsigned long long A, B, D;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b0), "f"(b1));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(D));
}

// smooth 8 bf16 values (one 16-byte word of x) by their inv_lambda: returns
// bf16x2 words of x_hat and folds |x_hat| into `amax2`
__device__ __forceinline__ void smooth8(const uint4 xv, const float* il, uint32_t (&hb)[4],
                                        __nv_bfloat162& amax2) {
  const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float p0, p1;
    mul2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u), il[2 * j], il[2 * j + 1], p0, p1);
    hb[j] = pack_bf16x2(p0, p1);
    amax2 = __hmax2(amax2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&hb[j])));
  }
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int PREC, int NT>
struct Cfg {
  static constexpr int kR = NT * 8;
  static constexpr int KW = 64;                                 // columns per warp block
  static constexpr int kKParts = kChunk / KW;                   // K slices per chunk
  static constexpr int kPhases = kConsumerWarps / 2 / kKParts;  // chunks in work per CTA
  static constexpr int kConsumers = kConsumerWarps / kPhases;   // warps reading one chunk
  static constexpr int kL1Bytes = NT ? kChunk * kR * 2 : 0;
  static constexpr int kIlBytes = kChunk * 4;
  static constexpr int kStageBytes = ((kXBytes + kL1Bytes + kIlBytes + 1023) / 1024) * 1024;
  static constexpr int kFixed = 1024 + 256 * 8 + 256;
  static constexpr int kFit = (kSmemLimit - kFixed) / kStageBytes;
  static constexpr int kStages = ((kFit > 8 ? 8 : kFit) / kPhases) * kPhases;
  static constexpr size_t kSmem = (size_t)kFixed + (size_t)kStages * kStageBytes;
  // the L1 tile rows are 2r bytes; the TMA swizzle span equals the row (32/64/128 B)
  static constexpr uint32_t kSwzMask = kR <= 16 ? 1u : (kR == 32 ? 3u : 7u);
  static_assert(kKParts * kPhases == kParts, "eight partial sums per row tile");
  static_assert((size_t)kParts * kRows * (kR > 0 ? kR : 1) * 4 <= (size_t)kStages * kStageBytes,
                "the reduction buffer fits in the stages");
  static_assert(2 * kStages * 8 + 4 <= 256, "barriers fit their reserve");
  static_assert(kStages >= 2 && kStages % kPhases == 0, "a stage is reused by one warp group only");
};

// PREC 0 = NVFP4 (group 16, E4M3 scales in the tiled layout), 1 = INT4
// (group 64, bf16 scales row-major, row pitch int4_act_scale_pitch). NT = r / 8
// tiles of the P output.
template <int PREC, int NT>
__global__ void __launch_bounds__(kThreadsQA, 1)
quant_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
                 QuantActArgs a, unsigned* err, unsigned long long wait_ns) {
  using C = Cfg<PREC, NT>;
  constexpr int kR = C::kR;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = base;                                       // S x kStageBytes
  uint64_t* full = reinterpret_cast<uint64_t*>(base + S * C::kStageBytes);
  uint64_t* empty = full + S;
  int* abort_flag = reinterpret_cast<int*>(empty + S);
  // NVFP4: per scale code, {1 / (e4m3(code) * s_tx), 1 if that step is 0}
  float2* rtab = reinterpret_cast<float2*>(base + S * C::kStageBytes + 256);
  // [kParts][32][r] partial P sums, written after the K loop when every
  // issued stage has been consumed
  float* red = reinterpret_cast<float*>(stages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kRows;
  const int M = a.M, K = a.K;
  const int nchunks = (K + kChunk - 1) / kChunk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  const float s_tx = PREC == 0 ? a.tensor_scale[1] : 1.0f;
  if (PREC == 0 && threadIdx.x < 256) {
    const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), s_tx);
    rtab[threadIdx.x] = d != 0.f ? make_float2(__frcp_rn(d), 0.f) : make_float2(0.f, 1.f);
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (NT) tma_prefetch_desc(&tm_l1);
      int c = 0;
      bool ok = true;
      for (; c < nchunks; ++c) {
        const int s = c % S;
        if (c >= S && !mbar_wait(&empty[s], ((c / S) - 1) & 1, wait_ns, err)) {
          ok = false;
          break;
        }
        uint8_t* st = stages + s * C::kStageBytes;
        const int kcols = min(kChunk, K - c * kChunk);
        const int nbox = kcols / 64;
        mbar_expect_tx(&full[s], nbox * kXBoxBytes + C::kL1Bytes + kcols * 4);
        for (int b = 0; b < nbox; ++b) tma_load_2d(st + b * kXBoxBytes, &tm_x, &full[s], c * kChunk + 64 * b, row0);
        if (NT) tma_load_2d(st + kXBytes, &tm_l1, &full[s], 0, c * kChunk);
        bulk_load(st + kXBytes + C::kL1Bytes, a.inv_lambda + (size_t)c * kChunk, (uint32_t)kcols * 4, &full[s]);
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit (bounded)
        for (int j = max(0, c - S); j < c; ++j) (void)mbar_wait(&full[j % S], (j / S) & 1, wait_ns, nullptr);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int rt = warp & 1;                     // row tile
  const int kp = (warp >> 1) % C::kKParts;     // K slice within a chunk
  const int phase = (warp >> 1) / C::kKParts;  // chunk phase
  const int rl = lane & 15, h = lane >> 4;
  const int lr = rt * 16 + rl;                 // local row
  const int m = row0 + lr;
  const bool row_ok = m < M;
  const float six_t = __fmul_rn(6.0f, s_tx);
  // this lane's outputs, advanced by one chunk per step: codes of columns
  // c*256 + kp*64 + 32h .. +31, and the scale word (NVFP4: the 4 scales of
  // 64-column atom 4c + kp in row m; INT4: scale 4c + kp of row m)
  const int m_c = row_ok ? m : 0;
  uint8_t* code_ptr = a.codes + (size_t)m_c * (K / 2) + kp * 32 + h * 16;
  uint8_t* scale_ptr =
      PREC == 0 ? static_cast<uint8_t*>(a.scales) + ((size_t)(m_c / 128) * (K / 64) + kp) * 512 + 16 * (m_c % 32) +
                      4 * ((m_c % 128) / 32)
                : static_cast<uint8_t*>(a.scales) + ((size_t)m_c * int4_act_scale_pitch(K) + kp) * 2;

  float acc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int t = 0; t < (NT > 0 ? NT : 1); ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  bool ok = true;
  for (int c = phase; c < nchunks; c += C::kPhases) {
    const int s = c % S;
    const uint8_t* st = stages + s * C::kStageBytes;
    if (!warp_wait(&full[s], (c / S) & 1, wait_ns, err)) {
      ok = false;
      break;
    }
    const int kcols = min(kChunk, K - c * kChunk);
    if (kp * C::KW < kcols) {  // warp-uniform: the block lies inside K
      const int cc = kp * C::KW + h * (C::KW / 2);  // first chunk column of this lane
      // this warp's x block: rows 16rt .. of box kp (128-byte lines, units swizzled by line)
      uint8_t* xblk = stages + s * C::kStageBytes + kp * kXBoxBytes + rt * 16 * 128;
      const uint8_t* xrow = xblk + rl * 128;
      const float* ils = reinterpret_cast<const float*>(st + kXBytes + C::kL1Bytes) + cc;
      // smooth 32 columns: x_hat words hb[0..15], |x_hat| maxima of the two 16-column halves
      uint32_t hb[16];
      __nv_bfloat162 amax2[2] = {__float2bfloat162_rn(0.f), __float2bfloat162_rn(0.f)};
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xrow + (((4 * h + v) ^ (lr & 7)) << 4));
        float il[8];
        *reinterpret_cast<float4*>(il) = *reinterpret_cast<const float4*>(ils + 8 * v);
        *reinterpret_cast<float4*>(il + 4) = *reinterpret_cast<const float4*>(ils + 8 * v + 4);
        uint32_t hv[4];
        smooth8(xv, il, hv, amax2[v >> 1]);
#pragma unroll
        for (int j = 0; j < 4; ++j) hb[4 * v + j] = hv[j];
      }
      // x_hat over the lane's own x words, for the P product
#pragma unroll
      for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4*>(xblk + rl * 128 + (((4 * h + v) ^ (lr & 7)) << 4)) =
            make_uint4(hb[4 * v], hb[4 * v + 1], hb[4 * v + 2], hb[4 * v + 3]);
      const size_t cstep = (size_t)c;

      if constexpr (PREC == 0) {
        // two NVFP4 groups of 16 per lane
        uint32_t code[4], sfw = 0;
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          const float amax = fmaxf(__low2float(amax2[gi]), __high2float(amax2[gi]));
          const uint32_t sf = cvt_e4m3(__fdiv_rn(amax, six_t)) & 0xFFu;
          const float2 rt_e = rtab[sf];
          float q[16];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mul2(__uint_as_float(hb[8 * gi + j] << 16), __uint_as_float(hb[8 * gi + j] & 0xFFFF0000u), rt_e.x,
                 rt_e.x, q[2 * j], q[2 * j + 1]);
          // a zero dequantisation step codes the whole group as +0
          const bool zero = rt_e.y != 0.f;
          code[2 * gi] = zero ? 0u : cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(q));
          code[2 * gi + 1] = zero ? 0u : cvt_e2m1x8(*reinterpret_cast<const float(*)[8]>(q + 8));
          sfw |= sf << (8 * gi);
        }
        // the row's four scales of this 64-column atom: lanes h = 0 and 1
        const uint32_t sfw_hi = __shfl_xor_sync(0xffffffffu, sfw, 16);
        if (row_ok) {
          *reinterpret_cast<uint4*>(code_ptr + cstep * 128) = make_uint4(code[0], code[1], code[2], code[3]);
          if (h == 0) *reinterpret_cast<uint32_t*>(scale_ptr + cstep * 4 * 512) = sfw | (sfw_hi << 16);
        }
      } else {
        // half an INT4 group of 64 per lane
        __nv_bfloat162 am = __hmax2(amax2[0], amax2[1]);
        float amax = fmaxf(__low2float(am), __high2float(am));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
        const uint32_t sb = f32_to_bf16_bits(__fdiv_rn(amax, 7.0f));
        const float sfv = bf16_bits_to_f32(sb);
        uint32_t code[4] = {0u, 0u, 0u, 0u};
        if (sfv != 0.f) {
          const float inv = __frcp_rn(sfv);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float q0, q1;
              const uint32_t hw = hb[4 * w + j];
              mul2(__uint_as_float(hw << 16), __uint_as_float(hw & 0xFFFF0000u), inv, inv, q0, q1);
              const int i0 = max(-8, min(7, __float2int_rn(q0)));
              const int i1 = max(-8, min(7, __float2int_rn(q1)));
              code[w] |= (((uint32_t)i0 & 0xFu) | (((uint32_t)i1 & 0xFu) << 4)) << (8 * j);
            }
          }
        }
        if (row_ok) {
          *reinterpret_cast<uint4*>(code_ptr + cstep * 128) = make_uint4(code[0], code[1], code[2], code[3]);
          if (h == 0) *reinterpret_cast<uint16_t*>(scale_ptr + cstep * 8) = (uint16_t)sb;
        }
      }

      if constexpr (NT > 0) {
        __syncwarp();
        // this block's share of P: x_hat[16 x KW] times rows kp*KW .. of the L1 tile
        const uint32_t l1base = smem_u32(st + kXBytes);
#pragma unroll
        for (int ks = 0; ks < C::KW / 16; ++ks) {
          uint32_t a0, a1, a2, a3;
          const int ar = lane & 15, au = 2 * ks + (lane >> 4);
          ldsm_x4(smem_u32(xblk) + ar * 128 + ((au ^ (ar & 7)) << 4), a0, a1, a2, a3);
          const int k0 = kp * C::KW + ks * 16;
#pragma unroll
          for (int t = 0; t < NT; t += 2) {
            uint32_t b0, b1, b2, b3;
            const int br = k0 + (lane & 7) + ((lane >> 3) & 1) * 8, bc = t + (lane >> 4);  // bc: 16-byte unit
            const uint32_t off = (uint32_t)(br * (2 * kR) + 16 * bc);
            ldsm_x4_t(l1base + (off ^ (((off >> 7) & C::kSwzMask) << 4)), b0, b1, b2, b3);
            mma_16816(acc[t], a0, a1, a2, a3, b0, b1);
            mma_16816(acc[t + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
    }
    // the stage may be refilled (by the async proxy) once every lane is past
    // its reads and writes of it: the P MMAs (which use the last reads of the
    // stage) are kept ahead of the release
    if constexpr (NT > 0) {
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) consumed(acc[t][i]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  if (!ok && lane == 0) *abort_flag = 1;
  named_sync(1, kConsumerWarps * 32);
  // after a timed-out stage, copies may still be landing in the stages: write
  // nothing more
  if (*abort_flag) return;
  if constexpr (NT > 0) {
    // fixed-order reduction of the eight K parts, then one bf16 rounding
    const int part = phase * C::kKParts + kp;
    const int g = lane >> 2, t4 = lane & 3;
    float* rb = red + (size_t)part * kRows * kR;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int j = t * 8 + 2 * t4;
      rb[(rt * 16 + g) * kR + j] = acc[t][0];
      rb[(rt * 16 + g) * kR + j + 1] = acc[t][1];
      rb[(rt * 16 + g + 8) * kR + j] = acc[t][2];
      rb[(rt * 16 + g + 8) * kR + j + 1] = acc[t][3];
    }
    named_sync(1, kConsumerWarps * 32);
    for (int e = threadIdx.x; e < kRows * kR; e += kConsumerWarps * 32) {
      const int er = e / kR, j = e % kR;
      const int mm = row0 + er;
      if (mm >= M) continue;
      float v = red[e];
#pragma unroll
      for (int p = 1; p < kParts; ++p) v += red[p * kRows * kR + e];
      a.P[(size_t)mm * kR + j] = (uint16_t)f32_to_bf16_bits(v);
    }
  }
}

template <int PREC, int NT>
cudaError_t launch_t(const QuantActArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  using C = Cfg<PREC, NT>;
  constexpr int kR = C::kR;
  CUtensorMap tm_x, tm_l1;
  if (!make_tmap_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, a.K, a.M, (uint64_t)a.K * 2, 64, kRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (NT) {
    const CUtensorMapSwizzle swz = kR == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : (kR == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    if (!make_tmap_2d(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L1, kR, a.K, (uint64_t)kR * 2, kR, kChunk, swz))
      return cudaErrorInvalidValue;
  } else {
    tm_l1 = tm_x;
  }
  auto k = quant_act_kernel<PREC, NT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = (a.M + kRows - 1) / kRows;
  k<<<grid, kThreadsQA, C::kSmem, s>>>(tm_x, tm_l1, a, err, wait_ns);
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
