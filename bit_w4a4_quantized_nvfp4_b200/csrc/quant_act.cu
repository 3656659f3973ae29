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
// Consumers: 8 warps cover one chunk, each a block of 16 rows x 64 columns
// (row tile rt, K slice kp); the consumer warps form kPhases groups of 8 that
// take chunks round-robin, so kPhases chunks are in work at once. Inside a
// block a lane holds 16 columns (one NVFP4 group, a quarter of an INT4 group)
// of two rows, p and p + 8: the two groups' dependency chains interleave, and
// the lane's 16 inv_lambda values serve both rows. The warp writes x_hat back
// over its x block in the stage and multiplies it by its K slice of the L1
// tile on tensor cores (mma.sync bf16, fp32 accumulate), so P needs no
// cross-warp exchange until the end, where the partial sums of each row tile
// are added in a fixed order and rounded to bf16 once.
//
// Stage reuse: chunk c lives in stage c % S and the groups take chunks
// round-robin, so S is a multiple of kPhases: a stage is then always refilled
// for the group that released it, and no warp can wait on a full barrier more
// than one phase ahead of it (otherwise a parity wait could pass on the wrong
// phase). The NVFP4 dequantisation step d = e4m3(s) * s_tx and its reciprocal
// depend only on the 8-bit scale code, so each CTA tabulates them once for
// all 256 codes.
//
// Programmatic dependent launch: the kernel lets the next kernel in the
// stream be scheduled at once (it waits for this one before it reads any
// output), and reads or writes nothing that an earlier kernel may touch
// (x, inv_lambda, the tensor scales, L1, the outputs) before
// griddepcontrol.wait; only barrier set-up and L2 prefetches precede it.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRows = 32;                   // rows per CTA
constexpr int kChunk = 256;                 // K columns per stage
constexpr int kXBytes = kRows * kChunk * 2;
constexpr int kXBoxBytes = kRows * 64 * 2;  // one [32 rows][64 cols] box, 128-byte swizzle
constexpr int kKParts = kChunk / 64;        // 64-column K slices per chunk
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

// per half: |max(|a|, |b|)| in magnitude (the sign bits are garbage and are
// cleared by the caller); one instruction for abs + max of a bf16 pair
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// per 16-bit half: unsigned maximum
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// element i of four float4
__device__ __forceinline__ float f4at(const float4 (&v)[4], int i) {
  const float4 q = v[i >> 2];
  return (i & 3) == 0 ? q.x : (i & 3) == 1 ? q.y : (i & 3) == 2 ? q.z : q.w;
}

// smooth 16 bf16 values (two 16-byte words of x) by their inv_lambda: x_hat
// as 8 bf16x2 words, and the running |x_hat| maximum of the 16 (in both halves)
__device__ __forceinline__ uint32_t smooth16(const uint4 xa, const uint4 xb, const float4 (&il)[4],
                                             uint32_t (&hb)[8]) {
  const uint32_t w[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
  uint32_t am = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float p0, p1;
    mul2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u), f4at(il, 2 * j), f4at(il, 2 * j + 1),
         p0, p1);
    hb[j] = pack_bf16x2(p0, p1);
    am = absmax_bf16x2(am, hb[j]);
  }
  return am & 0x7FFF7FFFu;
}

// 16 NVFP4 codes of a group: E2M1 of fl(x_hat * rcp) for the 8 x_hat words
// (element 2j of the group in the low nibble of byte j)
__device__ __forceinline__ uint2 e2m1_group(const uint32_t (&hb)[8], float rcp) {
  float q[16];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    mul2(__uint_as_float(hb[j] << 16), __uint_as_float(hb[j] & 0xFFFF0000u), rcp, rcp, q[2 * j], q[2 * j + 1]);
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w[h])
        : "f"(q[8 * h]), "f"(q[8 * h + 1]), "f"(q[8 * h + 2]), "f"(q[8 * h + 3]), "f"(q[8 * h + 4]),
          "f"(q[8 * h + 5]), "f"(q[8 * h + 6]), "f"(q[8 * h + 7]));
  }
  return make_uint2(w[0], w[1]);
}

// bf16 bits of the larger of the two (non-negative) halves
__device__ __forceinline__ uint32_t max_half(uint32_t am) {
  const uint32_t lo = am & 0xFFFFu, hi = am >> 16;
  return lo > hi ? lo : hi;
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int PREC, int NT>
struct Cfg {
  static constexpr int kR = NT * 8;
  static constexpr int kConsumerWarps = NT > 4 ? 16 : 24;      // registers: 16 warps when P holds 6-8 tiles
  static constexpr int kPhases = kConsumerWarps / 8;           // chunks in work per CTA
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;
  // registers per thread: the most that fits in the 64K-entry register file
  // when the CTA's warps are counted in groups of four (8-register steps)
  static constexpr int kMaxRegs = ((65536 / ((kConsumerWarps + 1 + 3) / 4 * 4 * 32)) / 8) * 8;
  static constexpr int kParts = kPhases * kKParts;             // partial P sums per row tile
  static constexpr int kL1Bytes = NT ? kChunk * kR * 2 : 0;
  static constexpr int kIlBytes = kChunk * 4;
  static constexpr int kStageBytes = ((kXBytes + kL1Bytes + kIlBytes + 1023) / 1024) * 1024;
  static constexpr int kFixed = 1024 + 256 * 8 + 256;
  static constexpr int kFit = (kSmemLimit - kFixed) / kStageBytes;
  static constexpr int kStages = ((kFit > 9 ? 9 : kFit) / kPhases) * kPhases;
  static constexpr size_t kSmem = (size_t)kFixed + (size_t)kStages * kStageBytes;
  // the L1 tile rows are 2r bytes; the TMA swizzle span equals the row (32/64/128 B)
  static constexpr uint32_t kSwzMask = kR <= 16 ? 1u : (kR == 32 ? 3u : 7u);
  static_assert((size_t)kParts * kRows * (kR > 0 ? kR : 1) * 4 <= (size_t)kStages * kStageBytes,
                "the reduction buffer fits in the stages");
  static_assert(2 * kStages * 8 + 4 <= 256, "barriers fit their reserve");
  static_assert(kStages >= kPhases && kStages % kPhases == 0, "a stage is reused by one warp group only");
};

// PREC 0 = NVFP4 (group 16, E4M3 scales in the tiled layout), 1 = INT4
// (group 64, bf16 scales row-major, row pitch int4_act_scale_pitch). NT = r / 8
// tiles of the P output.
template <int PREC, int NT>
__global__ void __maxnreg__((Cfg<PREC, NT>::kMaxRegs))
quant_act_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_l1,
                 QuantActArgs a, unsigned* err, unsigned long long wait_ns) {
  using C = Cfg<PREC, NT>;
  constexpr int kR = C::kR;
  constexpr int S = C::kStages;
  constexpr int CW = C::kConsumerWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align<1024>(smem_raw);
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

  if (threadIdx.x == 0) launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == CW && lane == 0) {
    tma_prefetch_desc(&tm_x);
    if (NT) tma_prefetch_desc(&tm_l1);
    // only the first two chunks: a deeper prefetch (all S stages) queues ahead
    // of the first chunk's own loads and delays the start (measured)
    for (int c = 0; c < nchunks && c < 2; ++c)
      for (int b = 0; b < min(kChunk, K - c * kChunk) / 64; ++b) tma_prefetch_l2_2d(&tm_x, c * kChunk + 64 * b, row0);
  }
  __syncthreads();  // the barriers are initialised
  // every input may be the previous kernel's output, every output may still
  // be read by it
  grid_dependency_wait();
  // the producer starts its loads at once; the consumers first tabulate the
  // scale steps (named barrier 1: consumer warps only)
  const float s_tx = PREC == 0 && warp < CW ? a.tensor_scale[1] : 1.0f;
  if (PREC == 0 && threadIdx.x < 256) {
    const float d = __fmul_rn(e4m3_to_f32(threadIdx.x), s_tx);
    rtab[threadIdx.x] = d != 0.f ? make_float2(__frcp_rn(d), 0.f) : make_float2(0.f, 1.f);
  }
  if (warp < CW) named_sync(1, CW * 32);

  if (warp == CW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
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
  const int rt = warp & 1;                 // row tile
  const int kp = (warp >> 1) & 3;          // K slice within a chunk
  const int phase = warp >> 3;             // chunk phase
  const int p = lane & 7, cq = lane >> 3;  // rows p and p + 8 of the tile, columns 16 cq .. 16 cq + 15
  const int lr0 = rt * 16 + p;             // local rows lr0, lr0 + 8
  const int m0 = row0 + lr0, m1 = m0 + 8;
  const bool ok0 = m0 < M, ok1 = m1 < M;
  const float six_t = __fmul_rn(6.0f, s_tx);
  // this lane's x words in a block: 16-byte units 2cq, 2cq + 1 of rows p, p + 8
  // (128-byte swizzle: unit u of row r sits at (u ^ (r & 7)) << 4)
  const uint32_t xoff0 = (uint32_t)(kp * kXBoxBytes + lr0 * 128 + (((2 * cq) ^ p) << 4));
  const uint32_t xoff1 = (uint32_t)(kp * kXBoxBytes + lr0 * 128 + (((2 * cq + 1) ^ p) << 4));
  const uint32_t iloff = (uint32_t)(kXBytes + C::kL1Bytes + (kp * 64 + 16 * cq) * 4);
  // outputs, advanced by one chunk per step
  uint8_t* code0 = a.codes + (size_t)(ok0 ? m0 : 0) * (K / 2) + kp * 32 + cq * 8;
  uint8_t* code1 = a.codes + (size_t)(ok1 ? m1 : 0) * (K / 2) + kp * 32 + cq * 8;
  uint8_t* sc0;
  uint8_t* sc1;
  if constexpr (PREC == 0) {
    auto at = [&](int m) {
      return static_cast<uint8_t*>(a.scales) + ((size_t)(m / 128) * (K / 64) + kp) * 512 + 16 * (m % 32) +
             4 * ((m % 128) / 32) + cq;
    };
    sc0 = at(ok0 ? m0 : 0);
    sc1 = at(ok1 ? m1 : 0);
  } else {
    sc0 = static_cast<uint8_t*>(a.scales) + ((size_t)(ok0 ? m0 : 0) * int4_act_scale_pitch(K) + kp) * 2;
    sc1 = static_cast<uint8_t*>(a.scales) + ((size_t)(ok1 ? m1 : 0) * int4_act_scale_pitch(K) + kp) * 2;
  }
  // P fragments: A from this warp's x_hat block, B from rows kp*64 .. of the L1 tile
  const int ar = lane & 15;
  const uint32_t aoff = (uint32_t)(kp * kXBoxBytes + (rt * 16 + ar) * 128);
  const int ab = lane >> 4;

  float acc[NT > 0 ? NT : 1][4];
#pragma unroll
  for (int t = 0; t < (NT > 0 ? NT : 1); ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  bool ok = true;
  for (int c = phase; c < nchunks; c += C::kPhases) {
    const int s = c % S;
    uint8_t* st = stages + s * C::kStageBytes;
    if (!warp_wait(&full[s], (c / S) & 1, wait_ns, err)) {
      ok = false;
      break;
    }
    const int kcols = min(kChunk, K - c * kChunk);
    if (kp * 64 < kcols) {  // warp-uniform: the block lies inside K
      const uint4 xa0 = *reinterpret_cast<const uint4*>(st + xoff0);
      const uint4 xb0 = *reinterpret_cast<const uint4*>(st + xoff1);
      const uint4 xa1 = *reinterpret_cast<const uint4*>(st + xoff0 + 8 * 128);
      const uint4 xb1 = *reinterpret_cast<const uint4*>(st + xoff1 + 8 * 128);
      float4 il[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) il[v] = *reinterpret_cast<const float4*>(st + iloff + 16 * v);
      uint32_t hb0[8], hb1[8];
      const uint32_t am0 = smooth16(xa0, xb0, il, hb0);
      const uint32_t am1 = smooth16(xa1, xb1, il, hb1);
      // x_hat over the lane's own x words, for the P product
      *reinterpret_cast<uint4*>(st + xoff0) = make_uint4(hb0[0], hb0[1], hb0[2], hb0[3]);
      *reinterpret_cast<uint4*>(st + xoff1) = make_uint4(hb0[4], hb0[5], hb0[6], hb0[7]);
      *reinterpret_cast<uint4*>(st + xoff0 + 8 * 128) = make_uint4(hb1[0], hb1[1], hb1[2], hb1[3]);
      *reinterpret_cast<uint4*>(st + xoff1 + 8 * 128) = make_uint4(hb1[4], hb1[5], hb1[6], hb1[7]);
      const size_t cstep = (size_t)c;

      if constexpr (PREC == 0) {
        // one NVFP4 group of 16 per row
        const uint32_t sf0 = cvt_e4m3(__fdiv_rn(__uint_as_float(max_half(am0) << 16), six_t));
        const uint32_t sf1 = cvt_e4m3(__fdiv_rn(__uint_as_float(max_half(am1) << 16), six_t));
        const float2 r0 = rtab[sf0], r1 = rtab[sf1];
        uint2 c0 = e2m1_group(hb0, r0.x);
        uint2 c1 = e2m1_group(hb1, r1.x);
        // a zero dequantisation step codes the whole group as +0
        if (r0.y != 0.f) c0 = make_uint2(0u, 0u);
        if (r1.y != 0.f) c1 = make_uint2(0u, 0u);
        if (ok0) {
          *reinterpret_cast<uint2*>(code0 + cstep * 128) = c0;
          sc0[cstep * 4 * 512] = (uint8_t)sf0;
        }
        if (ok1) {
          *reinterpret_cast<uint2*>(code1 + cstep * 128) = c1;
          sc1[cstep * 4 * 512] = (uint8_t)sf1;
        }
      } else {
        // a quarter of an INT4 group of 64 per row: the group maximum over the
        // four lanes cq = 0..3 of each row (both rows in one word: bf16 bits of
        // non-negative values order like unsigned integers)
        uint32_t am = max_half(am0) | (max_half(am1) << 16);
        am = max_u16x2(am, __shfl_xor_sync(0xffffffffu, am, 8));
        am = max_u16x2(am, __shfl_xor_sync(0xffffffffu, am, 16));
        const uint32_t sb0 = f32_to_bf16_bits(__fdiv_rn(__uint_as_float(am << 16), 7.0f));
        const uint32_t sb1 = f32_to_bf16_bits(__fdiv_rn(__uint_as_float(am & 0xFFFF0000u), 7.0f));
        auto quant = [&](const uint32_t (&hb)[8], uint32_t sb) {
          const float sfv = bf16_bits_to_f32(sb);
          uint2 code = make_uint2(0u, 0u);
          if (sfv != 0.f) {
            const float inv = __frcp_rn(sfv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float q0, q1;
              mul2(__uint_as_float(hb[j] << 16), __uint_as_float(hb[j] & 0xFFFF0000u), inv, inv, q0, q1);
              const int i0 = max(-8, min(7, __float2int_rn(q0)));
              const int i1 = max(-8, min(7, __float2int_rn(q1)));
              const uint32_t byte = ((uint32_t)i0 & 0xFu) | (((uint32_t)i1 & 0xFu) << 4);
              if (j < 4) code.x |= byte << (8 * j);
              else code.y |= byte << (8 * (j - 4));
            }
          }
          return code;
        };
        const uint2 c0 = quant(hb0, sb0), c1 = quant(hb1, sb1);
        if (ok0) {
          *reinterpret_cast<uint2*>(code0 + cstep * 128) = c0;
          if (cq == 0) *reinterpret_cast<uint16_t*>(sc0 + cstep * 8) = (uint16_t)sb0;
        }
        if (ok1) {
          *reinterpret_cast<uint2*>(code1 + cstep * 128) = c1;
          if (cq == 0) *reinterpret_cast<uint16_t*>(sc1 + cstep * 8) = (uint16_t)sb1;
        }
      }

      if constexpr (NT > 0) {
        __syncwarp();
        // this block's share of P: x_hat[16 x 64] times rows kp*64 .. of the L1 tile
        const uint32_t sb = smem_u32(st);
        const uint32_t l1base = sb + kXBytes;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(sb + aoff + (((2 * ks + ab) ^ (ar & 7)) << 4), a0, a1, a2, a3);
          const int k0 = kp * 64 + ks * 16;
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
  named_sync(1, CW * 32);
  // after a timed-out stage, copies may still be landing in the stages: write
  // nothing more
  if (*abort_flag) return;
  if constexpr (NT > 0) {
    // fixed-order reduction of the partial sums, then one bf16 rounding
    const int part = phase * kKParts + kp;
    const int g = lane >> 2, t4 = lane & 3;
    float* rb = red + (size_t)part * kRows * kR;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int j = t * 8 + 2 * t4;
      *reinterpret_cast<float2*>(rb + (rt * 16 + g) * kR + j) = make_float2(acc[t][0], acc[t][1]);
      *reinterpret_cast<float2*>(rb + (rt * 16 + g + 8) * kR + j) = make_float2(acc[t][2], acc[t][3]);
    }
    named_sync(1, CW * 32);
    for (int e = threadIdx.x; e < kRows * kR; e += CW * 32) {
      const int er = e / kR, j = e % kR;
      const int mm = row0 + er;
      if (mm >= M) continue;
      float v = red[e];
#pragma unroll
      for (int q = 1; q < C::kParts; ++q) v += red[q * kRows * kR + e];
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
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(k), (int)C::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.M + kRows - 1) / kRows);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k, tm_x, tm_l1, a, err, wait_ns);
  if (e != cudaSuccess) return e;
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
