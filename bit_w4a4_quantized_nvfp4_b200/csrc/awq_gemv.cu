// K3 at one or two activation rows — the AWQ W4A16 GEMV of the modulation /
// adaptive-norm projections (blog "Introducing Nunchaku 4-bit inference in
// Diffusers", section "Introducing Nunchaku Lite": these projections are
// memory-bound). The weight stream is the whole cost, so the arithmetic per
// weight is cut to what the stream can hide:
//
// * Unpacking in fp16 without any offset: a nibble at bits 0-3 (16-19) of a
//   word, masked out, IS the fp16 subnormal q * 2^-24; one at bits 4-7
//   (20-23) is 16 q * 2^-24. One shift by 8 brings the upper byte's nibbles
//   down, so the 8 nibbles of a word give four fp16 pairs (k, k+4) with one
//   shift and four and operations. The activations of the odd pairs are
//   stored divided by 16, so every product is q x 2^-24, exact in fp32, and
//   the tensor cores (mma.sync m16n8k16, f16 inputs, fp32 accumulation) form
//   C_g = 2^-24 sum_k q_k x_k per group. The zero point needs the group sum
//   X_g = sum_k x_k once per group:
//       sum_k (q_k - z_g) x_k = 2^24 C_g - z_g X_g.
// * Activations in fp16, exactly: every group of 64 values of a row is
//   scaled by a power of two 2^e that puts its largest magnitude in
//   [2^14, 2^15) (bf16 has 8 significant bits, fp16 11), and the group's
//   result is scaled back by 2^-e together with the group scale.
// * All eight columns of the MMA do useful work at M = 1: column c of the
//   B operand (A = 16 weight rows) holds the activations of group c only
//   (zeros elsewhere), so one accumulator tile collects eight groups' dot
//   products at once and each group's scale is applied once per 8 x 64
//   weights of a row, not per MMA. At M = 2 the columns are (row m, group)
//   for four groups. An MMA's result is ready some 90 cycles after issue,
//   and the pipe takes one every ~8 cycles per SM sub-partition, so each
//   warp keeps four independent accumulator chains and issues them
//   interleaved (the MMAs are volatile, so their order is kept).
//
// Data movement: a producer warp streams 64-row x 512-K weight stages (two
// 64 x 256-K boxes, 128-byte swizzle, 16 KB) through a 4-stage TMA ring with
// full/empty mbarriers; two warp groups (stage phases) take alternate stages,
// four row tiles of 16 rows each; the CTA's activations, scales and zero
// points are bulk-copied into shared memory once, the activations on one
// barrier and the scales and zero points on another, so that the activation
// conversion starts as soon as x has landed and the scales are waited for
// only before a group's result is first scaled. With programmatic dependent
// launch the CTA's first weight stages and its scales and zero points are
// prefetched into L2 before the wait for the previous kernel in the stream (a
// prefetch only moves data closer, L2 being the point of coherence) and
// nothing is read into the SM before it; the later stages are prefetched
// right after the first loads.
//
// K order inside a group: the lane that owns a group's 32 bytes of a row uses
// its nibbles as pairs (8j+i, 8j+i+4), j = word, i = 0..3; every 8-element
// block of x is stored as the fp16 pairs (0,4) (1,5)/16 (2,6) (3,7)/16, so the
// dot product is unchanged. The eight 16-byte blocks of group g sit at block
// positions j ^ (g & 7), so that the lanes that read block j of eight groups
// hit different banks; the lanes whose B entries are zero load nothing.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRowsG = 64;                  // weight rows (output columns) per CTA
constexpr int kStageKG = 512;               // K per stage: 8 groups, two 256-K boxes
constexpr int kBoxBytesG = kRowsG * 128;    // one 64-row x 128-byte box: 8 KB
constexpr int kStageBytesG = 2 * kBoxBytesG;
constexpr int kPhasesG = 2;                 // warp groups taking alternate stages
constexpr int kStagesG = 4;                 // a multiple of kPhasesG
constexpr int kComputeWarpsG = 4 * kPhasesG;
constexpr int kThreadsG = (kComputeWarpsG + 1) * 32;
constexpr int kGemvSmemLimit = 232448;
static_assert(kStagesG % kPhasesG == 0, "a stage is reused by one warp group only");

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// f16x2 of (hi, lo) rounded to nearest
__device__ __forceinline__ uint32_t f16x2(float hi, float lo) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// the 8 nibbles of w (k = 0..7 of a run) -> fp16 pairs (q_i, q_{i+4}) x 2^-24
// for i = 0, 2 and x 16 * 2^-24 for i = 1, 3 (subnormals, exact)
struct Pairs {
  uint32_t p[4];
};
__device__ __forceinline__ Pairs unpack8(uint32_t w) {
  const uint32_t v = w >> 8;
  Pairs r;
  r.p[0] = w & 0x000F000Fu;
  r.p[1] = w & 0x00F000F0u;
  r.p[2] = v & 0x000F000Fu;
  r.p[3] = v & 0x00F000F0u;
  return r;
}

// 16 bytes of shared memory into v if pred, else v unchanged (its zeros stay)
__device__ __forceinline__ void lds128_if(uint32_t (&v)[4], bool pred, uint32_t addr) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t@p ld.shared.v4.b32 {%0, %1, %2, %3}, [%5];\n\t}"
      : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3])
      : "r"((uint32_t)pred), "r"(addr));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

struct GemvLayout {
  int kp;        // K padded to whole stages
  int ngp;       // groups of kp
  int x_pitch;   // bytes per activation row (2 kp)
  int sz_pitch;  // bytes per weight row of scales / zero points (2 ng)
  int off_x, off_xs, off_s, off_z, off_red, off_bar, total;
  __host__ __device__ GemvLayout(int M, int K) {
    kp = ((K + kStageKG - 1) / kStageKG) * kStageKG;
    ngp = kp / 64;
    x_pitch = 2 * kp;
    sz_pitch = 2 * (K / 64);
    off_x = kStagesG * kStageBytesG;
    off_xs = off_x + M * x_pitch;                   // {2^-e, X'} per (row, group), fp32 [M][ngp][2]
    off_s = off_xs + M * ngp * 8;
    off_z = off_s + ((kRowsG * sz_pitch + 15) / 16) * 16;
    off_red = off_z + ((kRowsG * sz_pitch + 15) / 16) * 16;
    off_bar = off_red + (kPhasesG - 1) * 4 * 32 * 2 * 4;
    total = off_bar + 2 * kStagesG * 8 + 8 + 8 + 8;
  }
};

// MT = 1, 2 or 4: the rows of the MMA's eight columns (eight groups per
// column block at MT = 1, four at MT = 2, two at MT = 4); the launch's a.M <= MT
// rows are real, the rest zeros.
template <int MT>
__global__ void __launch_bounds__(kThreadsG, 2)
awq_gemv_kernel(const __grid_constant__ CUtensorMap tm_q, AwqArgs a, unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align<1024>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, N = a.N;
  const int ng = K / 64;
  const int nst = (K + kStageKG - 1) / kStageKG;
  const int n0 = blockIdx.x * kRowsG;
  const int M = a.M;
  const GemvLayout L(MT, K);
  uint8_t* xs = base + L.off_x;
  float2* xgs = reinterpret_cast<float2*>(base + L.off_xs);  // {2^-e, sum of the group's x 2^e}
  const uint16_t* ss = reinterpret_cast<const uint16_t*>(base + L.off_s);
  const uint16_t* zs = reinterpret_cast<const uint16_t*>(base + L.off_z);
  float* red = reinterpret_cast<float*>(base + L.off_red);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.off_bar);
  uint64_t* empty = full + kStagesG;
  uint64_t* xbar = empty + kStagesG;
  uint64_t* szbar = xbar + 1;
  int* abort_flag = reinterpret_cast<int*>(szbar + 1);
  const uint32_t sz_bytes = (uint32_t)(min(kRowsG, N - n0) * L.sz_pitch);

  if (threadIdx.x == 0) launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesG; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    mbar_init(xbar, 1);
    mbar_init(szbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kComputeWarpsG && lane == 0) {
    // Only hints before the previous kernel in the stream has finished: the
    // tensor map, the first weight stages and this CTA's scales and zero
    // points are pulled towards L2.
    tma_prefetch_desc(&tm_q);
    for (int c = 0; c < nst && c < kStagesG; ++c) {
      tma_prefetch_l2_2d(&tm_q, c * (kStageKG / 2), n0);
      tma_prefetch_l2_2d(&tm_q, c * (kStageKG / 2) + 128, n0);
    }
    bulk_prefetch_l2(a.s + (size_t)n0 * ng, sz_bytes);
    bulk_prefetch_l2(a.z + (size_t)n0 * ng, sz_bytes);
  }
  __syncthreads();
  grid_dependency_wait();

  if (warp == kComputeWarpsG) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int c = 0;
      bool ok = true;
      auto issue_stage = [&](int cc) {
        const int s = cc % kStagesG;
        uint8_t* dst = base + s * kStageBytesG;
        mbar_expect_tx(&full[s], kStageBytesG);
        tma_load_2d(dst, &tm_q, &full[s], cc * (kStageKG / 2), n0);
        tma_load_2d(dst + kBoxBytesG, &tm_q, &full[s], cc * (kStageKG / 2) + 128, n0);
      };
      mbar_expect_tx(xbar, (uint32_t)(M * 2 * K));
      for (int m = 0; m < M; ++m) bulk_load(xs + m * L.x_pitch, a.x + (size_t)m * K, (uint32_t)(2 * K), xbar);
      mbar_expect_tx(szbar, 2 * sz_bytes);
      bulk_load(base + L.off_s, a.s + (size_t)n0 * ng, sz_bytes, szbar);
      bulk_load(base + L.off_z, a.z + (size_t)n0 * ng, sz_bytes, szbar);
      for (; c < nst && c < kStagesG; ++c) issue_stage(c);
      for (int cc = kStagesG; cc < nst; ++cc) {
        tma_prefetch_l2_2d(&tm_q, cc * (kStageKG / 2), n0);
        tma_prefetch_l2_2d(&tm_q, cc * (kStageKG / 2) + 128, n0);
      }
      for (; c < nst; ++c) {
        const int s = c % kStagesG;
        if (!mbar_wait(&empty[s], ((c / kStagesG) - 1) & 1, wait_ns, err)) {
          ok = false;
          break;
        }
        issue_stage(c);
      }
      // let the copies already issued land before the CTA can exit (bounded)
      (void)mbar_wait(xbar, 0, wait_ns, ok ? err : nullptr);
      (void)mbar_wait(szbar, 0, wait_ns, ok ? err : nullptr);
      if (!ok)
        for (int j = max(0, c - kStagesG); j < c; ++j)
          (void)mbar_wait(&full[j % kStagesG], (j / kStagesG) & 1, wait_ns, nullptr);
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  bool ok = __all_sync(0xffffffffu, mbar_wait(xbar, 0, wait_ns, err));
  if (ok) {
    // per (row, group), four threads of a warp, two 16-byte blocks (16
    // values) each: 2^e from the group's largest magnitude, then the values
    // as fp16 x 2^e (odd pairs / 16) in pair order, written back in place to
    // block position j ^ (g & 7) (so that lanes reading block j of eight
    // consecutive groups hit different banks), and the group's sum of x 2^e;
    // groups past K are zeros
    const int total = MT * L.ngp * 4;
    for (int base0 = 0; base0 < total; base0 += kComputeWarpsG * 32) {
      const int idx = base0 + threadIdx.x;
      const bool valid = idx < total;
      const int jp = idx & 3, gt = idx >> 2;
      const int m = valid ? gt / L.ngp : 0, g = valid ? gt % L.ngp : 0;
      const bool live = valid && g < ng && m < M;
      uint4* grp = reinterpret_cast<uint4*>(xs + m * L.x_pitch + 128 * g);
      uint4 u[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) u[h] = live ? grp[2 * jp + h] : make_uint4(0, 0, 0, 0);
      // per-half unsigned maxima of the magnitude bits (bf16 order = magnitude order)
      uint32_t m2 = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h)
        m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(u[h].x & 0x7FFF7FFFu, u[h].y & 0x7FFF7FFFu),
                                   __vmaxu2(u[h].z & 0x7FFF7FFFu, u[h].w & 0x7FFF7FFFu)));
      uint32_t amax = max(m2 & 0xFFFFu, m2 >> 16);
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // bf16 biased exponent E: |x| < 2^(E - 126), so 2^(141 - E) puts the
      // largest magnitude in [2^14, 2^15); clamped so both powers are normal
      const int ex = min(max(141 - (int)(amax >> 7), -126), 126);
      const float sc = __uint_as_float((uint32_t)(ex + 127) << 23);
      uint4 outv[2];
      float gsum = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t w[4] = {u[h].x, u[h].y, u[h].z, u[h].w};
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[2 * e] = bf16_bits_to_f32(w[e] & 0xFFFFu) * sc;
          v[2 * e + 1] = bf16_bits_to_f32(w[e] >> 16) * sc;
        }
        gsum += ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
        outv[h] = make_uint4(f16x2(v[4], v[0]), f16x2(v[5] * 0.0625f, v[1] * 0.0625f), f16x2(v[6], v[2]),
                             f16x2(v[7] * 0.0625f, v[3] * 0.0625f));
      }
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 1);
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 2);
      // every lane of the group has read its blocks (the shuffles above
      // consumed the loaded values) before any lane overwrites one
      if (valid) {
#pragma unroll
        for (int h = 0; h < 2; ++h) grp[(2 * jp + h) ^ (g & 7)] = outv[h];
      }
      if (valid && jp == 0) xgs[m * L.ngp + g] = make_float2(__uint_as_float((uint32_t)(127 - ex) << 23), gsum);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarpsG * 32) : "memory");

  const int rt = warp & 3, kh = warp >> 2;  // row tile, stage phase
  const int gid = lane >> 2, t = lane & 3;
  const int r_lo = rt * 16 + gid, r_hi = r_lo + 8;
  const int n_lo = n0 + r_lo, n_hi = n0 + r_hi;
  const int pl = r_lo * ng, ph = r_hi * ng;  // rows of the scale / zero-point tables
  // Column c of the accumulator tile is batch row c / G, group c % G of the
  // column block. This lane's columns 2t and 2t + 1: at G >= 2 both in batch
  // row m_c (groups 2t % G and 2t % G + 1).
  constexpr int G = 8 / MT;
  const int m_c = (2 * t) / G;
  const int gi0 = (2 * t) % G;
  float tot_lo = 0.f, tot_hi = 0.f;

  // columns 2t, 2t+1 of the tile are groups ga, ga + 1 of the block starting
  // at group gb0 (batch row m_c): y += s 2^-e (2^24 C - z X')
  auto finish = [&](const float (&c)[4], int gb0) {
    const int ga = gb0 + gi0, gb = ga + 1;
    const int ga_c = min(ga, ng - 1), gb_c = min(gb, ng - 1);
    const float2 xa = xgs[m_c * L.ngp + ga], xb = xgs[m_c * L.ngp + gb];
    const float t0 = fmaf(16777216.f, c[0], -bf16_bits_to_f32(zs[pl + ga_c]) * xa.y);
    const float t1 = fmaf(16777216.f, c[1], -bf16_bits_to_f32(zs[pl + gb_c]) * xb.y);
    const float t2 = fmaf(16777216.f, c[2], -bf16_bits_to_f32(zs[ph + ga_c]) * xa.y);
    const float t3 = fmaf(16777216.f, c[3], -bf16_bits_to_f32(zs[ph + gb_c]) * xb.y);
    tot_lo = fmaf(bf16_bits_to_f32(ss[pl + ga_c]) * xa.x, t0, tot_lo);
    tot_lo = fmaf(bf16_bits_to_f32(ss[pl + gb_c]) * xb.x, t1, tot_lo);
    tot_hi = fmaf(bf16_bits_to_f32(ss[ph + ga_c]) * xa.x, t2, tot_hi);
    tot_hi = fmaf(bf16_bits_to_f32(ss[ph + gb_c]) * xb.x, t3, tot_hi);
  };
  auto ld_w = [&](const uint8_t* box, int r, int ch) {
    return *reinterpret_cast<const uint4*>(box + r * 128 + ((ch ^ (r & 7)) << 4));
  };

  bool sz_ready = false;
  for (int c = kh; c < nst && ok; c += kPhasesG) {
    const int s = c % kStagesG;
    if (!warp_wait(&full[s], (c / kStagesG) & 1, wait_ns, err)) {
      ok = false;
      break;
    }
    const uint8_t* st = base + s * kStageBytesG;
    const int g0 = c * 8;
    float keep = 0.f;
    if constexpr (MT == 1) {
      // lane (gid, t): rows r_lo, r_hi, groups t (box 0) and t + 4 (box 1);
      // B column gid holds group gid: lane (gid, t) supplies it in its first
      // register when gid == t and in its second when gid == t + 4, and zeros
      // otherwise (those lanes load nothing)
      const int ga = g0 + t, gb = g0 + t + 4;
      const uint32_t xa_base = smem_u32(xs + 128 * ga), xb_base = smem_u32(xs + 128 * gb);
      const bool a_act = gid == t, b_act = gid == t + 4;
      // x blocks double-buffered: block j + 1 is loaded before block j's MMAs
      uint32_t xa[2][4] = {}, xb[2][4] = {};
      lds128_if(xa[0], a_act, xa_base + ((0 ^ (ga & 7)) << 4));
      lds128_if(xb[0], b_act, xb_base + ((0 ^ (gb & 7)) << 4));
      float acc[4][4] = {};
      uint4 L0, H0, L1, H1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if ((j & 3) == 0) {  // the 16-byte half j / 4 of each group's 32 bytes
          const int h = j >> 2;
          L0 = ld_w(st, r_lo, 2 * t + h);
          H0 = ld_w(st, r_hi, 2 * t + h);
          L1 = ld_w(st + kBoxBytesG, r_lo, 2 * t + h);
          H1 = ld_w(st + kBoxBytesG, r_hi, 2 * t + h);
        }
        if (j + 1 < 8) {
          lds128_if(xa[(j + 1) & 1], a_act, xa_base + (((j + 1) ^ (ga & 7)) << 4));
          lds128_if(xb[(j + 1) & 1], b_act, xb_base + (((j + 1) ^ (gb & 7)) << 4));
        }
        const int jj = j & 3;
        const Pairs al0 = unpack8(word_of(L0, jj)), ah0 = unpack8(word_of(H0, jj));
        const Pairs al1 = unpack8(word_of(L1, jj)), ah1 = unpack8(word_of(H1, jj));
#pragma unroll
        for (int i = 0; i < 4; ++i)
          mma_f16(acc[i], al0.p[i], ah0.p[i], al1.p[i], ah1.p[i], xa[j & 1][i], xb[j & 1][i]);
      }
      float cc[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) cc[e] = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
      keep = cc[0] + cc[1] + cc[2] + cc[3];
      if (!sz_ready) {
        if (!warp_wait(szbar, 0, wait_ns, err)) { ok = false; break; }
        sz_ready = true;
      }
      finish(cc, g0);
    } else {
      // blocks of G groups (8 / G per stage, each inside one box). Lane
      // (gid, t): rows r_lo, r_hi, group gl = t % G of the block, share
      // sigma = t / G of that group's 8 words (W = 2G words: all of them at
      // G = 4, half at G = 2). B column gid = (batch row gid / G, group
      // gid % G): lane (gid, t) supplies the activations of its slot pairs
      // when gid % G == gl, from the same share.
      constexpr int W = 2 * G;
      const int gl = t % G, sigma = t / G;
      const bool act = (gid % G) == gl;
      const int xm = gid / G;
#pragma unroll
      for (int kbl = 0; kbl < 8 / G; ++kbl) {
        const int gb0 = g0 + G * kbl;
        const uint8_t* box = st + ((G * kbl) >> 2) * kBoxBytesG;
        const int gib = ((G * kbl) & 3) + gl;  // the lane's group within the box
        const int gx = gb0 + gl;
        const uint32_t x_base = smem_u32(xs + xm * L.x_pitch + 128 * gx);
        // x blocks double-buffered: block j + 1 is loaded before block j's MMAs
        uint32_t v[2][4] = {};
        lds128_if(v[0], act, x_base + (((sigma * W) ^ (gx & 7)) << 4));
        float acc[4][4] = {};
        uint4 Lw, Hw;
#pragma unroll
        for (int j = 0; j < W; ++j) {
          if ((j & 3) == 0) {  // the 16-byte chunk holding words sigma W + j ..
            const int ch = 2 * gib + (sigma * W + j) / 4;
            Lw = ld_w(box, r_lo, ch);
            Hw = ld_w(box, r_hi, ch);
          }
          if (j + 1 < W) lds128_if(v[(j + 1) & 1], act, x_base + (((sigma * W + j + 1) ^ (gx & 7)) << 4));
          const int jj = j & 3;
          const Pairs pl_ = unpack8(word_of(Lw, jj)), ph_ = unpack8(word_of(Hw, jj));
          const uint32_t(&vv)[4] = v[j & 1];
          mma_f16(acc[2 * (j & 1)], pl_.p[0], ph_.p[0], pl_.p[1], ph_.p[1], vv[0], vv[1]);
          mma_f16(acc[2 * (j & 1) + 1], pl_.p[2], ph_.p[2], pl_.p[3], ph_.p[3], vv[2], vv[3]);
        }
        float cc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) cc[e] = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
        keep += cc[0] + cc[1] + cc[2] + cc[3];
        if (!sz_ready) {
          if (!warp_wait(szbar, 0, wait_ns, err)) { ok = false; break; }
          sz_ready = true;
        }
        finish(cc, gb0);
      }
    }
    // release the stage only once its weights have gone through the MMAs
    consumed(keep);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // lanes of one row and batch row: MT = 1 all four of a quad, MT = 2 pairs,
  // MT = 4 each lane its own batch row
  if constexpr (MT <= 2) {
    tot_lo += __shfl_xor_sync(0xffffffffu, tot_lo, 1);
    tot_hi += __shfl_xor_sync(0xffffffffu, tot_hi, 1);
  }
  if constexpr (MT == 1) {
    tot_lo += __shfl_xor_sync(0xffffffffu, tot_lo, 2);
    tot_hi += __shfl_xor_sync(0xffffffffu, tot_hi, 2);
  }
  if (!ok && lane == 0) *abort_flag = 1;
  if (kh > 0) {
    float* rb = red + (size_t)((kh - 1) * 4 + rt) * 32 * 2;
    rb[2 * lane] = tot_lo;
    rb[2 * lane + 1] = tot_hi;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarpsG * 32) : "memory");
  if (*abort_flag || kh > 0) return;
#pragma unroll
  for (int q = 1; q < kPhasesG; ++q) {
    const float* rb = red + (size_t)((q - 1) * 4 + rt) * 32 * 2;
    tot_lo += rb[2 * lane];
    tot_hi += rb[2 * lane + 1];
  }
  const bool writer = (2 * t) % G == 0 && m_c < M;
  if (!writer) return;
  if (n_lo < N) {
    const float bb = a.bias ? bf16_bits_to_f32(a.bias[n_lo]) : 0.f;
    a.y[(size_t)m_c * N + n_lo] = (uint16_t)f32_to_bf16_bits(__fadd_rn(tot_lo, bb));
  }
  if (n_hi < N) {
    const float bb = a.bias ? bf16_bits_to_f32(a.bias[n_hi]) : 0.f;
    a.y[(size_t)m_c * N + n_hi] = (uint16_t)f32_to_bf16_bits(__fadd_rn(tot_hi, bb));
  }
}

}  // namespace

static int gemv_rows(int M) { return M <= 2 ? M : 4; }

bool awq_gemv_fits(int M, int K) {
  return M >= 1 && M <= 4 && (size_t)GemvLayout(gemv_rows(M), K).total + 1024 <= (size_t)kGemvSmemLimit;
}

cudaError_t launch_awq_gemv(const AwqArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  if (!awq_gemv_fits(a.M, a.K)) return cudaErrorInvalidValue;
  const int mt = gemv_rows(a.M);
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q, (uint64_t)a.K / 2, (uint64_t)a.N, (uint64_t)a.K / 2,
                    128, kRowsG, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)GemvLayout(mt, a.K).total + 1024;
  auto kern = mt == 1 ? awq_gemv_kernel<1> : (mt == 2 ? awq_gemv_kernel<2> : awq_gemv_kernel<4>);
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((a.N + kRowsG - 1) / kRowsG);
  cfg.blockDim = dim3(kThreadsG);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm_q, a, err, wait_ns);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace svdq
