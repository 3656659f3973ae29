// K3 at one or two activation rows — the AWQ W4A16 GEMV of the modulation /
// adaptive-norm projections (blog "Introducing Nunchaku 4-bit inference in
// Diffusers", section "Introducing Nunchaku Lite": these projections are
// memory-bound). The weight stream is the whole cost, so the arithmetic per
// weight is cut to what the stream can hide:
//
// * Dequantisation without the zero point: each nibble q becomes the bf16 of
//   128 + q with one mask-and-or (the 8 nibbles of a 32-bit word give four
//   bf16 pairs (k, k+4) with three shifts and four and-or operations). The
//   tensor cores then form C_g = sum_k (128 + q_k) x_k in fp32 over a group
//   g of 64, and the group's exact result follows from the activation group
//   sum X_g = sum_k x_k once per group:
//       sum_k (q_k - z_g) x_k = C_g - (128 + z_g) X_g,
//   y = sum_g s_g (C_g - (128 + z_g) X_g) + bias. Products (128 + q) x are
//   exact in fp32; C_g is ~130 |X_g| in size, so fp32 accumulation costs
//   about 2^-24 * 130 |X_g| per step, far below the bf16 output rounding.
// * All eight columns of the MMA do useful work at M = 1: column c of the
//   B operand (mma.sync m16n8k16, A = 16 weight rows) holds the activation
//   entries of group c only (zeros elsewhere), so one accumulator tile
//   collects eight groups' dot products at once and the per-group scale,
//   zero point and X_g are applied once per 8 x 64 weights of a row, not per
//   MMA. At M = 2 the columns are (row m, group) for four groups.
//
// Data movement as in the batched kernel: a producer warp streams 64-row x
// 512-K weight stages (two 64 x 256-K boxes, 128-byte swizzle, 16 KB) through
// a 4-stage TMA ring with full/empty mbarriers; two warp groups (stage
// phases) take alternate stages, four row tiles of 16 rows each; the CTA's
// activations, scales and zero points are bulk-copied into shared memory once.
// With programmatic dependent launch every weight tile of the CTA is
// prefetched into L2 before the wait for the previous kernel in the stream
// (a prefetch only moves data closer, L2 being the point of coherence) and
// nothing is read into the SM before it.
//
// K order inside a group: the lane that owns a group's 32 bytes of a row uses
// its nibbles as pairs (8j+i, 8j+i+4), j = word, i = 0..3; every 8-element
// block of x is stored as the bf16 pairs (0,4) (1,5) (2,6) (3,7) (the same
// permutation the batched kernel uses), so the dot product is unchanged.
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

__device__ __forceinline__ void mma_16816g(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// nibbles i and i+4 of w -> bf16x2 (128 + q_i, 128 + q_{i+4})
template <int I>
__device__ __forceinline__ uint32_t nib_pair(uint32_t w) {
  return ((w >> (4 * I)) & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ uint32_t word_of(const uint4& a, const uint4& b, int j) {
  const uint4& v = j < 4 ? a : b;
  const int i = j & 3;
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t prmt_g(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

struct GemvLayout {
  int kp;        // K padded to whole stages
  int ngp;       // groups of kp
  int x_pitch;   // bytes per activation row (2 kp)
  int sz_pitch;  // bytes per weight row of scales / zero points (2 ng)
  int off_x, off_xs, off_s, off_z, off_zero, off_red, off_bar, total;
  __host__ __device__ GemvLayout(int M, int K) {
    kp = ((K + kStageKG - 1) / kStageKG) * kStageKG;
    ngp = kp / 64;
    x_pitch = 2 * kp;
    sz_pitch = 2 * (K / 64);
    off_x = kStagesG * kStageBytesG;
    off_xs = off_x + M * x_pitch;                   // X_g sums, fp32 [M][ngp]
    off_s = off_xs + ((M * ngp * 4 + 15) / 16) * 16;
    off_z = off_s + ((kRowsG * sz_pitch + 15) / 16) * 16;
    off_zero = off_z + ((kRowsG * sz_pitch + 15) / 16) * 16;
    off_red = off_zero + 128;
    off_bar = off_red + (kPhasesG - 1) * 4 * 32 * 2 * 4;
    total = off_bar + 2 * kStagesG * 8 + 8 + 8;
  }
};

template <int M>
__global__ void __launch_bounds__(kThreadsG, 2)
awq_gemv_kernel(const __grid_constant__ CUtensorMap tm_q, AwqArgs a, unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, N = a.N;
  const int ng = K / 64;
  const int nst = (K + kStageKG - 1) / kStageKG;
  const int n0 = blockIdx.x * kRowsG;
  const GemvLayout L(M, K);
  uint8_t* xs = base + L.off_x;
  float* xsum = reinterpret_cast<float*>(base + L.off_xs);
  const uint16_t* ss = reinterpret_cast<const uint16_t*>(base + L.off_s);
  const uint16_t* zs = reinterpret_cast<const uint16_t*>(base + L.off_z);
  uint8_t* zero = base + L.off_zero;
  float* red = reinterpret_cast<float*>(base + L.off_red);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.off_bar);
  uint64_t* empty = full + kStagesG;
  uint64_t* xbar = empty + kStagesG;
  int* abort_flag = reinterpret_cast<int*>(xbar + 1);

  if (threadIdx.x == 0) launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesG; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kComputeWarpsG && lane == 0) {
    // Only hints before the previous kernel in the stream has finished: the
    // tensor map and every weight tile of this CTA are pulled towards L2.
    tma_prefetch_desc(&tm_q);
    for (int c = 0; c < nst; ++c) {
      tma_prefetch_l2_2d(&tm_q, c * (kStageKG / 2), n0);
      tma_prefetch_l2_2d(&tm_q, c * (kStageKG / 2) + 128, n0);
    }
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
      const uint32_t sz_bytes = (uint32_t)(min(kRowsG, N - n0) * L.sz_pitch);
      mbar_expect_tx(xbar, (uint32_t)(M * 2 * K) + 2 * sz_bytes);
      bulk_load(base + L.off_s, a.s + (size_t)n0 * ng, sz_bytes, xbar);
      bulk_load(base + L.off_z, a.z + (size_t)n0 * ng, sz_bytes, xbar);
      for (int m = 0; m < M; ++m) bulk_load(xs + m * L.x_pitch, a.x + (size_t)m * K, (uint32_t)(2 * K), xbar);
      for (; c < nst && c < kStagesG; ++c) issue_stage(c);
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
      if (!ok)
        for (int j = max(0, c - kStagesG); j < c; ++j)
          (void)mbar_wait(&full[j % kStagesG], (j / kStagesG) & 1, wait_ns, nullptr);
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  bool ok = __all_sync(0xffffffffu, mbar_wait(xbar, 0, wait_ns, err));
  if (ok) {
    // per (row, group): the group sum X_g in a fixed order, then the group's
    // 64 values permuted in place into pair order; groups past K are zeros
    for (int t = threadIdx.x; t < M * L.ngp; t += kComputeWarpsG * 32) {
      const int m = t / L.ngp, g = t % L.ngp;
      uint4* p = reinterpret_cast<uint4*>(xs + m * L.x_pitch + 128 * g);
      float sum = 0.f;
      if (g < ng) {
#pragma unroll
        for (int b = 0; b < 8; b += 2) {
          const uint4 u = p[b], v = p[b + 1];
          const uint32_t w[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) sum += bf16_bits_to_f32(w[e] & 0xFFFFu) + bf16_bits_to_f32(w[e] >> 16);
          p[b] = make_uint4(prmt_g(u.x, u.z, 0x5410u), prmt_g(u.x, u.z, 0x7632u), prmt_g(u.y, u.w, 0x5410u),
                            prmt_g(u.y, u.w, 0x7632u));
          p[b + 1] = make_uint4(prmt_g(v.x, v.z, 0x5410u), prmt_g(v.x, v.z, 0x7632u), prmt_g(v.y, v.w, 0x5410u),
                                prmt_g(v.y, v.w, 0x7632u));
        }
      } else {
#pragma unroll
        for (int b = 0; b < 8; ++b) p[b] = make_uint4(0, 0, 0, 0);
      }
      xsum[m * L.ngp + g] = sum;
    }
    if (threadIdx.x < 8) reinterpret_cast<uint4*>(zero)[threadIdx.x] = make_uint4(0, 0, 0, 0);
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarpsG * 32) : "memory");

  const int rt = warp & 3, kh = warp >> 2;  // row tile, stage phase
  const int gid = lane >> 2, t = lane & 3;
  const int r_lo = rt * 16 + gid, r_hi = r_lo + 8;
  const int n_lo = n0 + r_lo, n_hi = n0 + r_hi;
  // the two groups (columns 2t, 2t+1 of the accumulator tile) and the batch
  // row this lane's accumulator values belong to
  const int m_c = M == 1 ? 0 : (t >> 1);
  float tot_lo = 0.f, tot_hi = 0.f;

  // apply one sub-block's scales, zero points and group sums: columns 2t, 2t+1
  // of the tile are groups ga, ga + 1 (of batch row m_c)
  auto finish = [&](const float (&c)[4], int ga) {
    const int gb = ga + 1;
    const int ga_c = min(ga, ng - 1), gb_c = min(gb, ng - 1);
    const float xa = xsum[m_c * L.ngp + ga], xb = xsum[m_c * L.ngp + gb];
    const int pl = r_lo * (L.sz_pitch / 2), ph = r_hi * (L.sz_pitch / 2);
    const float s0 = bf16_bits_to_f32(ss[pl + ga_c]), s1 = bf16_bits_to_f32(ss[pl + gb_c]);
    const float s2 = bf16_bits_to_f32(ss[ph + ga_c]), s3 = bf16_bits_to_f32(ss[ph + gb_c]);
    const float z0 = bf16_bits_to_f32(zs[pl + ga_c]) + 128.f, z1 = bf16_bits_to_f32(zs[pl + gb_c]) + 128.f;
    const float z2 = bf16_bits_to_f32(zs[ph + ga_c]) + 128.f, z3 = bf16_bits_to_f32(zs[ph + gb_c]) + 128.f;
    tot_lo = fmaf(s0, fmaf(-z0, xa, c[0]), tot_lo);
    tot_lo = fmaf(s1, fmaf(-z1, xb, c[1]), tot_lo);
    tot_hi = fmaf(s2, fmaf(-z2, xa, c[2]), tot_hi);
    tot_hi = fmaf(s3, fmaf(-z3, xb, c[3]), tot_hi);
  };
  auto ld_w = [&](const uint8_t* box, int r, int ch) {
    return *reinterpret_cast<const uint4*>(box + r * 128 + ((ch ^ (r & 7)) << 4));
  };

  for (int c = kh; c < nst && ok; c += kPhasesG) {
    const int s = c % kStagesG;
    if (!warp_wait(&full[s], (c / kStagesG) & 1, wait_ns, err)) {
      ok = false;
      break;
    }
    const uint8_t* st = base + s * kStageBytesG;
    const int g0 = c * 8;
    float keep = 0.f;
    if constexpr (M == 1) {
      // lane (gid, t): rows r_lo, r_hi, groups t (box 0) and t + 4 (box 1);
      // B column gid holds group gid: lane (gid, t) supplies it in its first
      // register when gid == t and in its second when gid == t + 4
      const uint8_t* xa_src = gid == t ? xs + 128 * (g0 + t) : zero;
      const uint8_t* xb_src = gid == t + 4 ? xs + 128 * (g0 + t + 4) : zero;
      float ca[4] = {0.f, 0.f, 0.f, 0.f}, cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // the 16-byte half h of each group's 32 bytes
        const uint4 L0 = ld_w(st, r_lo, 2 * t + h), H0 = ld_w(st, r_hi, 2 * t + h);
        const uint4 L1 = ld_w(st + kBoxBytesG, r_lo, 2 * t + h), H1 = ld_w(st + kBoxBytesG, r_hi, 2 * t + h);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = 4 * h + jj;
          const uint4 xa = *reinterpret_cast<const uint4*>(xa_src + 16 * j);
          const uint4 xb = *reinterpret_cast<const uint4*>(xb_src + 16 * j);
          const uint32_t wl0 = word_of(L0, L0, jj), wh0 = word_of(H0, H0, jj);
          const uint32_t wl1 = word_of(L1, L1, jj), wh1 = word_of(H1, H1, jj);
          float(&acc)[4] = (j & 1) ? cb : ca;
          mma_16816g(acc, nib_pair<0>(wl0), nib_pair<0>(wh0), nib_pair<0>(wl1), nib_pair<0>(wh1), xa.x, xb.x);
          mma_16816g(acc, nib_pair<1>(wl0), nib_pair<1>(wh0), nib_pair<1>(wl1), nib_pair<1>(wh1), xa.y, xb.y);
          mma_16816g(acc, nib_pair<2>(wl0), nib_pair<2>(wh0), nib_pair<2>(wl1), nib_pair<2>(wh1), xa.z, xb.z);
          mma_16816g(acc, nib_pair<3>(wl0), nib_pair<3>(wh0), nib_pair<3>(wl1), nib_pair<3>(wh1), xa.w, xb.w);
        }
      }
      const float cc[4] = {ca[0] + cb[0], ca[1] + cb[1], ca[2] + cb[2], ca[3] + cb[3]};
      keep = cc[0] + cc[1] + cc[2] + cc[3];
      finish(cc, g0 + 2 * t);
    } else {
      // two sub-blocks of four groups (one box each); lane (gid, t): rows
      // r_lo, r_hi, group t of the box; B column gid = (row gid / 4, group gid % 4)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const uint8_t* box = st + b * kBoxBytesG;
        const int gb0 = g0 + 4 * b;
        const uint4 La = ld_w(box, r_lo, 2 * t), Lb = ld_w(box, r_lo, 2 * t + 1);
        const uint4 Ha = ld_w(box, r_hi, 2 * t), Hb = ld_w(box, r_hi, 2 * t + 1);
        const uint8_t* x_src = (gid & 3) == t ? xs + (gid >> 2) * L.x_pitch + 128 * (gb0 + t) : zero;
        float ca[4] = {0.f, 0.f, 0.f, 0.f}, cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(x_src + 16 * j);
          const uint32_t wl = word_of(La, Lb, j), wh = word_of(Ha, Hb, j);
          mma_16816g(ca, nib_pair<0>(wl), nib_pair<0>(wh), nib_pair<1>(wl), nib_pair<1>(wh), v.x, v.y);
          mma_16816g(cb, nib_pair<2>(wl), nib_pair<2>(wh), nib_pair<3>(wl), nib_pair<3>(wh), v.z, v.w);
        }
        const float cc[4] = {ca[0] + cb[0], ca[1] + cb[1], ca[2] + cb[2], ca[3] + cb[3]};
        keep += cc[0] + cc[1] + cc[2] + cc[3];
        finish(cc, gb0 + 2 * (t & 1));
      }
    }
    // release the stage only once its weights have gone through the MMAs
    consumed(keep);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // lanes of one row and batch row: M = 1 all four of a quad, M = 2 pairs
  tot_lo += __shfl_xor_sync(0xffffffffu, tot_lo, 1);
  tot_hi += __shfl_xor_sync(0xffffffffu, tot_hi, 1);
  if constexpr (M == 1) {
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
  for (int ph = 1; ph < kPhasesG; ++ph) {
    const float* rb = red + (size_t)((ph - 1) * 4 + rt) * 32 * 2;
    tot_lo += rb[2 * lane];
    tot_hi += rb[2 * lane + 1];
  }
  const bool writer = M == 1 ? t == 0 : (t & 1) == 0;
  if (!writer) return;
  if (n_lo < N) {
    const float b = a.bias ? bf16_bits_to_f32(a.bias[n_lo]) : 0.f;
    a.y[(size_t)m_c * N + n_lo] = (uint16_t)f32_to_bf16_bits(__fadd_rn(tot_lo, b));
  }
  if (n_hi < N) {
    const float b = a.bias ? bf16_bits_to_f32(a.bias[n_hi]) : 0.f;
    a.y[(size_t)m_c * N + n_hi] = (uint16_t)f32_to_bf16_bits(__fadd_rn(tot_hi, b));
  }
}

}  // namespace

cudaError_t launch_awq_gemv(const AwqArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  if (a.M < 1 || a.M > 2) return cudaErrorInvalidValue;
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q, (uint64_t)a.K / 2, (uint64_t)a.N, (uint64_t)a.K / 2,
                    128, kRowsG, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)GemvLayout(a.M, a.K).total + 1024;
  if (smem > (size_t)kGemvSmemLimit) return cudaErrorInvalidValue;
  auto kern = a.M == 1 ? awq_gemv_kernel<1> : awq_gemv_kernel<2>;
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
