// K3 — AWQ W4A16 linear: INT4 weights (asymmetric, bf16 scale/zero per 64
// along K) times bf16 activations, for the memory-bound modulation /
// adaptive-norm projections (blog "Introducing Nunchaku 4-bit inference in
// Diffusers", section "Introducing Nunchaku Lite").
//
// At small M the weight stream is the whole cost, so the kernel is built to
// keep HBM busy: a producer warp streams 64-row x 256-K weight boxes (8 KB,
// 128-byte swizzle) through an 8-stage TMA pipeline, so that every SM has
// 100+ KB of weight reads in flight, and eight compute warps consume them
// from shared memory (full/empty mbarriers; the stage count is even and the
// two warp groups take alternate stages, so a stage is only refilled for the
// group that released it).
//
// Compute warp (row tile rt of 16 weight rows, stage phase kh): per 64-group
// it unpacks its two rows' nibbles to bf16 with bit operations ((128 + q) has
// an exact bf16 encoding; subtracting 128 + z leaves q - z exactly) and lets
// the tensor cores (mma.sync m16n8k16, fp32 accumulate) form the dot products
// with the activations; each group's partial sums are scaled by the group
// scale in fp32. The two phases' partial sums are added in a fixed order.
//
// K order inside a group: lane t of a row quad owns k = 16t .. 16t+15 (one
// 8-byte shared load per row). Its nibbles are used in pairs (k, k+4), fed to
// the MMA K slots in the order (0,4),(1,5) | (2,6),(3,7) | (8,12),(9,13) |
// (10,14),(11,15) for the four k16 steps; the activation fragments are built
// in the same order from two 16-byte loads of x, so the dot product is
// unchanged.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRowsA = 64;                          // weight rows (output columns) per CTA
constexpr int kStageK = 256;                        // K per stage: 4 groups, 128 bytes per row
constexpr int kStageBytesA = kRowsA * kStageK / 2;  // 8 KB
constexpr int kStagesA = 8;                         // even: see the header comment
constexpr int kComputeWarps = 8;                    // 4 row tiles x 2 stage phases
constexpr int kThreadsA = (kComputeWarps + 1) * 32;
constexpr int kMaxM = 16;                           // batch rows per launch (two m-tiles of 8)
static_assert(kStagesA % 2 == 0, "a stage is reused by one warp group only");

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// nibbles k and k+4 of `w` (k = sh/4) -> bf16x2 of (q - z); zz = bf16x2 of 128 + z
__device__ __forceinline__ uint32_t deq_pair(uint32_t w, int sh, uint32_t zz) {
  const uint32_t v = ((w >> sh) & 0x000F000Fu) | 0x43004300u;
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(zz));
  return r;
}

// byte permute: selector 0x5410 gives (a.lo, b.lo), 0x7632 gives (a.hi, b.hi)
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

struct SmemA {
  uint8_t stage[kStagesA][kStageBytesA];  // 1024-aligned
  float red[4][2][32][4];                 // phase-1 partial sums [rt][mt][lane][c]
  uint64_t full[kStagesA], empty[kStagesA];
  int abort_flag;
};

__global__ void __launch_bounds__(kThreadsA, 2)
awq_kernel(const __grid_constant__ CUtensorMap tm_q, AwqArgs a, unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  SmemA& sm = *reinterpret_cast<SmemA*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, N = a.N, M = a.M;
  const int ng = K / 64;
  const int nst = (K + kStageK - 1) / kStageK;
  const int n0 = blockIdx.x * kRowsA;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 4);
    }
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int c = 0;
      bool ok = true;
      for (; c < nst; ++c) {
        const int s = c % kStagesA;
        if (c >= kStagesA && !mbar_wait(&sm.empty[s], ((c / kStagesA) - 1) & 1, wait_ns, err)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&sm.full[s], kStageBytesA);
        tma_load_2d(sm.stage[s], &tm_q, &sm.full[s], c * (kStageK / 2), n0);
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit (bounded)
        for (int j = max(0, c - kStagesA); j < c; ++j)
          (void)mbar_wait(&sm.full[j % kStagesA], (j / kStagesA) & 1, wait_ns, nullptr);
      }
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  const int rt = warp & 3, kh = warp >> 2;
  const int gid = lane >> 2, t = lane & 3;
  const int r_lo = rt * 16 + gid, r_hi = r_lo + 8;  // rows within the CTA's 64
  const int n_lo = n0 + r_lo, n_hi = n0 + r_hi;
  const bool ok_lo = n_lo < N, ok_hi = n_hi < N;
  const int mt_count = (M + 7) / 8;
  // batch rows of this lane's B fragments (column gid of each m-tile)
  const uint16_t* x0 = gid < M ? a.x + (size_t)gid * K + 16 * t : nullptr;
  const uint16_t* x1 = gid + 8 < M ? a.x + (size_t)(gid + 8) * K + 16 * t : nullptr;
  const uint16_t* s_lo = a.s + (size_t)(ok_lo ? n_lo : 0) * ng;
  const uint16_t* s_hi = a.s + (size_t)(ok_hi ? n_hi : 0) * ng;
  const uint16_t* z_lo = a.z + (size_t)(ok_lo ? n_lo : 0) * ng;
  const uint16_t* z_hi = a.z + (size_t)(ok_hi ? n_hi : 0) * ng;

  float tot[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) tot[i][0] = tot[i][1] = tot[i][2] = tot[i][3] = 0.f;

  bool ok = true;
  for (int c = kh; c < nst; c += 2) {
    const int s = c % kStagesA;
    // this stage's group scales and zero points (issued before the wait)
    const int g0 = c * 4, gn = min(4, ng - g0);
    uint32_t sv[4], zv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int g = min(g0 + j, ng - 1);
      sv[j] = (uint32_t)__ldg(s_lo + g) | ((uint32_t)__ldg(s_hi + g) << 16);
      zv[j] = (uint32_t)__ldg(z_lo + g) | ((uint32_t)__ldg(z_hi + g) << 16);
    }
    if (!warp_wait(&sm.full[s], (c / kStagesA) & 1, wait_ns, err)) {
      ok = false;
      break;
    }
    const uint8_t* st = sm.stage[s];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j < gn) {
        // weights: 8 bytes of rows r_lo and r_hi (group j, k = 16t ..), 128-byte swizzle
        const int u = 2 * j + (t >> 1), hoff = (t & 1) * 8;
        const uint2 wl = *reinterpret_cast<const uint2*>(st + r_lo * 128 + ((u ^ (r_lo & 7)) << 4) + hoff);
        const uint2 wh = *reinterpret_cast<const uint2*>(st + r_hi * 128 + ((u ^ (r_hi & 7)) << 4) + hoff);
        const uint32_t zzl = f32_to_bf16_bits(128.0f + bf16_bits_to_f32(zv[j] & 0xFFFFu)) * 0x10001u;
        const uint32_t zzh = f32_to_bf16_bits(128.0f + bf16_bits_to_f32(zv[j] >> 16)) * 0x10001u;
        uint32_t A[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t wlo = (q < 2) ? wl.x : wl.y;
          const uint32_t whi = (q < 2) ? wh.x : wh.y;
          const int sh0 = (q & 1) * 8;
          A[q][0] = deq_pair(wlo, sh0, zzl);
          A[q][1] = deq_pair(whi, sh0, zzh);
          A[q][2] = deq_pair(wlo, sh0 + 4, zzl);
          A[q][3] = deq_pair(whi, sh0 + 4, zzh);
        }
        const float sc_lo = bf16_bits_to_f32(sv[j] & 0xFFFFu), sc_hi = bf16_bits_to_f32(sv[j] >> 16);
        const int kof = (g0 + j) * 64;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          if (mt < mt_count) {
            const uint16_t* xp = mt ? x1 : x0;
            uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
            if (xp) {
              xa = __ldg(reinterpret_cast<const uint4*>(xp + kof));
              xb = __ldg(reinterpret_cast<const uint4*>(xp + kof + 8));
            }
            // pairs (k, k+4): (0,4) (1,5) | (2,6) (3,7) | (8,12) (9,13) | (10,14) (11,15)
            const uint32_t B[4][2] = {{prmt(xa.x, xa.z, 0x5410u), prmt(xa.x, xa.z, 0x7632u)},
                                      {prmt(xa.y, xa.w, 0x5410u), prmt(xa.y, xa.w, 0x7632u)},
                                      {prmt(xb.x, xb.z, 0x5410u), prmt(xb.x, xb.z, 0x7632u)},
                                      {prmt(xb.y, xb.w, 0x5410u), prmt(xb.y, xb.w, 0x7632u)}};
            float cc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q) mma_16816(cc, A[q], B[q][0], B[q][1]);
            tot[mt][0] = fmaf(sc_lo, cc[0], tot[mt][0]);
            tot[mt][1] = fmaf(sc_lo, cc[1], tot[mt][1]);
            tot[mt][2] = fmaf(sc_hi, cc[2], tot[mt][2]);
            tot[mt][3] = fmaf(sc_hi, cc[3], tot[mt][3]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
  }

  // add the two phases' partial sums (phase 0 + phase 1) and store
  if (!ok && lane == 0) sm.abort_flag = 1;
  if (kh == 1) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) sm.red[rt][mt][lane][i] = tot[mt][i];
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarps * 32) : "memory");
  if (sm.abort_flag || kh == 1) return;
  const float b_lo = (a.bias && ok_lo) ? bf16_bits_to_f32(a.bias[n_lo]) : 0.f;
  const float b_hi = (a.bias && ok_hi) ? bf16_bits_to_f32(a.bias[n_hi]) : 0.f;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    if (mt >= mt_count) continue;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = mt * 8 + 2 * t + i;  // column 2t + i of the MMA tile
      if (m >= M) continue;
      const float v_lo = tot[mt][i] + sm.red[rt][mt][lane][i];
      const float v_hi = tot[mt][2 + i] + sm.red[rt][mt][lane][2 + i];
      if (ok_lo) a.y[(size_t)m * N + n_lo] = (uint16_t)f32_to_bf16_bits(__fadd_rn(v_lo, b_lo));
      if (ok_hi) a.y[(size_t)m * N + n_hi] = (uint16_t)f32_to_bf16_bits(__fadd_rn(v_hi, b_hi));
    }
  }
}

}  // namespace

cudaError_t launch_awq(const AwqArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q, (uint64_t)a.K / 2, (uint64_t)a.N, (uint64_t)a.K / 2,
                    kStageK / 2, kRowsA, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(SmemA) + 1024;
  cudaError_t e = cudaFuncSetAttribute(awq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (a.N + kRowsA - 1) / kRowsA;
  // batch rows are taken 16 at a time; each block of rows re-reads the weights
  for (int m0 = 0; m0 < a.M; m0 += kMaxM) {
    AwqArgs b = a;
    b.M = min(kMaxM, a.M - m0);
    b.x = a.x + (size_t)m0 * a.K;
    b.y = a.y + (size_t)m0 * a.N;
    awq_kernel<<<grid, kThreadsA, smem, s>>>(tm_q, b, err, wait_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace svdq
