// K3 — AWQ W4A16 linear: INT4 weights (asymmetric, bf16 scale/zero per 64
// along K) times bf16 activations, for the memory-bound modulation /
// adaptive-norm projections (blog "Introducing Nunchaku 4-bit inference in
// Diffusers", section "Introducing Nunchaku Lite").
//
// At small M the weight stream is the whole cost, so the kernel is built to
// keep HBM busy: a producer warp streams 64-row x 256-K weight boxes (8 KB,
// 128-byte swizzle) through a 6-stage TMA pipeline, so that every SM has
// ~100 KB of weight reads in flight, and twelve compute warps consume them
// from shared memory (full/empty mbarriers; the three warp groups take every
// third stage and the stage count is a multiple of three, so a stage is only
// refilled for the group that released it).
//
// The CTA's activations (up to 16 rows) and its rows' group scales and zero
// points (one contiguous range each) are copied into shared memory once, at
// the start, by bulk copies; the compute warps then permute the activations in
// place into MMA-fragment order, so that the inner loop reads each B fragment
// with one 16-byte load.
//
// Compute warp (row tile rt of 16 weight rows, stage phase kh of 3): per 64-group
// it unpacks its two rows' nibbles to bf16 with bit operations ((128 + q) has
// an exact bf16 encoding; subtracting 128 + z leaves q - z exactly) and lets
// the tensor cores (mma.sync m16n8k16, fp32 accumulate) form the dot products
// with the activations; each group's partial sums are scaled by the group
// scale in fp32. The three phases' partial sums are added in a fixed order.
//
// K order inside a group: lane t of a row quad owns k = 16t .. 16t+15 (one
// 8-byte shared load per row). Its nibbles are used in pairs (k, k+4), fed to
// the MMA K slots in the order (0,4),(1,5) | (2,6),(3,7) | (8,12),(9,13) |
// (10,14),(11,15) for the four k16 steps; each 16-element block of x is
// stored as the bf16 pairs (0,4) (1,5) (2,6) (3,7) (8,12) (9,13) (10,14)
// (11,15), so the dot product is unchanged.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kRowsA = 64;                          // weight rows (output columns) per CTA
constexpr int kStageK = 256;                        // K per stage: 4 groups, 128 bytes per row
constexpr int kStageBytesA = kRowsA * kStageK / 2;  // 8 KB
constexpr int kPhasesA = 3;                         // warp groups taking every third stage
constexpr int kStagesA = 6;                         // a multiple of kPhasesA: see the header comment
constexpr int kComputeWarps = 4 * kPhasesA;         // 4 row tiles x 3 stage phases
constexpr int kThreadsA = (kComputeWarps + 1) * 32;
constexpr int kMaxM = 16;                           // batch rows per launch (two m-tiles of 8)
constexpr int kAwqSmemLimit = 232448;               // dynamic shared memory per CTA on sm_100
static_assert(kStagesA % kPhasesA == 0, "a stage is reused by one warp group only");

// (no side effects: left non-volatile so independent groups' MMAs can be interleaved)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
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

// Shared-memory plan of one CTA (dynamic size: it depends on M and K).
struct AwqLayout {
  int x_pitch;    // bytes per activation row: 2K + 16 (the pad spreads rows over banks)
  int sz_pitch;   // bytes per weight row of scales / zeros: 2 * (K / 64)
  int off_x, off_s, off_z, off_bar, total;
  __host__ __device__ AwqLayout(int M, int K) {
    const int ng = K / 64;
    x_pitch = 2 * K + 16;
    sz_pitch = 2 * ng;
    off_x = kStagesA * kStageBytesA;
    off_s = off_x + M * x_pitch;
    off_z = ((off_s + kRowsA * sz_pitch + 15) / 16) * 16;
    off_bar = ((off_z + kRowsA * sz_pitch + 15) / 16) * 16;
    total = off_bar + 2 * kStagesA * 8 + 16 + 16 + (kPhasesA - 1) * 4 * 2 * 32 * 4 * 4;
  }
};

__global__ void __launch_bounds__(kThreadsA, 2)
awq_kernel(const __grid_constant__ CUtensorMap tm_q, AwqArgs a, unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_align<1024>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = a.K, N = a.N, M = a.M;
  const int ng = K / 64;
  const int nst = (K + kStageK - 1) / kStageK;
  const int n0 = blockIdx.x * kRowsA;
  const AwqLayout L(M, K);
  uint8_t* xs = base + L.off_x;
  const uint8_t* ss = base + L.off_s;
  const uint8_t* zs = base + L.off_z;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.off_bar);
  uint64_t* empty = full + kStagesA;
  uint64_t* xbar = empty + kStagesA;
  int* abort_flag = reinterpret_cast<int*>(xbar + 2);
  float* red = reinterpret_cast<float*>(abort_flag + 4);  // phases 1.. partial sums [kh-1][rt][mt][lane][4]

  // the next kernel in the stream may be scheduled as SMs free up; it waits
  // for this one before it reads anything this one writes
  if (threadIdx.x == 0) launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kComputeWarps && lane == 0) {
    // Before the previous kernel in the stream has finished, only hints: the
    // tensor map and the first weight tiles are pulled towards L2. Any input
    // (weights, scales, zero points, x, bias) may have been written by that
    // kernel, so nothing is read into shared memory or registers until
    // griddepcontrol.wait below has returned.
    tma_prefetch_desc(&tm_q);
    for (int c = 0; c < nst && c < kStagesA; ++c) tma_prefetch_l2_2d(&tm_q, c * (kStageK / 2), n0);
  }
  __syncthreads();
  grid_dependency_wait();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    int c = 0;
    bool ok = true;
    auto issue_stage = [&](int cc) {
      const int s = cc % kStagesA;
      mbar_expect_tx(&full[s], kStageBytesA);
      tma_load_2d(base + s * kStageBytesA, &tm_q, &full[s], cc * (kStageK / 2), n0);
    };
    if (lane == 0) {
      // this CTA's rows of scales and zero points (contiguous: rows n0 ..
      // n0 + rows - 1, 16-byte aligned), the activations (one bulk copy per
      // row) and the first weight stages, which need no release
      const uint32_t sz_bytes = (uint32_t)(min(kRowsA, N - n0) * L.sz_pitch);
      mbar_expect_tx(xbar, (uint32_t)(M * 2 * K) + 2 * sz_bytes);
      bulk_load(base + L.off_s, a.s + (size_t)n0 * ng, sz_bytes, xbar);
      bulk_load(base + L.off_z, a.z + (size_t)n0 * ng, sz_bytes, xbar);
      for (; c < nst && c < kStagesA; ++c) issue_stage(c);
      for (int m = 0; m < M; ++m) bulk_load(xs + m * L.x_pitch, a.x + (size_t)m * K, (uint32_t)(2 * K), xbar);
      for (; c < nst; ++c) {
        const int s = c % kStagesA;
        if (!mbar_wait(&empty[s], ((c / kStagesA) - 1) & 1, wait_ns, err)) {
          ok = false;
          break;
        }
        issue_stage(c);
      }
      // let the copies already issued land before the CTA can exit (bounded)
      (void)mbar_wait(xbar, 0, wait_ns, ok ? err : nullptr);
      if (!ok)
        for (int j = max(0, c - kStagesA); j < c; ++j)
          (void)mbar_wait(&full[j % kStagesA], (j / kStagesA) & 1, wait_ns, nullptr);
    }
    return;
  }

  // ---------------------------------------------------------------- compute
  bool ok = __all_sync(0xffffffffu, mbar_wait(xbar, 0, wait_ns, err));
  // permute every 16-element block of x in place into fragment-pair order
  if (ok) {
    const int blocks = M * (K / 16);
    for (int b = threadIdx.x; b < blocks; b += kComputeWarps * 32) {
      const int m = b / (K / 16), kb = b % (K / 16);
      uint4* pp = reinterpret_cast<uint4*>(xs + m * L.x_pitch + kb * 32);
      const uint4 u = pp[0], v = pp[1];
      pp[0] = make_uint4(prmt(u.x, u.z, 0x5410u), prmt(u.x, u.z, 0x7632u), prmt(u.y, u.w, 0x5410u),
                         prmt(u.y, u.w, 0x7632u));
      pp[1] = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                         prmt(v.y, v.w, 0x7632u));
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarps * 32) : "memory");

  const int rt = warp & 3, kh = warp >> 2;  // row tile, stage phase
  const int gid = lane >> 2, t = lane & 3;
  const int r_lo = rt * 16 + gid, r_hi = r_lo + 8;  // rows within the CTA's 64
  const int n_lo = n0 + r_lo, n_hi = n0 + r_hi;
  const bool ok_lo = n_lo < N, ok_hi = n_hi < N;
  const int mt_count = (M + 7) / 8;
  // this lane's B-fragment rows (column gid of each m-tile), 16t into each group
  const uint8_t* x0 = gid < M ? xs + gid * L.x_pitch + 32 * t : nullptr;
  const uint8_t* x1 = gid + 8 < M ? xs + (gid + 8) * L.x_pitch + 32 * t : nullptr;

  float tot[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) tot[i][0] = tot[i][1] = tot[i][2] = tot[i][3] = 0.f;

  const bool vec_sz = (ng & 3) == 0;  // 4 groups of a row are one aligned 8-byte word
  for (int c = kh; c < nst && ok; c += kPhasesA) {
    const int s = c % kStagesA;
    const int g0 = c * 4, gn = min(4, ng - g0);
    if (!warp_wait(&full[s], (c / kStagesA) & 1, wait_ns, err)) {
      ok = false;
      break;
    }
    const uint8_t* st = base + s * kStageBytesA;
    // this stage's scales and zero points of rows r_lo / r_hi: 4 groups each
    uint32_t sv[2][2], zv[2][2];  // [row lo/hi][groups 0-1 / 2-3], bf16 pairs
    if (vec_sz) {
      const uint2 a0 = *reinterpret_cast<const uint2*>(ss + r_lo * L.sz_pitch + 8 * c);
      const uint2 a1 = *reinterpret_cast<const uint2*>(ss + r_hi * L.sz_pitch + 8 * c);
      const uint2 b0 = *reinterpret_cast<const uint2*>(zs + r_lo * L.sz_pitch + 8 * c);
      const uint2 b1 = *reinterpret_cast<const uint2*>(zs + r_hi * L.sz_pitch + 8 * c);
      sv[0][0] = a0.x; sv[0][1] = a0.y; sv[1][0] = a1.x; sv[1][1] = a1.y;
      zv[0][0] = b0.x; zv[0][1] = b0.y; zv[1][0] = b1.x; zv[1][1] = b1.y;
    } else {
      const uint16_t* sl = reinterpret_cast<const uint16_t*>(ss + r_lo * L.sz_pitch);
      const uint16_t* sh = reinterpret_cast<const uint16_t*>(ss + r_hi * L.sz_pitch);
      const uint16_t* zl = reinterpret_cast<const uint16_t*>(zs + r_lo * L.sz_pitch);
      const uint16_t* zh = reinterpret_cast<const uint16_t*>(zs + r_hi * L.sz_pitch);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int ga = min(g0 + 2 * h2, ng - 1), gb = min(g0 + 2 * h2 + 1, ng - 1);
        sv[0][h2] = sl[ga] | ((uint32_t)sl[gb] << 16);
        sv[1][h2] = sh[ga] | ((uint32_t)sh[gb] << 16);
        zv[0][h2] = zl[ga] | ((uint32_t)zl[gb] << 16);
        zv[1][h2] = zh[ga] | ((uint32_t)zh[gb] << 16);
      }
    }
    // one 64-group: dequantise rows r_lo / r_hi and accumulate into tot
    auto group = [&](int j) {
      const int g = g0 + j;
      // weights: 8 bytes of rows r_lo and r_hi (group j, k = 16t ..), 128-byte swizzle
      const int u = 2 * j + (t >> 1), hoff = (t & 1) * 8;
      const uint2 wl = *reinterpret_cast<const uint2*>(st + r_lo * 128 + ((u ^ (r_lo & 7)) << 4) + hoff);
      const uint2 wh = *reinterpret_cast<const uint2*>(st + r_hi * 128 + ((u ^ (r_hi & 7)) << 4) + hoff);
      // (row lo, row hi) of this group: scales to fp32, 128 + z as bf16 pairs
      const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
      const uint32_t z2 = prmt(zv[0][j >> 1], zv[1][j >> 1], sel);
      const uint32_t s2 = prmt(sv[0][j >> 1], sv[1][j >> 1], sel);
      uint32_t z128;
      asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(z128) : "r"(z2), "r"(0x43004300u));
      const uint32_t zzl = prmt(z128, z128, 0x1010u), zzh = prmt(z128, z128, 0x3232u);
      const float sc_lo = __uint_as_float(s2 << 16), sc_hi = __uint_as_float(s2 & 0xFFFF0000u);
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
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        if (mt < mt_count) {
          const uint8_t* xp = mt ? x1 : x0;
          uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
          if (xp) {
            xa = *reinterpret_cast<const uint4*>(xp + 128 * g);
            xb = *reinterpret_cast<const uint4*>(xp + 128 * g + 16);
          }
          // two independent partial chains, added once
          float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
          mma_16816(c0, A[0], xa.x, xa.y);
          mma_16816(c1, A[1], xa.z, xa.w);
          mma_16816(c0, A[2], xb.x, xb.y);
          mma_16816(c1, A[3], xb.z, xb.w);
          tot[mt][0] = fmaf(sc_lo, c0[0] + c1[0], tot[mt][0]);
          tot[mt][1] = fmaf(sc_lo, c0[1] + c1[1], tot[mt][1]);
          tot[mt][2] = fmaf(sc_hi, c0[2] + c1[2], tot[mt][2]);
          tot[mt][3] = fmaf(sc_hi, c0[3] + c1[3], tot[mt][3]);
        }
      }
    };
    if (gn == 4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) group(j);
    } else {
      for (int j = 0; j < gn; ++j) group(j);
    }
    // release the stage only once its weights have gone through the MMAs
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) consumed(tot[mt][i]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // add the phases' partial sums (phase 0 + phase 1 + phase 2) and store
  if (!ok && lane == 0) *abort_flag = 1;
  if (kh > 0) {
    float* rb = red + ((size_t)(kh - 1) * 4 + rt) * 2 * 32 * 4;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) rb[(mt * 32 + lane) * 4 + i] = tot[mt][i];
  }
  asm volatile("bar.sync 1, %0;" ::"r"(kComputeWarps * 32) : "memory");
  if (*abort_flag || kh > 0) return;
#pragma unroll
  for (int ph = 1; ph < kPhasesA; ++ph) {
    const float* rb = red + ((size_t)(ph - 1) * 4 + rt) * 2 * 32 * 4;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) tot[mt][i] += rb[(mt * 32 + lane) * 4 + i];
  }
  const float b_lo = (a.bias && ok_lo) ? bf16_bits_to_f32(a.bias[n_lo]) : 0.f;
  const float b_hi = (a.bias && ok_hi) ? bf16_bits_to_f32(a.bias[n_hi]) : 0.f;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    if (mt >= mt_count) continue;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int m = mt * 8 + 2 * t + i;  // column 2t + i of the MMA tile
      if (m >= M) continue;
      const float v_lo = tot[mt][i];
      const float v_hi = tot[mt][2 + i];
      if (ok_lo) a.y[(size_t)m * N + n_lo] = (uint16_t)f32_to_bf16_bits(__fadd_rn(v_lo, b_lo));
      if (ok_hi) a.y[(size_t)m * N + n_hi] = (uint16_t)f32_to_bf16_bits(__fadd_rn(v_hi, b_hi));
    }
  }
}

}  // namespace

int awq_rows_per_launch(int K) {
  // as many batch rows (up to 16) as leave the CTA's shared memory within bounds
  int mb = kMaxM;
  while (mb > 0 && AwqLayout(mb, K).total + 1024 > kAwqSmemLimit) --mb;
  return mb;
}

cudaError_t launch_awq(const AwqArgs& a, unsigned* err, unsigned long long wait_ns, cudaStream_t s) {
  // up to four rows: the GEMV kernel, whose MMA columns hold groups as well as
  // batch rows (when its shared memory plan fits the row length)
  if (awq_gemv_fits(a.M, a.K)) return launch_awq_gemv(a, err, wait_ns, s);
  CUtensorMap tm_q;
  if (!make_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.q, (uint64_t)a.K / 2, (uint64_t)a.N, (uint64_t)a.K / 2,
                    kStageK / 2, kRowsA, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int mb = awq_rows_per_launch(a.K);
  if (mb < 1) return cudaErrorInvalidValue;
  const int grid = (a.N + kRowsA - 1) / kRowsA;
  // batch rows are taken mb at a time; each block of rows re-reads the weights
  for (int m0 = 0; m0 < a.M; m0 += mb) {
    AwqArgs b = a;
    b.M = min(mb, a.M - m0);
    b.x = a.x + (size_t)m0 * a.K;
    b.y = a.y + (size_t)m0 * a.N;
    const size_t smem = (size_t)AwqLayout(b.M, a.K).total + 1024;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(awq_kernel), (int)smem);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: this grid may start while the previous
    // kernel in the stream finishes (see the kernel's wait before x)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreadsA);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, awq_kernel, tm_q, b, err, wait_ns);
    if (e != cudaSuccess) return e;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace svdq
