// K2 — NVFP4 W4A4 GEMM with the low-rank up-projection and bias fused
// (blog "Introducing Nunchaku 4-bit inference in Diffusers", section
// "Background: SVDQuant and Nunchaku", figure caption: the up-projection is
// fused into the 4-bit compute kernel).
//
//   y[m,n] = alpha * ( sum_b sx[m,b] sw[n,b] sum_{k in b} qx[m,k] qw[n,k]
//                      + sum_j P[m,j] (hi[n,j] + lo[n,j]) ) + bias[n]
// with alpha = s_tx * s_tw and hi + lo = bf16 split of L2 / alpha (prepared by
// svdq_pack_weight), so that alpha * (P (hi + lo)) = P L2 to ~2^-16 relative.
//
// sm_100a design (persistent, warp-specialised, one CTA per SM):
//   warp 0      TMA producer: A/B code tiles (128B-swizzled, K-major), the
//               matching UE4M3 scale atoms (bulk copies), and per tile one
//               extra stage holding the P tile and the prepared L2 tile.
//   warp 1      TMEM allocator and single-thread MMA issuer: per K stage,
//               tcgen05.cp moves the scale atoms shared -> tensor memory, then
//               4 x tcgen05.mma kind::mxf4nvf4 (K = 64 each) accumulate into a
//               128 x 256 fp32 accumulator in TMEM; after the K loop,
//               tcgen05.mma kind::f16 adds P (hi + lo) into the same accumulator.
//   warps 2..5  epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31), y = alpha*acc + bias, convert, stage through
//               128B-swizzled shared memory, TMA store.
// Tile 128 (M) x 256 (N), K stage 256 (128 bytes of packed E2M1 per row),
// 3-stage smem ring. Every mbarrier wait is bounded in wall time.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256, BK = 256;        // BK in FP4 elements
constexpr int kStages = 3;
constexpr int kABytes = BM * BK / 2;               // 16 KB
constexpr int kBBytes = BN * BK / 2;               // 32 KB
constexpr int kSfaBytes = 4 * 512;                 // 4 K-atoms x 128 rows
constexpr int kSfbBytes = 2 * 4 * 512;             // 2 row blocks x 4 K-atoms
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr int kEpiWarps = 4;
constexpr int kStageOutBytes = 32 * 128;           // 32 rows x 128 bytes
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;                    // 256 fp32 columns
constexpr uint32_t kSfCol = 256;                   // 2 buffers x (16 SFA + 32 SFB) columns

constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(BM >> 4) << 24);

struct Smem {
  uint8_t stage[kStages][kStageBytes];               // each 1024-aligned (kStageBytes % 1024 == 0)
  uint8_t out[kEpiWarps][2][kStageOutBytes];
  float bias[kEpiWarps][BN];                         // per warp: no cross-warp barrier needed
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full, acc_empty, mma_done;
  uint32_t tmem_base;
};
static_assert(kStageBytes % 1024 == 0, "stage alignment");

struct Params {
  const uint8_t* x_scales;
  const uint8_t* w_scales;
  const float* tensor_scale;
  const uint16_t* bias;
  int M, N, K, r;
  int tiles_m, tiles_n;
  int out_f32;
  unsigned* err;
  unsigned long long wait_ns;
};

__global__ void __launch_bounds__(kThreads, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_l,
                  const __grid_constant__ CUtensorMap tm_y, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int nk = (p.K + BK - 1) / BK;
  const int katoms = p.K / 64;
  const bool has_lr = p.r > 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, kEpiWarps);
    mbar_init(&sm.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_y);
    if (has_lr) {
      tma_prefetch_desc(&tm_p);
      tma_prefetch_desc(&tm_l);
    }
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int tm = tile / p.tiles_n, tn = tile % p.tiles_n;
        const int m0 = tm * BM, n0 = tn * BN;
        const int rb0 = 2 * tn, rb1 = 2 * tn + 1;
        const bool has_rb1 = rb1 * 128 < p.N;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          const int kat = min(4, katoms - 4 * kb);
          const uint32_t sf_bytes = (uint32_t)kat * 512;
          uint8_t* st = sm.stage[s];
          mbar_expect_tx(&sm.full[s], kABytes + kBBytes + sf_bytes * (has_rb1 ? 3 : 2));
          tma_load_2d(st, &tm_a, &sm.full[s], kb * (BK / 2), m0);
          tma_load_2d(st + kABytes, &tm_b, &sm.full[s], kb * (BK / 2), n0);
          uint8_t* sfa = st + kABytes + kBBytes;
          uint8_t* sfb = sfa + kSfaBytes;
          bulk_load(sfa, p.x_scales + ((size_t)tm * katoms + 4 * kb) * 512, sf_bytes, &sm.full[s]);
          bulk_load(sfb, p.w_scales + ((size_t)rb0 * katoms + 4 * kb) * 512, sf_bytes, &sm.full[s]);
          if (has_rb1)
            bulk_load(sfb + 4 * 512, p.w_scales + ((size_t)rb1 * katoms + 4 * kb) * 512, sf_bytes, &sm.full[s]);
        }
        if (!ok) break;
        if (has_lr) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          uint8_t* st = sm.stage[s];
          const int pc = p.r / 8, lc = 2 * p.r / 8;  // 8-column boxes
          mbar_expect_tx(&sm.full[s], (uint32_t)(pc * BM * 16 + lc * BN * 16));
          for (int c = 0; c < pc; ++c) tma_load_2d(st + c * BM * 16, &tm_p, &sm.full[s], 8 * c, m0);
          for (int c = 0; c < lc; ++c) tma_load_2d(st + kABytes + c * BN * 16, &tm_l, &sm.full[s], 8 * c, n0);
          ++it;
        }
      }
      if (!ok) {
        // let the copies already issued (stages it-1 .. it-kStages) land
        // before the CTA exits
        for (uint32_t d = 1; d <= (uint32_t)kStages && d <= it; ++d) {
          const uint32_t j = it - d;
          (void)mbar_wait(&sm.full[j % kStages], (j / kStages) & 1, p.wait_ns, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        if (!mbar_wait(&sm.acc_empty, (local & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.full[s], (it / kStages) & 1, p.wait_ns, p.err)) { ok = false; break; }
          tc_fence_after();
          const int kat = min(4, katoms - 4 * kb);
          const uint32_t st = smem_u32(sm.stage[s]);
          const uint32_t sfa = st + kABytes + kBBytes, sfb = sfa + kSfaBytes;
          const uint32_t sf_col = kSfCol + (uint32_t)(it & 1) * 48;
          for (int j = 0; j < kat; ++j) {
            tc_cp_32x128b_warpx4(tmem + sf_col + 4 * j, make_sdesc(sfa + 512 * j, 512, 128, kLayoutNone));
            tc_cp_32x128b_warpx4(tmem + sf_col + 16 + 8 * j, make_sdesc(sfb + 512 * j, 512, 128, kLayoutNone));
            tc_cp_32x128b_warpx4(tmem + sf_col + 16 + 8 * j + 4,
                                 make_sdesc(sfb + 2048 + 512 * j, 512, 128, kLayoutNone));
          }
          for (int j = 0; j < kat; ++j) {
            const uint64_t ad = make_sdesc(st + 32 * j, 16, 1024, kLayoutSw128);
            const uint64_t bd = make_sdesc(st + kABytes + 32 * j, 16, 1024, kLayoutSw128);
            mma_nvfp4(tmem + kAccCol, ad, bd, kIdescNvfp4, tmem + sf_col + 4 * j, tmem + sf_col + 16 + 8 * j,
                      (kb > 0 || j > 0) ? 1u : 0u);
          }
          tc_commit(&sm.empty[s]);
        }
        if (!ok) break;
        if (has_lr) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.full[s], (it / kStages) & 1, p.wait_ns, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = smem_u32(sm.stage[s]);
          const int half = p.r / 16;  // k16 steps per copy of P
          for (int i = 0; i < 2 * half; ++i) {
            const int ip = i % half;
            const uint64_t ad = make_sdesc(st + 2 * ip * BM * 16, BM * 16, 128, kLayoutNone);
            const uint64_t bd = make_sdesc(st + kABytes + 2 * i * BN * 16, BN * 16, 128, kLayoutNone);
            mma_bf16(tmem + kAccCol, ad, bd, kIdescBf16, 1u);
          }
          tc_commit(&sm.empty[s]);
          ++it;
        }
        tc_commit(&sm.acc_full);
      }
      // every MMA this thread issued has completed before tensor memory is freed
      tc_commit(&sm.mma_done);
      (void)mbar_wait(&sm.mma_done, 0, p.wait_ns, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int e = warp - 2;              // epilogue warp index (staging buffers)
    const float alpha = __fmul_rn(p.tensor_scale[0], p.tensor_scale[1]);
    int local = 0;
    uint32_t chunk_ctr = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int tm = tile / p.tiles_n, tn = tile % p.tiles_n;
      const int m0 = tm * BM, n0 = tn * BN;
      float* bias = sm.bias[e];
      __syncwarp();
      for (int c = lane; c < BN; c += 32) {
        const int n = n0 + c;
        bias[c] = (p.bias && n < p.N) ? bf16_bits_to_f32(p.bias[n]) : 0.f;
      }
      __syncwarp();
      if (!mbar_wait(&sm.acc_full, local & 1, p.wait_ns, p.err)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + kAccCol + ((uint32_t)(32 * q) << 16);
      const int nchunks = p.out_f32 ? BN / 32 : BN / 64;
      for (int c = 0; c < nchunks; ++c, ++chunk_ctr) {
        const int b = chunk_ctr & 1;
        uint8_t* buf = sm.out[e][b];
        uint32_t v[32], v2[32];
        if (p.out_f32) {
          tmem_ld32(tbase + 32 * c, v);
          tmem_ld_wait();
        } else {
          tmem_ld32(tbase + 64 * c, v);
          tmem_ld32(tbase + 64 * c + 32, v2);
          tmem_ld_wait();
        }
        if (c == nchunks - 1) {
          // accumulator fully read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.acc_empty);
        }
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        if (p.out_f32) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) o[i] = fmaf(alpha, __uint_as_float(v[4 * u + i]), bias[32 * c + 4 * u + i]);
            *reinterpret_cast<float4*>(buf + lane * 128 + ((u ^ (lane & 7)) * 16)) = make_float4(o[0], o[1], o[2], o[3]);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int col = 8 * u + 2 * i;
              const uint32_t a0 = col < 32 ? v[col] : v2[col - 32];
              const uint32_t a1 = col + 1 < 32 ? v[col + 1] : v2[col + 1 - 32];
              const float y0 = fmaf(alpha, __uint_as_float(a0), bias[64 * c + col]);
              const float y1 = fmaf(alpha, __uint_as_float(a1), bias[64 * c + col + 1]);
              w4[i] = f32_to_bf16_bits(y0) | (f32_to_bf16_bits(y1) << 16);
            }
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((u ^ (lane & 7)) * 16)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int col0 = p.out_f32 ? n0 + 32 * c : n0 + 64 * c;
          if (m0 + 32 * q < p.M && col0 < p.N) tma_store_2d(&tm_y, buf, col0, m0 + 32 * q);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const GemmArgs& a, cudaStream_t s) {
  CUtensorMap tm_a, tm_b, tm_p, tm_l, tm_y;
  const uint64_t kb = (uint64_t)a.K / 2;
  bool ok = make_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.x_codes, kb, a.M, kb, 128, BM,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_tmap_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, kb, a.N, kb, 128, BN,
                          CU_TENSOR_MAP_SWIZZLE_128B);
  if (a.r > 0) {
    ok = ok && make_tmap_2d(&tm_p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.P, a.r, a.M, (uint64_t)a.r * 2, 8, BM,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && make_tmap_2d(&tm_l, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lr_up, 2 * a.r, a.N, (uint64_t)a.r * 4, 8,
                            BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    tm_p = tm_a;
    tm_l = tm_a;
  }
  if (a.out == 1)
    ok = ok && make_tmap_2d(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.y, a.N, a.M, (uint64_t)a.N * 4, 32, 32,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_tmap_2d(&tm_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, a.N, a.M, (uint64_t)a.N * 2, 64, 32,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;

  Params p;
  p.x_scales = static_cast<const uint8_t*>(a.x_scales);
  p.w_scales = static_cast<const uint8_t*>(a.w_scales);
  p.tensor_scale = a.tensor_scale;
  p.bias = a.bias;
  p.M = a.M; p.N = a.N; p.K = a.K; p.r = a.r;
  p.tiles_m = (a.M + BM - 1) / BM;
  p.tiles_n = (a.N + BN - 1) / BN;
  p.out_f32 = a.out == 1;
  p.err = a.err;
  p.wait_ns = a.wait_ns;

  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < a.num_sms ? tiles : a.num_sms;
  gemm_nvfp4_kernel<<<grid, kThreads, smem, s>>>(tm_a, tm_b, tm_p, tm_l, tm_y, p);
  return cudaGetLastError();
}

}  // namespace svdq
