// Tensor-core rate probe: how fast this device runs the block-scaled NVFP4
// MMA that the GEMM issues (tcgen05.mma.cta_group::2.kind::mxf4nvf4
// .block_scale.block16, 256 x 256 x 64 per CTA pair), with nothing else
// running. Every CTA pair keeps one GEMM stage of operands (A and B codes,
// 128-byte swizzled, and their UE4M3 scale atoms) in shared memory for the
// whole launch: no TMA loads, no epilogue, so the measured time is the MMA
// issue and execution rate alone. It is the measured denominator of the
// GEMM's roofline.
//
// mode 0: per 256-wide K stage, 4 MMAs of N = 256 (the GEMM's main loop
//         without its operand stream);
// mode 1: as 0, plus 12 tcgen05.cp scale copies per stage (shows what the
//         scale copies cost the tensor pipe);
// mode 2: the same work as 8 MMAs of N = 128 per stage (two N halves);
// mode 3: the same work as 16 MMAs of N = 64 per stage;
// mode 4: as mode 2, but the 4 MMAs of each N half issued back to back into
//         the same accumulator (instead of alternating the halves).
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int kPA = 16384, kPB = 16384, kPSfa = 2048, kPSfb = 4096;
constexpr int kPStage = kPA + kPB + kPSfa + kPSfb;
constexpr uint32_t kPSfaCol = 448, kPSfbCol = 464;
// M = 256 (the pair), N = 256, E2M1 x E2M1 with UE4M3 scales per 16 (the GEMM's descriptor)
constexpr uint32_t kPIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t kPIdesc128 = (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t kPIdesc64 = (1u << 7) | (1u << 10) | ((uint32_t)(64 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
probe_mma_kernel(int iters, int mode, unsigned* err, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* st = smem_align<1024>(smem_raw);
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5;
  const bool leader = cluster_rank() == 0;

  // operands: a fixed nonzero pattern (finite E2M1 codes; every scale 1.0)
  uint32_t* w = reinterpret_cast<uint32_t*>(st);
  for (int i = threadIdx.x; i < (kPA + kPB) / 4; i += blockDim.x) w[i] = 0x2A7135B9u ^ (uint32_t)(i * 0x9E3779B1u);
  for (int i = (kPA + kPB) / 4 + threadIdx.x; i < kPStage / 4; i += blockDim.x) w[i] = 0x38383838u;
  fence_proxy_async_smem();  // generic-proxy writes before the tensor core reads them
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(&tmem_base, 512);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (leader && warp == 1) {
    const uint32_t s0 = smem_u32(st);
    const uint32_t sfa = s0 + kPA + kPB, sfb = sfa + kPSfa;
    uint64_t dcp[12], da[4], db[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      dcp[3 * j] = make_sdesc(sfa + 512 * j, 512, 128, kLayoutNone);
      dcp[3 * j + 1] = make_sdesc(sfb + 512 * j, 512, 128, kLayoutNone);
      dcp[3 * j + 2] = make_sdesc(sfb + 2048 + 512 * j, 512, 128, kLayoutNone);
      da[j] = make_sdesc(s0 + 32 * j, 16, 1024, kLayoutSw128);
      db[j] = make_sdesc(s0 + kPA + 32 * j, 16, 1024, kLayoutSw128);
    }
    if (elect_one()) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tc_cp_32x128b_warpx4_pair(tmem + kPSfaCol + 4 * j, dcp[3 * j]);
        tc_cp_32x128b_warpx4_pair(tmem + kPSfbCol + 8 * j, dcp[3 * j + 1]);
        tc_cp_32x128b_warpx4_pair(tmem + kPSfbCol + 8 * j + 4, dcp[3 * j + 2]);
      }
      for (int it = 0; it < iters; ++it) {
        if (mode == 1) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_cp_32x128b_warpx4_pair(tmem + kPSfaCol + 4 * j, dcp[3 * j]);
            tc_cp_32x128b_warpx4_pair(tmem + kPSfbCol + 8 * j, dcp[3 * j + 1]);
            tc_cp_32x128b_warpx4_pair(tmem + kPSfbCol + 8 * j + 4, dcp[3 * j + 2]);
          }
        }
        if (mode <= 1) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvfp4_pair(tmem, da[j], db[j], kPIdesc, tmem + kPSfaCol + 4 * j, tmem + kPSfbCol + 8 * j,
                           (it > 0 || j > 0) ? 1u : 0u);
        } else if (mode == 2) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
              mma_nvfp4_pair(tmem + 128 * hh, da[j], db[j] + (uint64_t)((64 * 128) >> 4) * hh, kPIdesc128,
                             tmem + kPSfaCol + 4 * j, tmem + kPSfbCol + 8 * j, (it > 0 || j > 0) ? 1u : 0u);
        } else if (mode == 4) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_nvfp4_pair(tmem + 128 * hh, da[j], db[j] + (uint64_t)((64 * 128) >> 4) * hh, kPIdesc128,
                             tmem + kPSfaCol + 4 * j, tmem + kPSfbCol + 8 * j, (it > 0 || j > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hh = 0; hh < 4; ++hh)
              mma_nvfp4_pair(tmem + 64 * hh, da[j], db[j] + (uint64_t)((32 * 128) >> 4) * hh, kPIdesc64,
                             tmem + kPSfaCol + 4 * j, tmem + kPSfbCol + 8 * j, (it > 0 || j > 0) ? 1u : 0u);
        }
      }
      // both CTAs learn when every MMA has completed
      tc_commit_pair(&done, 0x3);
    }
    __syncwarp();
  }
  if (threadIdx.x == 0) (void)mbar_wait(&done, 0, wait_ns, err);
  __syncthreads();
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
  __syncwarp();
  cluster_sync();
}

}  // namespace

cudaError_t launch_probe_mma(int iters, int mode, int num_sms, unsigned* err, unsigned long long wait_ns,
                             cudaStream_t s) {
  // More than half of an SM's shared memory, so that no two CTAs share an SM:
  // every pair takes all 512 tensor-memory columns, and two pairs whose CTAs
  // crossed over two SMs would each wait for the other's columns.
  const size_t smem = 120 * 1024;
  static_assert(kPStage + 1024 <= 120 * 1024, "one stage fits");
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(probe_mma_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  probe_mma_kernel<<<2 * (num_sms / 2), 128, smem, s>>>(iters, mode, err, wait_ns);
  return cudaGetLastError();
}

}  // namespace svdq
