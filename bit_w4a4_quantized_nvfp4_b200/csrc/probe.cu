// Diagnostic kernels: the device format conversions used by the quantisers,
// applied element-wise (so they can be compared with the CPU oracle on every
// fp32 bit pattern), and a bounded wait that is made to run out.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

__global__ void probe_convert_kernel(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3,
                                     uint16_t* bf16) {
  const long long base = (blockIdx.x * (long long)blockDim.x + threadIdx.x) * 8;
  for (long long i0 = base; i0 < n; i0 += (long long)gridDim.x * blockDim.x * 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (i0 + j < n) ? in[i0 + j] : 0.f;
    if (e2m1) {
      const uint32_t w = cvt_e2m1x8(v);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (i0 + j < n) e2m1[i0 + j] = (uint8_t)((w >> (4 * j)) & 0xFu);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (i0 + j >= n) break;
      if (e4m3) e4m3[i0 + j] = (uint8_t)cvt_e4m3(v[j]);
      if (bf16) bf16[i0 + j] = (uint16_t)f32_to_bf16_bits(v[j]);
    }
  }
}

__global__ void probe_wait_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up after limit_ns.
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, limit_ns, err);
  __syncthreads();
}

}  // namespace

cudaError_t launch_probe_convert(const float* in, long long n, uint8_t* e2m1, uint8_t* e4m3,
                                 uint16_t* bf16, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n + 8 * 256 - 1) / (8 * 256);
  if (blocks > 148 * 64) blocks = 148 * 64;
  probe_convert_kernel<<<(unsigned)blocks, 256, 0, s>>>(in, n, e2m1, e4m3, bf16);
  return cudaGetLastError();
}

cudaError_t launch_probe_wait(unsigned* err, unsigned long long limit_ns, cudaStream_t s) {
  probe_wait_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace svdq
