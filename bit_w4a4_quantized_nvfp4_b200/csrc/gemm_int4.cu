// K2 (INT4 variant) — symmetric INT4 W4A4 GEMM with per-64 group scales, the
// low-rank up-projection and bias fused (svdq_w4a4 / int4 / group 64:
// Diffusers "Nunchaku Lite" page, table "Supported quantization types").
//
//   y[m,n] = sum_g sx[m,g] sw[g,n] * (sum_{k in g} qx[m,k] qw[n,k]) + sum_j P[m,j] L2[j,n] + bias[n]
//
// B200 has no 4-bit integer MMA, so the packed codes are widened to int8 in
// shared memory and multiplied with tcgen05.mma kind::i8. Each 64-wide group
// needs its own scale, so every group gets its own int32 accumulator in
// tensor memory (three buffers in rotation, so the MMAs run up to two groups
// ahead of the drain) that the epilogue warps drain into an fp32 running sum
// held in registers; the int32 group sums are exact. The low-rank term P L2
// is one tcgen05.mma kind::f16 per tile into a fourth TMEM region.
//
// Roles (416 threads): warps 0-3 producers (load packed codes one group ahead,
// sign-extend to int8, write the K-major core-matrix layout, arrive on the
// stage barrier), warp 4 TMEM allocator + MMA issuer, warps 5-12 epilogue, two
// per TMEM lane quadrant, each holding the running sums of 64 columns.
// The epilogue turns each exact int32 group sum s (|s| <= 64 * 64) into fp32
// without the conversion unit: the bits of s + 0x4B400000 are the float
// 2^23 + 2^22 + s, so one integer add and one float subtraction give s
// exactly; the scaling then runs as packed f32x2 multiplies and FMAs.
// Tile 128 x 128, one 64-wide group per pipeline stage, 4 stages.
// INT4 weight scales are stored group-major [K/64, N] so one group's 128
// column scales are contiguous.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 128, BKG = 64;     // one group per stage
constexpr int kStages = 4;
constexpr int kOpBytes = 128 * BKG;             // int8 tile, 8 KB
constexpr int kChunkStride = 128 * 16;          // bytes between 16-byte K chunks
constexpr int kMaxR = 64;
constexpr int kLrBytes = 128 * kMaxR * 2;       // 16 KB
constexpr int kProdWarps = 4, kEpiWarps = 8;
constexpr int kThreads = 32 * (kProdWarps + 1 + kEpiWarps);
constexpr uint32_t kTmemCols = 512;
constexpr int kAccBufs = 3;                     // int32 group accumulators, 128 columns each
constexpr uint32_t kLrCol = 128 * kAccBufs;     // 384: the low-rank fp32 accumulator

// kind::i8: D s32, A/B signed int8, K-major, M = 128, N = 128
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);
// kind::f16: D f32, A/B bf16
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(BM >> 4) << 24);

struct Smem {
  uint8_t a[kStages][kOpBytes];
  uint8_t b[kStages][kOpBytes];
  uint8_t p[kLrBytes];
  uint8_t l[kLrBytes];
  float sw[kEpiWarps][BN / 2];
  uint64_t full[kStages], empty[kStages];
  uint64_t accf[kAccBufs], acce[kAccBufs];
  uint64_t lr_full, lr_empty, lr_accf, lr_acce, mma_done;
  uint32_t tmem_base;
};

struct Params {
  const uint8_t* xc;
  const uint16_t* xs;   // [M, NG]
  const uint8_t* wc;
  const uint16_t* ws;   // [NG, N]
  const uint16_t* P;    // [M, r]
  const uint16_t* lr;   // [N, r]
  const uint16_t* bias;
  void* y;
  int M, N, K, r, NG;
  int tiles_m, tiles_n;
  int out;              // 0 bf16, 1 f32, 2 int32 group sums
  unsigned* err;
  unsigned long long wait_ns;
};

// 8 packed int4 (two's complement, element 2j in the low nibble) -> 8 int8
__device__ __forceinline__ uint2 widen8(uint32_t w) {
  const uint32_t lo = __vsub4((w & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
  const uint32_t hi = __vsub4(((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_int4_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const bool has_lr = p.r > 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 32 * kProdWarps);
      mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&sm.accf[i], 1);
      mbar_init(&sm.acce[i], kEpiWarps);
    }
    mbar_init(&sm.lr_full, 32 * kProdWarps);
    mbar_init(&sm.lr_empty, 1);
    mbar_init(&sm.lr_accf, 1);
    mbar_init(&sm.lr_acce, kEpiWarps);
    mbar_init(&sm.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kProdWarps) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < kProdWarps) {
    // ------------------------------------------------------------ producers
    const int t = threadIdx.x;  // row within the tile
    uint32_t it = 0, tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tl) {
      const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN;
      const int m = m0 + t, n = n0 + t;
      if (has_lr) {
        if (!mbar_wait(&sm.lr_empty, (tl & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
        for (int c = 0; c < p.r / 8; ++c) {
          uint4 vp = make_uint4(0, 0, 0, 0), vl = make_uint4(0, 0, 0, 0);
          if (m < p.M) vp = *reinterpret_cast<const uint4*>(p.P + (size_t)m * p.r + 8 * c);
          if (n < p.N) vl = *reinterpret_cast<const uint4*>(p.lr + (size_t)n * p.r + 8 * c);
          *reinterpret_cast<uint4*>(sm.p + c * kChunkStride + t * 16) = vp;
          *reinterpret_cast<uint4*>(sm.l + c * kChunkStride + t * 16) = vl;
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.lr_full);
      }
      // this row's packed codes of one group, loaded a group ahead of their use
      auto load_codes = [&](int g, uint4 (&ca)[2], uint4 (&cb)[2]) {
        ca[0] = ca[1] = cb[0] = cb[1] = make_uint4(0, 0, 0, 0);
        if (g < p.NG && m < p.M) {
          const uint4* src = reinterpret_cast<const uint4*>(p.xc + (size_t)m * (p.K / 2) + 32 * g);
          ca[0] = src[0];
          ca[1] = src[1];
        }
        if (g < p.NG && n < p.N) {
          const uint4* src = reinterpret_cast<const uint4*>(p.wc + (size_t)n * (p.K / 2) + 32 * g);
          cb[0] = src[0];
          cb[1] = src[1];
        }
      };
      uint4 na[2], nb2[2];
      load_codes(0, na, nb2);
      for (int g = 0; g < p.NG; ++g, ++it) {
        const int s = it % kStages;
        const uint4 ca[2] = {na[0], na[1]}, cb[2] = {nb2[0], nb2[1]};
        load_codes(g + 1, na, nb2);
        if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t wa[4] = {ca[h].x, ca[h].y, ca[h].z, ca[h].w};
          const uint32_t wb[4] = {cb[h].x, cb[h].y, cb[h].z, cb[h].w};
#pragma unroll
          for (int q = 0; q < 2; ++q) {  // 16 int8 = one chunk from two words
            const uint2 a0 = widen8(wa[2 * q]), a1 = widen8(wa[2 * q + 1]);
            const uint2 b0 = widen8(wb[2 * q]), b1 = widen8(wb[2 * q + 1]);
            const int c = 2 * h + q;
            *reinterpret_cast<uint4*>(sm.a[s] + c * kChunkStride + t * 16) = make_uint4(a0.x, a0.y, a1.x, a1.y);
            *reinterpret_cast<uint4*>(sm.b[s] + c * kChunkStride + t * 16) = make_uint4(b0.x, b0.y, b1.x, b1.y);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.full[s]);
      }
    }
  } else if (warp == kProdWarps) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop and forms the descriptors; the elected
    // lane issues the tcgen05 ops.
    {
      uint32_t it = 0, gc = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tl) {
        for (int g = 0; g < p.NG; ++g, ++it, ++gc) {
          const int s = it % kStages;
          const int ab = gc % kAccBufs;
          if (!warp_wait(&sm.full[s], (it / kStages) & 1, p.wait_ns, p.err)) { ok = false; break; }
          if (!warp_wait(&sm.acce[ab], ((gc / kAccBufs) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_u32(sm.a[s]), b = smem_u32(sm.b[s]);
          uint64_t da[2], db[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            da[k] = make_sdesc(a + 2 * k * kChunkStride, kChunkStride, 128, kLayoutNone);
            db[k] = make_sdesc(b + 2 * k * kChunkStride, kChunkStride, 128, kLayoutNone);
          }
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 2; ++k) mma_i8(tmem + 128 * ab, da[k], db[k], kIdescI8, k ? 1u : 0u);
            tc_commit(&sm.empty[s]);
            tc_commit(&sm.accf[ab]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (has_lr) {
          if (!warp_wait(&sm.lr_full, tl & 1, p.wait_ns, p.err)) { ok = false; break; }
          if (!warp_wait(&sm.lr_acce, (tl & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pa = smem_u32(sm.p), la = smem_u32(sm.l);
          for (int k = 0; k < p.r / 16; ++k) {
            const uint64_t da = make_sdesc(pa + 2 * k * kChunkStride, kChunkStride, 128, kLayoutNone);
            const uint64_t db = make_sdesc(la + 2 * k * kChunkStride, kChunkStride, 128, kLayoutNone);
            if (elect_one()) mma_bf16(tmem + kLrCol, da, db, kIdescBf16, k ? 1u : 0u);
            __syncwarp();
          }
          if (elect_one()) {
            tc_commit(&sm.lr_empty);
            tc_commit(&sm.lr_accf);
          }
          __syncwarp();
        }
      }
      if (elect_one()) tc_commit(&sm.mma_done);
      __syncwarp();
      (void)warp_wait(&sm.mma_done, 0, p.wait_ns, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - (kProdWarps + 1);   // 0..7
    const int q = warp & 3;                    // TMEM lane quadrant
    const int h = ew >> 2;                     // columns [64 h, 64 h + 64)
    float* sw = sm.sw[ew];
    uint32_t gc = 0, tl = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tl) {
      const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN + 64 * h;
      const int m = m0 + 32 * q + lane;
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      bool ok = true;
      // this lane's two column scales and its row scale of a group (loaded a group ahead)
      auto load_scales = [&](int g, uint32_t& w2, float& sx) {
        w2 = 0;
        sx = 0.f;
        if (g < p.NG) {
          const int n = n0 + 2 * lane;
          if (n < p.N) w2 = *reinterpret_cast<const uint32_t*>(p.ws + (size_t)g * p.N + n);
          if (m < p.M) sx = bf16_bits_to_f32(p.xs[(size_t)m * p.NG + g]);
        }
      };
      uint32_t nw2;
      float nsx;
      load_scales(0, nw2, nsx);
      for (int g = 0; g < p.NG; ++g, ++gc) {
        const int ab = gc % kAccBufs;
        const uint32_t w2 = nw2;
        const float sx = nsx;
        load_scales(g + 1, nw2, nsx);
        // this group's 64 column scales, shared by the warp's lanes
        __syncwarp();
        *reinterpret_cast<float2*>(sw + 2 * lane) = make_float2(bf16_bits_to_f32(w2 & 0xFFFFu), bf16_bits_to_f32(w2 >> 16));
        __syncwarp();
        if (!mbar_wait(&sm.accf[ab], (gc / kAccBufs) & 1, p.wait_ns, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tb = tmem + 128 * ab + 64 * h + ((uint32_t)(32 * q) << 16);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + 32 * c, v);
          tmem_ld_wait();
          if (c == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acce[ab]);
          }
          if (p.out == 2) {
            if (m < p.M) {
              int32_t* o = static_cast<int32_t*>(p.y) + ((size_t)m * p.N + n0 + 32 * c) * p.NG + g;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n0 + 32 * c + j < p.N) o[(size_t)j * p.NG] = (int32_t)v[j];
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 s4 = *reinterpret_cast<const float4*>(sw + 32 * c + j);
              // exact int32 -> fp32 through the bits of 2^23 + 2^22 + s
              const float2 f01 = __fadd2_rn(make_float2(__uint_as_float(v[j] + 0x4B400000u),
                                                        __uint_as_float(v[j + 1] + 0x4B400000u)),
                                            make_float2(-12582912.0f, -12582912.0f));
              const float2 f23 = __fadd2_rn(make_float2(__uint_as_float(v[j + 2] + 0x4B400000u),
                                                        __uint_as_float(v[j + 3] + 0x4B400000u)),
                                            make_float2(-12582912.0f, -12582912.0f));
              const float2 s01 = __fmul2_rn(make_float2(s4.x, s4.y), make_float2(sx, sx));
              const float2 s23 = __fmul2_rn(make_float2(s4.z, s4.w), make_float2(sx, sx));
              const float2 a01 = __ffma2_rn(s01, f01, make_float2(acc[32 * c + j], acc[32 * c + j + 1]));
              const float2 a23 = __ffma2_rn(s23, f23, make_float2(acc[32 * c + j + 2], acc[32 * c + j + 3]));
              acc[32 * c + j] = a01.x;
              acc[32 * c + j + 1] = a01.y;
              acc[32 * c + j + 2] = a23.x;
              acc[32 * c + j + 3] = a23.y;
            }
          }
        }
      }
      if (!ok) break;
      if (has_lr) {
        if (!mbar_wait(&sm.lr_accf, tl & 1, p.wait_ns, p.err)) break;
        tc_fence_after();
        const uint32_t tb = tmem + kLrCol + 64 * h + ((uint32_t)(32 * q) << 16);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + 32 * c, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) acc[32 * c + j] += __uint_as_float(v[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.lr_acce);
      }
      if (p.out == 2 || m >= p.M) continue;
      // y = acc + bias; each thread writes its row's 64 columns
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int nb = n0 + 8 * c;
        if (nb >= p.N) break;  // N % 8 == 0: a group of 8 columns is all in or all out
        float o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = acc[8 * c + j] + (p.bias ? bf16_bits_to_f32(p.bias[nb + j]) : 0.f);
        if (p.out == 1) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.y) + (size_t)m * p.N + nb);
          dst[0] = make_float4(o[0], o[1], o[2], o[3]);
          dst[1] = make_float4(o[4], o[5], o[6], o[7]);
        } else {
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) w[j] = f32_to_bf16_bits(o[2 * j]) | (f32_to_bf16_bits(o[2 * j + 1]) << 16);
          *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.y) + (size_t)m * p.N + nb) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kProdWarps) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_int4(const GemmArgs& a, cudaStream_t s) {
  Params p;
  p.xc = a.x_codes;
  p.xs = static_cast<const uint16_t*>(a.x_scales);
  p.wc = a.w_codes;
  p.ws = static_cast<const uint16_t*>(a.w_scales);
  p.P = a.P;
  p.lr = a.lr_up;
  p.bias = a.bias;
  p.y = a.y;
  p.M = a.M; p.N = a.N; p.K = a.K; p.r = a.r; p.NG = a.K / 64;
  p.tiles_m = (a.M + BM - 1) / BM;
  p.tiles_n = (a.N + BN - 1) / BN;
  p.out = a.out;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_int4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < a.num_sms ? tiles : a.num_sms;
  gemm_int4_kernel<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace svdq
