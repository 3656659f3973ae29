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
// Data movement. A TMA warp streams each group's packed codes (128 rows x 32
// bytes of A and of B) through an 8-deep shared-memory ring, and the group
// scales in blocks of 8 groups (the tile's 128 x 8 activation scales and
// 8 x 128 weight scales) through a 3-deep ring, so no global load sits in the
// widening or in the drain.
//
// Widening. A nibble shifted into the high half of a byte is, read as int8,
// 16 q exactly (its sign bit lands on the byte's sign bit). So the odd
// elements of a packed word are w & 0xF0F0F0F0 and the even ones
// (w << 4) & 0xF0F0F0F0: three operations per eight codes. Both operands are
// widened the same way and laid out in the same K order (a word's even
// elements, then its odd ones), so every int32 group sum is 256 times the
// true one, still exact (|sum| <= 64 * 128 * 128 = 2^20).
//
// Drain. Each accumulator buffer is preloaded with 0x4B400000 and the MMAs
// accumulate onto it, so the int32 result is the bit pattern of the float
// 2^23 + 2^22 + 256 s, exact while |256 s| < 2^22. One packed subtraction
// gives 256 s as fp32; the scales are multiplied in with packed f32x2 ops,
// sx / 256 (exact) taking out the factor 256. After reading a buffer the
// epilogue writes the preload back before releasing it to the MMA warp.
//
// Roles (384 threads, 12 warps, so that each SM sub-partition holds three and
// a thread may use up to 168 registers): warps 0-1 producers (two tile rows
// per thread: widen the rows' codes from the packed ring into the K-major
// int8 stage), warp 2 TMEM allocator + MMA issuer, warps 3-10 epilogue (two
// per TMEM lane quadrant, each holding the running sums of 64 columns),
// warp 11 TMA.
// Tile 128 x 128, one group per int8 stage, 4 stages.
// INT4 activation scales are row-major [M, K/64] with the row pitch padded to
// a multiple of 8 groups; weight scales are group-major [K/64, N].
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 128, BKG = 64;     // one group per stage
constexpr int kStages = 4;                      // int8 stages
constexpr int kPk = 8;                          // packed-code ring (one group each)
constexpr int kSc = 3;                          // scale ring (8 groups each)
constexpr int kScG = 8;                         // groups per scale block
constexpr int kOpBytes = 128 * BKG;             // int8 tile, 8 KB
constexpr int kPkBytes = 128 * BKG / 2;         // packed tile, 4 KB
constexpr int kChunkStride = 128 * 16;          // bytes between 16-byte K chunks
constexpr int kMaxR = 64;
constexpr int kLrBytes = 128 * kMaxR * 2;       // 16 KB
constexpr int kProdWarps = 2, kEpiWarps = 8;
constexpr int kMmaWarp = kProdWarps, kTmaWarp = kProdWarps + 1 + kEpiWarps;
constexpr int kThreads = 32 * (kTmaWarp + 1);
constexpr uint32_t kTmemCols = 512;
constexpr int kAccBufs = 3;                     // int32 group accumulators, 128 columns each
constexpr uint32_t kLrCol = 128 * kAccBufs;     // 384: the low-rank fp32 accumulator
constexpr uint32_t kMagic = 0x4B400000u;        // float bits of 2^23 + 2^22

// kind::i8: D s32, A/B signed int8, K-major, M = 128, N = 128
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                              ((uint32_t)(BM >> 4) << 24);
// kind::f16: D f32, A/B bf16
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(BM >> 4) << 24);

struct Smem {
  uint8_t a[kStages][kOpBytes];
  uint8_t b[kStages][kOpBytes];
  uint8_t pa[kPk][kPkBytes];                    // [128 rows][32 bytes], as TMA writes it
  uint8_t pb[kPk][kPkBytes];
  uint16_t sx[kSc][128 * kScG];                 // [128 rows][8 groups] bf16
  uint16_t sw[kSc][kScG * 128];                 // [8 groups][128 columns] bf16
  uint8_t p[kLrBytes];
  uint8_t l[kLrBytes];
  float swf[kEpiWarps][kScG][64];               // each epilogue warp's column scales, fp32
  float sxf[kEpiWarps][kScG][32];               // and its rows' activation scales / 256
  uint64_t full[kStages], empty[kStages];
  uint64_t pk_full[kPk], pk_empty[kPk];
  uint64_t sc_full[kSc], sc_empty[kSc];
  uint64_t accf[kAccBufs], acce[kAccBufs];
  uint64_t lr_full, lr_empty, lr_accf, lr_acce, mma_done;
  uint32_t tmem_base;
};

struct Params {
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

// 16 times the even / odd int4 elements of a packed word, as four int8 each
__device__ __forceinline__ uint32_t even16(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t odd16(uint32_t w) { return w & 0xF0F0F0F0u; }

// Each thread writes `v` into 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
      "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_xc, const __grid_constant__ CUtensorMap tm_wc,
                 const __grid_constant__ CUtensorMap tm_xs, const __grid_constant__ CUtensorMap tm_ws,
                 const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_align<1024>(smem_raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int nblk = (p.NG + kScG - 1) / kScG;  // scale blocks per tile
  const bool has_lr = p.r > 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], kProdWarps);
      mbar_init(&sm.empty[s], 1);
    }
    for (int s = 0; s < kPk; ++s) {
      mbar_init(&sm.pk_full[s], 1);
      mbar_init(&sm.pk_empty[s], kProdWarps);
    }
    for (int s = 0; s < kSc; ++s) {
      mbar_init(&sm.sc_full[s], 1);
      mbar_init(&sm.sc_empty[s], kEpiWarps);
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
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  const bool is_epi = warp > kMmaWarp && warp < kTmaWarp;
  const int ew = warp - (kMmaWarp + 1);        // epilogue warp 0..7
  const int q = warp & 3;                      // its TMEM lane quadrant
  const int h = ew >> 2;                       // its columns [64 h, 64 h + 64)
  if (is_epi) {
    // preload every accumulator buffer before the first MMA
#pragma unroll
    for (int b = 0; b < kAccBufs; ++b) {
      const uint32_t tb = tmem + 128 * b + 64 * h + ((uint32_t)(32 * q) << 16);
      tmem_fill32(tb, kMagic);
      tmem_fill32(tb + 32, kMagic);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&tm_xc);
      tma_prefetch_desc(&tm_wc);
      tma_prefetch_desc(&tm_xs);
      tma_prefetch_desc(&tm_ws);
      uint32_t it = 0, scc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN;
        for (int g = 0; g < p.NG; ++g, ++it) {
          if (g % kScG == 0) {
            const int ss = scc % kSc;
            if (!mbar_wait(&sm.sc_empty[ss], ((scc / kSc) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
            mbar_expect_tx(&sm.sc_full[ss], 2 * 128 * kScG * 2);
            tma_load_2d(sm.sx[ss], &tm_xs, &sm.sc_full[ss], g, m0);
            tma_load_2d(sm.sw[ss], &tm_ws, &sm.sc_full[ss], n0, g);
            ++scc;
          }
          const int ps = it % kPk;
          if (!mbar_wait(&sm.pk_empty[ps], ((it / kPk) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          mbar_expect_tx(&sm.pk_full[ps], 2 * kPkBytes);
          tma_load_2d(sm.pa[ps], &tm_xc, &sm.pk_full[ps], 32 * g, m0);
          tma_load_2d(sm.pb[ps], &tm_wc, &sm.pk_full[ps], 32 * g, n0);
        }
      }
      if (!ok) {
        // let the copies still in flight land before the CTA can exit (bounded)
        for (uint32_t j = it > (uint32_t)kPk ? it - kPk : 0u; j < it; ++j)
          (void)mbar_wait(&sm.pk_full[j % kPk], (j / kPk) & 1, p.wait_ns, nullptr);
        for (uint32_t j = scc > (uint32_t)kSc ? scc - kSc : 0u; j < scc; ++j)
          (void)mbar_wait(&sm.sc_full[j % kSc], (j / kSc) & 1, p.wait_ns, nullptr);
      }
    }
    __syncwarp();
  } else if (warp < kProdWarps) {
    // ------------------------------------------------------------ producers
    const int t0 = threadIdx.x;  // rows t0 and t0 + 64 of the tile
    uint32_t it = 0, tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tl) {
      const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN;
      if (has_lr) {
        if (!mbar_wait(&sm.lr_empty, (tl & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
        for (int rr = 0; rr < 2; ++rr) {
          const int t = t0 + 64 * rr, m = m0 + t, n = n0 + t;
          for (int c = 0; c < p.r / 8; ++c) {
            uint4 vp = make_uint4(0, 0, 0, 0), vl = make_uint4(0, 0, 0, 0);
            if (m < p.M) vp = *reinterpret_cast<const uint4*>(p.P + (size_t)m * p.r + 8 * c);
            if (n < p.N) vl = *reinterpret_cast<const uint4*>(p.lr + (size_t)n * p.r + 8 * c);
            *reinterpret_cast<uint4*>(sm.p + c * kChunkStride + t * 16) = vp;
            *reinterpret_cast<uint4*>(sm.l + c * kChunkStride + t * 16) = vl;
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&sm.lr_full);
      }
      for (int g = 0; g < p.NG; ++g, ++it) {
        const int ps = it % kPk, s = it % kStages;
        if (!warp_wait(&sm.pk_full[ps], (it / kPk) & 1, p.wait_ns, p.err)) { ok = false; break; }
        uint4 ra[2][2], rb[2][2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const uint4* sa = reinterpret_cast<const uint4*>(sm.pa[ps] + 32 * (t0 + 64 * rr));
          const uint4* sb = reinterpret_cast<const uint4*>(sm.pb[ps] + 32 * (t0 + 64 * rr));
          ra[rr][0] = sa[0];
          ra[rr][1] = sa[1];
          rb[rr][0] = sb[0];
          rb[rr][1] = sb[1];
        }
        if (!warp_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int t = t0 + 64 * rr;
          const uint32_t wa[8] = {ra[rr][0].x, ra[rr][0].y, ra[rr][0].z, ra[rr][0].w,
                                  ra[rr][1].x, ra[rr][1].y, ra[rr][1].z, ra[rr][1].w};
          const uint32_t wb[8] = {rb[rr][0].x, rb[rr][0].y, rb[rr][0].z, rb[rr][0].w,
                                  rb[rr][1].x, rb[rr][1].y, rb[rr][1].z, rb[rr][1].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // 16 int8 = one K chunk from two words
            *reinterpret_cast<uint4*>(sm.a[s] + c * kChunkStride + t * 16) =
                make_uint4(even16(wa[2 * c]), odd16(wa[2 * c]), even16(wa[2 * c + 1]), odd16(wa[2 * c + 1]));
            *reinterpret_cast<uint4*>(sm.b[s] + c * kChunkStride + t * 16) =
                make_uint4(even16(wb[2 * c]), odd16(wb[2 * c]), even16(wb[2 * c + 1]), odd16(wb[2 * c + 1]));
          }
        }
        // The packed stage is released only now: the int8 stores above use
        // the loaded codes, so every lane's shared loads have returned. (An
        // arrive right after issuing the loads can complete before they read
        // the stage, and the next TMA write then overtakes them.)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.full[s]);
          mbar_arrive(&sm.pk_empty[ps]);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop and forms the descriptors; the elected
    // lane issues the tcgen05 ops.
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
          // onto the preloaded buffer
#pragma unroll
          for (int k = 0; k < 2; ++k) mma_i8(tmem + 128 * ab, da[k], db[k], kIdescI8, 1u);
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
  } else {
    // ------------------------------------------------------------ epilogue
    float (*swf)[64] = sm.swf[ew];
    float (*sxf)[32] = sm.sxf[ew];
    const int row = 32 * q + lane;             // this thread's row of the tile
    uint32_t gc = 0, scc = 0, tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tl) {
      const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN + 64 * h;
      const int m = m0 + row;
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      for (int blk = 0; blk < nblk && ok; ++blk) {
        // this block's scales: the warp's 64 column scales of 8 groups to fp32
        // in its own staging, and this row's 8 activation scales / 256
        const int ss = scc % kSc;
        if (!warp_wait(&sm.sc_full[ss], (scc / kSc) & 1, p.wait_ns, p.err)) { ok = false; break; }
        {
          const int jj = lane >> 2, c0 = (lane & 3) * 16;
          const uint4* src = reinterpret_cast<const uint4*>(sm.sw[ss] + jj * 128 + 64 * h + c0);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint4 v = src[u];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            float4* dst = reinterpret_cast<float4*>(&swf[jj][c0 + 8 * u]);
            dst[0] = make_float4(bf16_bits_to_f32(w[0] & 0xFFFFu), bf16_bits_to_f32(w[0] >> 16),
                                 bf16_bits_to_f32(w[1] & 0xFFFFu), bf16_bits_to_f32(w[1] >> 16));
            dst[1] = make_float4(bf16_bits_to_f32(w[2] & 0xFFFFu), bf16_bits_to_f32(w[2] >> 16),
                                 bf16_bits_to_f32(w[3] & 0xFFFFu), bf16_bits_to_f32(w[3] >> 16));
          }
        }
        {
          const uint4 v = *reinterpret_cast<const uint4*>(sm.sx[ss] + row * kScG);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            sxf[2 * i][lane] = bf16_bits_to_f32(w[i] & 0xFFFFu) * (1.0f / 256.0f);
            sxf[2 * i + 1][lane] = bf16_bits_to_f32(w[i] >> 16) * (1.0f / 256.0f);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sc_empty[ss]);
        ++scc;
#pragma unroll 1
        for (int j = 0; j < kScG; ++j) {
          const int g = blk * kScG + j;
          if (g >= p.NG) break;
          const int ab = gc % kAccBufs;
          if (!warp_wait(&sm.accf[ab], (gc / kAccBufs) & 1, p.wait_ns, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tb = tmem + 128 * ab + 64 * h + ((uint32_t)(32 * q) << 16);
          const float sx = sxf[j][lane];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(tb + 32 * c, v);
            tmem_ld_wait();
            tmem_regs_ready(v);
            tmem_fill32(tb + 32 * c, kMagic);  // the preload for the buffer's next group
            if (c == 1) {
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.acce[ab]);
            }
            if (p.out == 2) {
              if (m < p.M) {
                int32_t* o = static_cast<int32_t*>(p.y) + ((size_t)m * p.N + n0 + 32 * c) * p.NG + g;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (n0 + 32 * c + i < p.N) o[(size_t)i * p.NG] = ((int32_t)(v[i] - kMagic)) >> 8;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 s4 = *reinterpret_cast<const float4*>(&swf[j][32 * c + i]);
                // 256 s, exact: the preloaded bits minus 2^23 + 2^22
                const float2 f01 = __fadd2_rn(make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                                              make_float2(-12582912.0f, -12582912.0f));
                const float2 f23 = __fadd2_rn(make_float2(__uint_as_float(v[i + 2]), __uint_as_float(v[i + 3])),
                                              make_float2(-12582912.0f, -12582912.0f));
                const float2 s01 = __fmul2_rn(make_float2(s4.x, s4.y), make_float2(sx, sx));
                const float2 s23 = __fmul2_rn(make_float2(s4.z, s4.w), make_float2(sx, sx));
                const float2 a01 = __ffma2_rn(s01, f01, make_float2(acc[32 * c + i], acc[32 * c + i + 1]));
                const float2 a23 = __ffma2_rn(s23, f23, make_float2(acc[32 * c + i + 2], acc[32 * c + i + 3]));
                acc[32 * c + i] = a01.x;
                acc[32 * c + i + 1] = a01.y;
                acc[32 * c + i + 2] = a23.x;
                acc[32 * c + i + 3] = a23.y;
              }
            }
          }
          ++gc;
        }
        // the staging is rewritten by the next block: every lane is done with it
        __syncwarp();
      }
      if (!ok) break;
      if (has_lr) {
        if (!warp_wait(&sm.lr_accf, tl & 1, p.wait_ns, p.err)) break;
        tc_fence_after();
        const uint32_t tb = tmem + kLrCol + 64 * h + ((uint32_t)(32 * q) << 16);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + 32 * c, v);
          tmem_ld_wait();
          tmem_regs_ready(v);
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
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_int4(const GemmArgs& a, cudaStream_t s) {
  Params p;
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
  // packed codes: [rows, K/2] bytes, one group = a 32-byte x 128-row box;
  // activation scales [M, pitch] bf16, box 8 groups x 128 rows; weight scales
  // [K/64, N] bf16, box 128 columns x 8 groups (rows / groups past the end read as 0)
  CUtensorMap tm_xc, tm_wc, tm_xs, tm_ws;
  const uint64_t kb = (uint64_t)a.K / 2;
  bool ok = make_tmap_2d(&tm_xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.x_codes, kb, a.M, kb, 32, BM,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_tmap_2d(&tm_wc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, kb, a.N, kb, 32, BN,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_tmap_2d(&tm_xs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x_scales, p.NG, a.M,
                          (uint64_t)int4_act_scale_pitch(a.K) * 2, kScG, BM, CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_tmap_2d(&tm_ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.w_scales, a.N, p.NG, (uint64_t)a.N * 2, BN,
                          kScG, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(gemm_int4_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n;
  const int grid = tiles < a.num_sms ? tiles : a.num_sms;
  gemm_int4_kernel<<<grid, kThreads, smem, s>>>(tm_xc, tm_wc, tm_xs, tm_ws, p);
  return cudaGetLastError();
}

}  // namespace svdq
