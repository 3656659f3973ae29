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
// sm_100a design: persistent, warp-specialised CTA pairs (cluster of 2). The
// pair computes a 256 (M) x 256 (N) tile with tcgen05.mma.cta_group::2: each
// CTA holds 128 rows of A and 128 rows of B in its own shared memory and 128
// accumulator lanes x 256 fp32 columns in its own tensor memory, so each SM
// streams half of B and the tensor cores run at their full per-SM rate.
//   warp 0      TMA producer (both CTAs): A/B code tiles (128B-swizzled,
//               K-major) and UE4M3 scale atoms for its own rows; both CTAs'
//               copies complete on the leader CTA's stage barrier. One extra
//               stage opens each tile with the P tile and the prepared L2 tile.
//   warp 1      TMEM allocator (both CTAs); in the leader CTA one thread
//               issues, per 256-wide K stage, tcgen05.cp of the scale atoms
//               (into both CTAs' tensor memory) and 4 x tcgen05.mma
//               kind::mxf4nvf4 (K = 64); before the K loop, tcgen05.mma
//               kind::f16 puts P (hi + lo) into the same accumulator.
//   warps 2..9  epilogue (both CTAs), two warps per TMEM lane quadrant, each
//               draining half of the 256 columns: tcgen05.ld, y = alpha*acc +
//               bias (read through the L1 cache), convert, stage 32 x 64
//               pieces in 128B-swizzled shared memory, TMA store. With the
//               fused QKV epilogue (svdq_w4a4_linear_qkv) a half is one head
//               of 128 columns: Q and K heads are RMS-normalised and rotated
//               before the store. With the GELU output mode the layer
//               output goes through GELU before its rounding (the
//               up-projection of the fused GELU-MLP).
// Accumulators: two 256-column buffers overlapping in 64 columns
// ([0,256) and [192,448); scales in [448,512)). Per tile, the epilogue half
// that holds the overlapped 64 columns drains them first and then releases
// the tile; the other half releases it as soon as it has finished the
// previous tile. The next tile's MMAs therefore start after an eighth of the
// drain, and the output stores run under the next tile's mainloop. One
// release barrier per accumulator buffer keeps the arrivals of consecutive
// tiles apart. Every mbarrier wait is bounded in wall time.
#include "device.cuh"
#include "kernels.h"

namespace svdq {
namespace {

constexpr int BM = 128, BN = 256, BK = 256;    // per-CTA rows, pair N, K per stage (FP4 elements)
constexpr int kStages = 5;
constexpr int kABytes = BM * BK / 2;            // 16 KB
constexpr int kBBytes = (BN / 2) * BK / 2;      // 16 KB (this CTA's half of the N tile)
constexpr int kSfaBytes = 4 * 512;              // 4 K-atoms x 128 rows
constexpr int kSfbBytes = 2 * 4 * 512;          // the pair's 256 N rows x 4 K-atoms (both CTAs)
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr uint32_t kStageTx = 2u * kStageBytes;
constexpr int kEpiWarps = 8;
constexpr int kSlotBytes = 32 * 128;            // 32 rows x 128 bytes (one TMA store box)
constexpr int kSlots = 1;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol0 = 0, kAccCol1 = 192;
constexpr uint32_t kSfaCol = 448, kSfbCol = 464;

constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
constexpr uint32_t kIdescBf16 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                ((uint32_t)(256 >> 4) << 24);

struct Smem {
  uint8_t stage[kStages][kStageBytes];          // 1024-aligned (kStageBytes % 1024 == 0)
  uint8_t out[kEpiWarps][kSlots][kSlotBytes];
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_free[2], mma_done;
  uint32_t tmem_base;
};
static_assert(kStageBytes % 1024 == 0, "stage alignment");

struct Params {
  const float* tensor_scale;
  const uint16_t* bias;
  int M, N, K, r;
  int tiles_m, tiles_n;   // tiles_m counts 256-row pair tiles
  int out_f32;
  unsigned* err;
  unsigned long long wait_ns;
  // fused QKV epilogue (qkv_heads > 0): N = 3 * qkv_heads * 128, Q, K, V in
  // that order; RMSNorm weights [128] of Q and K heads, eps, the rotary
  // tables in the packed layout of svdq_rope_pack
  int qkv_heads;
  const uint16_t* norm_q;
  const uint16_t* norm_k;
  float eps;
  const float* rope;
};

// Output of 32 columns of a Q or K head (head columns hc0 .. hc0 + 31, in
// registers as fp32 layer outputs y): u = y * inv * w, then the rotary
// embedding of each adjacent pair (2i, 2i+1) by the row's angle i, rounded to
// bf16 into 16-byte units u0 .. u0 + 3 of the 128B-swizzled staging row.
// The norm weights and the lane's row's cos/sin of 32 head columns hc0 ..
// hc0 + 31 (loaded ahead of their use: the tables come from L2). rope_lane
// points at the lane's row in its 32-row block of the packed table: a group
// of 4 rotary pairs (8 head columns) is a cos part and a sin part of
// [32 rows][4], so the warp's 32 rows read 512 contiguous bytes per load.
struct QkvTables {
  uint4 w[4];
  float4 c[4], s[4];
};
__device__ __forceinline__ void qkv_tables(QkvTables& t, int hc0, const uint16_t* w, const float* rope_lane) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int hc = hc0 + 8 * u;
    t.w[u] = __ldg(reinterpret_cast<const uint4*>(w + hc));
    t.c[u] = __ldg(reinterpret_cast<const float4*>(rope_lane + (hc / 8) * 256));
    t.s[u] = __ldg(reinterpret_cast<const float4*>(rope_lane + (hc / 8) * 256 + 128));
  }
}

// Output of 32 columns of a Q or K head (in registers as fp32 layer outputs
// y, with their tables): u = y * inv * w, then the rotary embedding of each
// adjacent pair (2i, 2i+1) by the row's angle i, rounded to bf16 into 16-byte
// units u0 .. u0 + 3 of the 128B-swizzled staging row.
__device__ __forceinline__ void qkv_out32(uint8_t* buf, int lane, const float (&y)[32], int u0, float inv,
                                          const QkvTables& t) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint32_t ww[4] = {t.w[u].x, t.w[u].y, t.w[u].z, t.w[u].w};
    const float cs[4] = {t.c[u].x, t.c[u].y, t.c[u].z, t.c[u].w}, sn[4] = {t.s[u].x, t.s[u].y, t.s[u].z, t.s[u].w};
    uint32_t w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a0 = y[8 * u + 2 * k] * inv * bf16_bits_to_f32(ww[k] & 0xFFFFu);
      const float a1 = y[8 * u + 2 * k + 1] * inv * bf16_bits_to_f32(ww[k] >> 16);
      const float o0 = fmaf(a0, cs[k], -a1 * sn[k]);
      const float o1 = fmaf(a0, sn[k], a1 * cs[k]);
      w4[k] = f32_to_bf16_bits(o0) | (f32_to_bf16_bits(o1) << 16);
    }
    *reinterpret_cast<uint4*>(buf + lane * 128 + (((u0 + u) ^ (lane & 7)) * 16)) =
        make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

// bf16 of 32 layer outputs into 16-byte units u0 .. u0 + 3 of the staging row
__device__ __forceinline__ void plain_out32(uint8_t* buf, int lane, const float (&y)[32], int u0) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w4[k] = f32_to_bf16_bits(y[8 * u + 2 * k]) | (f32_to_bf16_bits(y[8 * u + 2 * k + 1]) << 16);
    *reinterpret_cast<uint4*>(buf + lane * 128 + (((u0 + u) ^ (lane & 7)) * 16)) =
        make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

// y = alpha * acc + bias of 32 consecutive columns starting at column n
__device__ __forceinline__ void layer_out32(float (&y)[32], const uint32_t (&acc)[32], float alpha,
                                            const uint16_t* bias, int n) {
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const uint32_t bw = bias ? __ldg(reinterpret_cast<const uint32_t*>(bias + n + c)) : 0u;
    y[c] = fmaf(alpha, __uint_as_float(acc[c]), bf16_bits_to_f32(bw & 0xFFFFu));
    y[c + 1] = fmaf(alpha, __uint_as_float(acc[c + 1]), bf16_bits_to_f32(bw >> 16));
  }
}


// The column tile of tile sequence index t % tiles_n. With the fused QKV
// epilogue and a whole number of tiles per Q/K/V section, the column tiles of
// the three sections are interleaved (Q0, K0, V0, Q1, ...), so that the tiles
// a CTA pair takes in turn mix the costly Q/K epilogues with plain V ones.
__device__ __forceinline__ int column_tile(int t, int tiles_n, bool interleave) {
  if (!interleave) return t;
  const int per = tiles_n / 3;
  return (t % 3) * per + t / 3;
}

// Epilogue of the instance: kEpiPlain (y = alpha acc + bias), kEpiQkv (the
// fused QKV epilogue) or kEpiGelu (GELU of the layer output before its
// rounding: the up-projection of the fused GELU-MLP). Separate instances, so
// that the plain GEMM's register allocation carries neither.
constexpr int kEpiPlain = 0, kEpiQkv = 1, kEpiGelu = 2;

// GELU, erf form: y (1 + erf(y / sqrt 2)) / 2 in fp32
__device__ __forceinline__ float gelu_erf(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

template <int kEpi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                  const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_l,
                  const __grid_constant__ CUtensorMap tm_y, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_align<1024>(smem_raw));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_tiles = p.tiles_m * p.tiles_n;
  const int nk = (p.K + BK - 1) / BK;
  const bool has_lr = p.r > 0;
  // interleave the sections' column tiles when each section is whole tiles
  const bool qkv_mix = kEpi == kEpiQkv && p.tiles_n % 3 == 0 && p.qkv_heads % 2 == 0 && p.qkv_heads / 2 * 3 == p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full[0], 1);
    mbar_init(&sm.acc_full[1], 1);
    mbar_init(&sm.acc_free[0], 2 * kEpiWarps);
    mbar_init(&sm.acc_free[1], 2 * kEpiWarps);
    mbar_init(&sm.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_sfa);
    tma_prefetch_desc(&tm_sfb);
    tma_prefetch_desc(&tm_y);
    if (has_lr) {
      tma_prefetch_desc(&tm_p);
      tma_prefetch_desc(&tm_l);
    }
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // Programmatic dependent launch: the set-up above (barriers, tensor memory,
  // tensor-map prefetch) may overlap the previous kernel in the stream; every
  // input may be that kernel's output (the activation pass writes A, its
  // scales and P) and y may still be read by it, so all global traffic comes
  // after this wait. The next kernel may be scheduled at once: it waits for
  // this one before it touches anything this one reads or writes.
  if (threadIdx.x == 0) launch_dependents();
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        const int tm = tile / p.tiles_n, tn = column_tile(tile % p.tiles_n, p.tiles_n, qkv_mix);
        const int row0 = tm * 256 + (int)rank * BM;      // this CTA's A rows
        const int col0 = tn * BN + (int)rank * (BN / 2);  // this CTA's B rows
        if (has_lr) {
          // the low-rank stage opens the tile, so its loads are hidden behind
          // the K stages that follow it like any other stage's
          const int s = it % kStages;
          if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          uint8_t* st = sm.stage[s];
          const uint32_t fb = mapa_shared(smem_u32(&sm.full[s]), 0);
          const int pc = p.r / 8, lc = 2 * p.r / 8;  // 8-column groups
          if (leader) mbar_expect_tx(&sm.full[s], 2u * (uint32_t)(pc + lc) * BM * 16);
          // one copy each: [group][row][8 columns], the K-major core-matrix layout
          tma_load_3d_pair(st, &tm_p, fb, 0, row0, 0);
          tma_load_3d_pair(st + kABytes, &tm_l, fb, 0, col0, 0);
          ++it;
        }
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns, p.err)) { ok = false; break; }
          uint8_t* st = sm.stage[s];
          const uint32_t fb = mapa_shared(smem_u32(&sm.full[s]), 0);
          if (leader) mbar_expect_tx(&sm.full[s], kStageTx);
          tma_load_2d_pair(st, &tm_a, fb, kb * (BK / 2), row0);
          tma_load_2d_pair(st + kABytes, &tm_b, fb, kb * (BK / 2), col0);
          tma_load_3d_pair(st + kABytes + kBBytes, &tm_sfa, fb, 0, 4 * kb, row0 / 128);
          tma_load_3d_pair(st + kABytes + kBBytes + kSfaBytes, &tm_sfb, fb, 0, 4 * kb, 2 * tn);
        }
        if (!ok) break;
      }
      if (!ok && leader) {
        // let the copies already issued by both CTAs land before the pair exits
        for (uint32_t d = 1; d <= (uint32_t)kStages && d <= it; ++d) {
          const uint32_t j = it - d;
          (void)mbar_wait(&sm.full[j % kStages], (j / kStages) & 1, p.wait_ns, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    // The whole warp walks the loop; one lane issues the tcgen05 ops.
    if (leader) {
      uint32_t it = 0;
      bool ok = true;
      int i = 0;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++i) {
        const uint32_t acc = tmem + ((i & 1) ? kAccCol1 : kAccCol0);
        // tile i - 1 released: its overlapped columns are drained and tile
        // i - 2 (the previous user of this buffer) is drained completely
        if (i > 0 && !__all_sync(0xffffffffu, mbar_wait_cluster(&sm.acc_free[(i - 1) & 1], ((i - 1) >> 1) & 1,
                                                                 p.wait_ns, p.err))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (has_lr) {
          // P (hi + lo) first: it opens the accumulator of the tile
          const int s = it % kStages;
          if (!warp_wait(&sm.full[s], (it / kStages) & 1, p.wait_ns, p.err)) { ok = false; break; }
          const uint32_t st = smem_u32(sm.stage[s]);
          const int half = p.r / 16;  // k16 steps per copy of P
          for (int k = 0; k < 2 * half; ++k) {
            const int kp = k % half;
            const uint64_t ad = make_sdesc(st + 2 * kp * BM * 16, BM * 16, 128, kLayoutNone);
            const uint64_t bd = make_sdesc(st + kABytes + 2 * k * BM * 16, BM * 16, 128, kLayoutNone);
            if (elect_one()) mma_bf16_pair(acc, ad, bd, kIdescBf16, k > 0 ? 1u : 0u);
            __syncwarp();
          }
          if (elect_one()) tc_commit_pair(&sm.empty[s], 0x3);
          __syncwarp();
          ++it;
        }
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!warp_wait(&sm.full[s], (it / kStages) & 1, p.wait_ns, p.err)) { ok = false; break; }
          const uint32_t st = smem_u32(sm.stage[s]);
          const uint32_t sfa = st + kABytes + kBBytes, sfb = sfa + kSfaBytes;
          // Descriptors are formed by the whole warp (warp-uniform values) and
          // the ops issued by the elected lane; building them inside a
          // one-lane branch made every tcgen05 op markedly slower to issue.
          uint64_t dcp[12], da[4], db[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dcp[3 * j] = make_sdesc(sfa + 512 * j, 512, 128, kLayoutNone);
            dcp[3 * j + 1] = make_sdesc(sfb + 512 * j, 512, 128, kLayoutNone);
            dcp[3 * j + 2] = make_sdesc(sfb + 2048 + 512 * j, 512, 128, kLayoutNone);
            da[j] = make_sdesc(st + 32 * j, 16, 1024, kLayoutSw128);
            db[j] = make_sdesc(st + kABytes + 32 * j, 16, 1024, kLayoutSw128);
          }
          if (elect_one()) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_32x128b_warpx4_pair(tmem + kSfaCol + 4 * j, dcp[3 * j]);
              tc_cp_32x128b_warpx4_pair(tmem + kSfbCol + 8 * j, dcp[3 * j + 1]);
              tc_cp_32x128b_warpx4_pair(tmem + kSfbCol + 8 * j + 4, dcp[3 * j + 2]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_nvfp4_pair(acc, da[j], db[j], kIdescNvfp4, tmem + kSfaCol + 4 * j, tmem + kSfbCol + 8 * j,
                             (has_lr || kb > 0 || j > 0) ? 1u : 0u);
            tc_commit_pair(&sm.empty[s], 0x3);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair(&sm.acc_full[i & 1], 0x3);
        __syncwarp();
      }
      // every MMA issued has completed before tensor memory is freed
      if (elect_one()) tc_commit_pair(&sm.mma_done, 0x1);
      __syncwarp();
      (void)warp_wait(&sm.mma_done, 0, p.wait_ns, p.err);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int e = warp - 2;              // epilogue warp index (staging slots)
    const int h = e >> 2;                // column half: [128 h, 128 h + 128)
    const float alpha = __fmul_rn(p.tensor_scale[0], p.tensor_scale[1]);
    const int cols = p.out_f32 ? 32 : 64;          // columns per chunk
    const int nchunks = (BN / 2) / cols;           // chunks per half
    const int overlap_chunks = 64 / cols;          // chunks covering the 64 shared columns
    int i = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs, ++i) {
      const int tm = tile / p.tiles_n, tn = column_tile(tile % p.tiles_n, p.tiles_n, qkv_mix);
      const int row0 = tm * 256 + (int)rank * BM + 32 * q;
      const int n0 = tn * BN + 128 * h;
      const int b = i & 1;
      // buffer 0 shares its top 64 columns (half 1), buffer 1 its bottom 64 (half 0)
      const bool holds_overlap = (b == 0) == (h == 1);
      const uint32_t free_bar = mapa_shared(smem_u32(&sm.acc_free[b]), 0);
      if (!holds_overlap) {
        // this warp is done with the previous tile: release this one for it
        tc_fence_before();
        if (lane == 0) mbar_arrive_cluster(free_bar);
      }
      if (!mbar_wait(&sm.acc_full[b], (i >> 1) & 1, p.wait_ns, p.err)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (b ? kAccCol1 : kAccCol0) + 128 * h + ((uint32_t)(32 * q) << 16);
      if constexpr (kEpi == kEpiQkv) {
        // Fused QKV epilogue: the warp's half of the tile is one head of 128
        // columns, 2 tn + h. A Q or K head is normalised over its 128 columns
        // (RMSNorm of the layer output before its rounding) and rotated; a V
        // head takes the plain epilogue below.
        const int head = 2 * tn + h;
        const int sect = head / p.qkv_heads;
        const int cf = (b == 0 && h == 1) ? 1 : 0, cs = 1 - cf;  // chunk order: the shared columns first
        if (sect >= 2 || head * 128 >= p.N) {
          // V head (or past N): the layer output, 32 columns at a time
#pragma unroll 1
          for (int part = 0; part < 2; ++part) {
            const int c = part == 0 ? cf : cs;
            const int nc = tn * BN + 128 * h + 64 * c;
            if (lane == 0) bulk_wait_read<kSlots - 1>();
            __syncwarp();
            uint8_t* buf = sm.out[e][0];
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t v[32];
              float t[32];
              tmem_ld32(tbase + 64 * c + 32 * hh, v);
              tmem_ld_wait();
              tmem_regs_ready(v);
              if (holds_overlap && part == 0 && hh == 1) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(free_bar);
              }
              layer_out32(t, v, alpha, nc < p.N ? p.bias : nullptr, nc + 32 * hh);
              plain_out32(buf, lane, t, 4 * hh);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 < p.M && nc < p.N) tma_store_2d(&tm_y, buf, nc, row0);
              bulk_commit();
            }
          }
          continue;
        }
        {
          const uint16_t* wn = sect == 0 ? p.norm_q : p.norm_k;
          const int nh = head * 128;
          // the warp's 32 rows are one block of the packed table (a quadrant
          // wholly past M reads the last block: its rows are not stored)
          const int blk = (row0 < p.M ? row0 : p.M - 1) / 32;
          const float* rope_lane = p.rope + (size_t)blk * 4096 + 4 * lane;
          // the 64-column chunk that holds the shared columns (when this warp
          // holds them) first: its layer outputs stay in registers; the other
          // chunk is read once for the sum of squares and again for the output
          float ya[32], yb[32];
          // sum of squares in a fixed order, whatever the chunk order: per
          // chunk even and odd columns in increasing order, then chunk 0 +
          // chunk 1 (the result does not depend on the tile schedule)
          float sf0 = 0.f, sf1 = 0.f, ss0 = 0.f, ss1 = 0.f;
          {
            uint32_t v[32];
            tmem_ld32(tbase + 64 * cf, v);
            tmem_ld_wait();
            tmem_regs_ready(v);
            layer_out32(ya, v, alpha, p.bias, nh + 64 * cf);
            tmem_ld32(tbase + 64 * cf + 32, v);
            tmem_ld_wait();
            tmem_regs_ready(v);
            if (holds_overlap) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(free_bar);
            }
            layer_out32(yb, v, alpha, p.bias, nh + 64 * cf + 32);
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              sf0 = fmaf(ya[c], ya[c], sf0);
              sf1 = fmaf(ya[c + 1], ya[c + 1], sf1);
            }
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              sf0 = fmaf(yb[c], yb[c], sf0);
              sf1 = fmaf(yb[c + 1], yb[c + 1], sf1);
            }
          }
          // the first output slice's tables load under the sum-of-squares pass
          QkvTables tab;
          qkv_tables(tab, 64 * cf, wn, rope_lane);
#pragma unroll 1
          for (int qq = 0; qq < 4; ++qq) {
            uint32_t v16[16];
            tmem_ld16(tbase + 64 * cs + 16 * qq, v16);
            tmem_ld_wait();
            tmem_regs_ready(v16);
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const uint32_t bw =
                  p.bias ? __ldg(reinterpret_cast<const uint32_t*>(p.bias + nh + 64 * cs + 16 * qq + c)) : 0u;
              const float t0 = fmaf(alpha, __uint_as_float(v16[c]), bf16_bits_to_f32(bw & 0xFFFFu));
              const float t1 = fmaf(alpha, __uint_as_float(v16[c + 1]), bf16_bits_to_f32(bw >> 16));
              ss0 = fmaf(t0, t0, ss0);
              ss1 = fmaf(t1, t1, ss1);
            }
          }
          const float ss = (sf0 + sf1) + (ss0 + ss1);  // addition commutes: chunk 0 + chunk 1
          const float inv = rsqrtf(fmaf(ss, 1.0f / 128.0f, p.eps));
#pragma unroll 1
          for (int part = 0; part < 2; ++part) {
            if (lane == 0) bulk_wait_read<kSlots - 1>();
            __syncwarp();
            uint8_t* buf = sm.out[e][0];
            if (part == 0) {
              qkv_out32(buf, lane, ya, 0, inv, tab);
              qkv_tables(tab, 64 * cf + 32, wn, rope_lane);
              qkv_out32(buf, lane, yb, 4, inv, tab);
            } else {
#pragma unroll 1
              for (int hh = 0; hh < 2; ++hh) {
                qkv_tables(tab, 64 * cs + 32 * hh, wn, rope_lane);  // under the TMEM load
                uint32_t v[32];
                float t[32];
                tmem_ld32(tbase + 64 * cs + 32 * hh, v);
                tmem_ld_wait();
                tmem_regs_ready(v);
                layer_out32(t, v, alpha, p.bias, nh + 64 * cs + 32 * hh);
                qkv_out32(buf, lane, t, 4 * hh, inv, tab);
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 < p.M) tma_store_2d(&tm_y, buf, nh + 64 * (part == 0 ? cf : cs), row0);
              bulk_commit();
            }
          }
          continue;
        }
      }
      if constexpr (kEpi != kEpiQkv)
      for (int step = 0; step < nchunks; ++step) {
        // buffer 0's upper half drains from its top, everything else from the
        // bottom: the shared columns come first
        const int c = (b == 0 && h == 1) ? nchunks - 1 - step : step;
        uint8_t* buf = sm.out[e][step % kSlots];
        // this chunk's bias, the same for every lane (issued before the TMEM wait)
        float bv[64];
        const int nb = n0 + cols * c;
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
          uint32_t w = 0;
          if (p.bias && k < cols && nb + k < p.N) w = __ldg(reinterpret_cast<const uint32_t*>(p.bias + nb + k));
          bv[k] = bf16_bits_to_f32(w & 0xFFFFu);
          bv[k + 1] = bf16_bits_to_f32(w >> 16);
        }
        uint32_t v[32], v2[32];
        tmem_ld32(tbase + cols * c, v);
        if (!p.out_f32) tmem_ld32(tbase + cols * c + 32, v2);
        tmem_ld_wait();
        if (holds_overlap && step == overlap_chunks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(free_bar);
        }
        if (lane == 0) bulk_wait_read<kSlots - 1>();
        __syncwarp();
        if (p.out_f32) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float o0 = fmaf(alpha, __uint_as_float(v[4 * u]), bv[4 * u]);
            const float o1 = fmaf(alpha, __uint_as_float(v[4 * u + 1]), bv[4 * u + 1]);
            const float o2 = fmaf(alpha, __uint_as_float(v[4 * u + 2]), bv[4 * u + 2]);
            const float o3 = fmaf(alpha, __uint_as_float(v[4 * u + 3]), bv[4 * u + 3]);
            *reinterpret_cast<float4*>(buf + lane * 128 + ((u ^ (lane & 7)) * 16)) = make_float4(o0, o1, o2, o3);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float* bb = bv + 8 * u;
            uint32_t w4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int col = 8 * u + 2 * k;
              const uint32_t a0 = col < 32 ? v[col] : v2[col - 32];
              const uint32_t a1 = col + 1 < 32 ? v[col + 1] : v2[col + 1 - 32];
              float y0 = fmaf(alpha, __uint_as_float(a0), bb[2 * k]);
              float y1 = fmaf(alpha, __uint_as_float(a1), bb[2 * k + 1]);
              if constexpr (kEpi == kEpiGelu) {
                y0 = gelu_erf(y0);
                y1 = gelu_erf(y1);
              }
              w4[k] = f32_to_bf16_bits(y0) | (f32_to_bf16_bits(y1) << 16);
            }
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((u ^ (lane & 7)) * 16)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int cc = n0 + cols * c;
          if (row0 < p.M && cc < p.N) tma_store_2d(&tm_y, buf, cc, row0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  __syncwarp();  // the cluster barrier is .aligned: every warp reconverges first
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
  __syncwarp();
  cluster_sync();
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const GemmArgs& a, cudaStream_t s) {
  CUtensorMap tm_a, tm_b, tm_sfa, tm_sfb, tm_p, tm_l, tm_y;
  const uint64_t kb = (uint64_t)a.K / 2;
  const uint64_t katoms = (uint64_t)a.K / 64;
  const uint64_t rb_x = (uint64_t)(a.M + 127) / 128, rb_w = (uint64_t)(a.N + 127) / 128;
  bool ok = make_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.x_codes, kb, a.M, kb, 128, BM,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_tmap_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, kb, a.N, kb, 128, BN / 2,
                          CU_TENSOR_MAP_SWIZZLE_128B);
  // scale atoms: [row block][K atom][128 x 32-bit words]
  ok = ok && make_tmap_3d(&tm_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.x_scales, 128, katoms, rb_x, 512, katoms * 512,
                          128, 4, 1);
  ok = ok && make_tmap_3d(&tm_sfb, CU_TENSOR_MAP_DATA_TYPE_UINT32, a.w_scales, 128, katoms, rb_w, 512, katoms * 512,
                          128, 4, 2);
  if (a.r > 0) {
    // P [M, r] and lr_up [N, 2r] viewed as (8 columns, rows, column groups of 8):
    // one box lands in shared memory as [group][row][8], the layout the
    // kind::f16 MMA reads without swizzle
    ok = ok && make_tmap_3d(&tm_p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.P, 8, a.M, (uint64_t)a.r / 8,
                            (uint64_t)a.r * 2, 16, 8, BM, (uint32_t)a.r / 8);
    ok = ok && make_tmap_3d(&tm_l, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lr_up, 8, a.N, (uint64_t)a.r / 4,
                            (uint64_t)a.r * 4, 16, 8, BN / 2, (uint32_t)a.r / 4);
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
  p.tensor_scale = a.tensor_scale;
  p.bias = a.bias;
  p.M = a.M; p.N = a.N; p.K = a.K; p.r = a.r;
  p.tiles_m = (a.M + 255) / 256;
  p.tiles_n = (a.N + BN - 1) / BN;
  p.out_f32 = a.out == 1;
  p.err = a.err;
  p.wait_ns = a.wait_ns;
  p.qkv_heads = a.qkv_heads;
  p.norm_q = a.norm_q;
  p.norm_k = a.norm_k;
  p.eps = a.eps;
  p.rope = a.rope;

  const size_t smem = sizeof(Smem) + 1024;
  auto kern = p.qkv_heads > 0 ? gemm_nvfp4_kernel<kEpiQkv>
                              : (a.out == 3 ? gemm_nvfp4_kernel<kEpiGelu> : gemm_nvfp4_kernel<kEpiPlain>);
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n;
  const int pairs = a.num_sms / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm_a, tm_b, tm_sfa, tm_sfb, tm_p, tm_l, tm_y, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace svdq
