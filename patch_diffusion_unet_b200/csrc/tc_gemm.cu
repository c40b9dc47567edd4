// Tensor-core (tcgen05 / TMEM / TMA) GEMM for sm_100a, bf16 operands, fp32 accumulate.
// A pipeline stage carries two 64-wide K chunks (one TMA box of two chunks for the
// row-major operands, two 4-D boxes for the conv slab), halving TMA instructions and
// barrier hand-offs per FLOP.
//
// One kernel serves two contractions of the layer step:
//  * the displaced conv3x3 as an implicit GEMM (DistriConv2dPP, "DistriFusion源码探秘"
//    source walkthrough, Patch Parallelism section item 1): M = H*W output pixels,
//    N = Cout, K = 9*Cin.  The A tile of tap (r, s) is one TMA box of the haloed
//    per-patch slab [N][R+2][W][Cin] at (channel k0, column j0+s-1, slab row i0+r,
//    patch p).  The slab's halo rows hold the neighbour rows (stale on displaced
//    steps); the column padding is the TMA zero fill of out-of-range coordinates.
//  * the 1x1 projections to_q/to_k/to_v (one GEMM against the concatenated
//    [3C, C] weight, epilogue scattering into head-major Q/K/V) and to_out (+bias).
//
// Roles in a CTA of 192 threads: warp 0 issues TMA loads into a STAGES-deep ring,
// warp 1 issues tcgen05.mma from one elected thread into a 128 x BN fp32 TMEM
// accumulator, warps 2-5 drain TMEM (tcgen05.ld) through the epilogue.
// Every wait is bounded (see dfp_common.cuh).
#include <cstdio>

#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kStageBytes = 4 * 2048;   // the epilogue warps' transpose buffers

template <int BN> struct TmemCols { static constexpr uint32_t v = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256; };

struct TileInfo {
  int p, i0, j0, m0;  // conv: patch, patch-local first row, first column; plain: first row
};

__device__ __forceinline__ TileInfo tile_of(const TcGemmPlan& pl, int m_tile) {
  TileInfo t{};
  if (pl.conv) {
    const int per_patch = (pl.R / pl.rows_tile) * pl.tiles_per_row;
    const int lp = m_tile / per_patch;
    t.p = pl.p0 + lp;
    const int rem = m_tile - lp * per_patch;
    const int it = rem / pl.tiles_per_row;
    const int jt = rem - it * pl.tiles_per_row;
    t.i0 = it * pl.rows_tile;
    t.j0 = jt * pl.cols_tile;
  } else {
    t.m0 = pl.m_base + m_tile * kBM;
  }
  return t;
}

// Output row of this thread's accumulator lane (row) in tile `tile`, or -1 for none.
__device__ __forceinline__ long long out_row(const TcGemmPlan& plan, const Epilogue& epi, const TileInfo& tile,
                                             int row, bool valid_tile) {
  long long gm = -1;
  if (plan.conv) {
    const int rr = row / plan.cols_tile, jj = row - rr * plan.cols_tile;
    if (rr < plan.rows_tile && tile.j0 + jj < plan.W)
      gm = ((long long)tile.p * plan.R + tile.i0 + rr) * plan.W + tile.j0 + jj;
  } else if (tile.m0 + row < plan.M) {
    gm = tile.m0 + row;
  }
  if (!valid_tile) gm = -1;
  if (epi.subsample && gm >= 0) {
    // a stride-2 conv as the stride-1 conv sampled at even rows and columns: keep those
    // pixels, stored at their place in the half-resolution map
    const long long prow = gm / plan.W, col = gm - prow * plan.W;
    gm = ((prow | col) & 1) ? -1 : (prow >> 1) * (plan.W >> 1) + (col >> 1);
  }
  return gm;
}

// The residual of this thread's output row, read before the accumulator is ready (the
// loads overlap the tile's MMAs instead of stalling the epilogue chunk by chunk).
template <int BN>
__device__ __forceinline__ void prefetch_residual(const Epilogue& epi, long long gm, int n0, int N,
                                                  uint4 (&res)[BN / 8]) {
  if (epi.kind != 0 || !epi.residual || gm < 0) return;
  const uint4* r4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(epi.residual) + gm * epi.ldo + n0);
#pragma unroll
  for (int i = 0; i < BN / 8; ++i)
    if (n0 + 8 * i < N) res[i] = __ldg(r4 + i);
}

// Epilogue of one tile: drain the 128 x BN accumulator at TMEM address taddr (this warp's
// lanes) and store row gm (-1: nothing to store; the TMEM reads still run warp-wide).
// stage: this warp's 2 KB of shared memory.  A warp's 32 x 32 chunk goes through it so that
// each store instruction writes 8 whole 64-byte row segments rather than 32 scattered 16-byte
// pieces (the rows of a warp are 32 output rows, each lane holds one).
template <int BN>
__device__ __forceinline__ void epilogue_tile(const TcGemmPlan& plan, const Epilogue& epi, long long gm, int n0,
                                              uint32_t taddr, const uint4 (&res)[BN / 8], uint4* stage) {
  const int lane = threadIdx.x & 31;
  if (BN == 128 && epi.kind == 2) {
    // GEGLU: columns [0, 64) are values, [64, 128) the gates of the same features
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t rv[32], rg[32];
      tmem_ld32(taddr + c * 32, rv);
      tmem_ld32(taddr + 64 + c * 32, rg);
      tmem_wait_ld();
      if (gm < 0) continue;
      const int nv = n0 + c * 32, ng = n0 + 64 + c * 32;
      float w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float av = __uint_as_float(rv[i]) + __ldg(epi.bias + nv + i);
        const float g = __uint_as_float(rg[i]) + __ldg(epi.bias + ng + i);
        w[i] = av * (0.5f * g * (1.f + erff(g * 0.70710678118654752f)));
      }
      uint4* d4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(epi.out) + gm * epi.ldo + n0 / 2 + c * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = w[i * 8 + e];
        d4[i] = pack16(w8);
      }
    }
    return;
  }
  // store the 32 columns of chunk c (registers r, already loaded); warp-wide
  auto store_chunk = [&](int c, const uint32_t (&r)[32]) {
    const int n = n0 + c * 32;
    if (n >= plan.N) return;   // warp-uniform
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    __nv_bfloat16* dst;
    if (epi.kind == 0) {
      if (epi.bias) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += __ldg(epi.bias + n + i);
      }
      if (epi.residual) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float rr[8];
          unpack16(res[c * 4 + i], rr);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[i * 8 + e] += rr[e];
        }
      }
      if (epi.n_store && n + 32 > epi.n_store) {
        // only the first n_store columns exist in the output (a padded narrow layer)
        if (gm < 0) return;
        dst = static_cast<__nv_bfloat16*>(epi.out) + gm * epi.ldo + n;
        for (int i = 0; i < 32 && n + i < epi.n_store; ++i) dst[i] = __float2bfloat16_rn(v[i]);
        return;
      }
    }
    // the row through shared memory: 16-byte pieces swizzled by row (conflict-free both ways)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float w8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w8[e] = v[i * 8 + e];
      stage[lane * 4 + (i ^ ((lane >> 1) & 3))] = pack16(w8);
    }
    __syncwarp();
    // lane 4 rr + ch stores piece ch of rows rr, rr + 8, rr + 16, rr + 24
    const int ch = lane & 3;
    long long head_base = 0;
    void* base = epi.out;
    if (epi.kind != 0) {
      const int which = n / epi.C, cc = n - which * epi.C;
      base = which == 0 ? epi.q : (which == 1 ? epi.k : epi.v);
      head_base = (long long)(cc >> 6) * epi.L * 64 + (cc & 63);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rr = k * 8 + (lane >> 2);
      const long long g = __shfl_sync(0xffffffffu, gm, rr);
      const uint4 piece = stage[rr * 4 + (ch ^ ((rr >> 1) & 3))];
      if (g >= 0) {
        __nv_bfloat16* d = static_cast<__nv_bfloat16*>(base) +
                           (epi.kind == 0 ? g * epi.ldo + n : head_base + g * 64) + ch * 8;
        *reinterpret_cast<uint4*>(d) = piece;
      }
    }
    __syncwarp();   // the stage is read before the next chunk rewrites it
  };
  // the next chunk's TMEM load is in flight while this one is converted and stored
  uint32_t r[2][32];
  tmem_ld32(taddr, r[0]);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    if (c + 1 < BN / 32) tmem_ld32(taddr + (c + 1) * 32, r[(c + 1) & 1]);
    store_chunk(c, r[c & 1]);
    tmem_wait_ld();
  }
}

// Persistent: CTA b takes tiles b, b + gridDim.x, ...  Two TMEM accumulators let the
// epilogue of tile i overlap the main loop of tile i + 1; the TMA ring runs on across
// tiles.  Tile t = (m_tile = t / n_tiles_n, n_tile = t % n_tiles_n): the CTAs in flight
// share A tiles (all N tiles of an M tile are neighbours) and all share the weights.
template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               const TcGemmPlan plan, const Epilogue epi, int* err) {
  // A stage holds two 64-wide K chunks: [chunk][rows][64] for A (16 KB per chunk) and for B
  constexpr uint32_t kAChunk = kBM * kBK * 2;
  constexpr uint32_t kBChunk = BN * kBK * 2;
  constexpr uint32_t kABytes = 2 * kAChunk;
  constexpr uint32_t kBBytes = 2 * kBChunk;
  constexpr uint32_t kCols = TmemCols<BN>::v;            // one accumulator
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  uint4* sStage = reinterpret_cast<uint4*>(sB + STAGES * kBBytes);   // 4 epilogue warps x 2 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * kBBytes + kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;                // [2]
  uint64_t* acc_empty = bars + 2 * STAGES + 2;           // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles_n = plan.N / BN;
  const int n_tiles = plan.m_tiles * n_tiles_n;
  // K stages of two chunks; the conv pairs chunks within a tap (an odd last chunk of a
  // tap reads zeros past the channel count: A is zero there, so B's chunk does not matter)
  const int cpt = plan.conv ? plan.Cin / kBK : 0;                 // chunks per tap
  const int ppt = (cpt + 1) / 2;                                  // chunk pairs per tap
  const int num_kb = plan.conv ? 9 * ppt : (plan.K / kBK + 1) / 2;
  const uint32_t a_box_bytes =
      plan.conv ? (uint32_t)(2 * plan.rows_tile * plan.cols_tile * kBK * 2) : kABytes;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) { mbar_init(smem_u32(&full[s]), 1); mbar_init(smem_u32(&empty[s]), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&acc_full[i]), 1); mbar_init(smem_u32(&acc_empty[i]), 128); }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  // the set-up above touches no global memory: overlap it with the prior kernel's tail
  wait_prior_grid();
  allow_next_grid();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp walks the loop (coordinates are warp-uniform); one lane issues.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
    }
    int kg = 0;   // k-stages issued so far (ring position)
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
      const TileInfo tile = tile_of(plan, t / n_tiles_n);
      const int n0 = (t % n_tiles_n) * BN;
      for (int kb = 0; kb < num_kb; ++kb, ++kg) {
        const int s = kg % STAGES, round = kg / STAGES;
        if (round > 0 && !mbar_wait_warp(smem_u32(&empty[s]), (round - 1) & 1, err, kErrWaitStageFree)) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, s_abort != 0)) { ok = false; break; }
        const uint32_t fb = smem_u32(&full[s]);
        if (leader) {
          mbar_arrive_expect_tx(fb, a_box_bytes + kBBytes);
          if (plan.conv) {
            const int tap = kb / ppt, kc = 2 * (kb - tap * ppt);
            const int r = tap / 3, sx = tap - 3 * (tap / 3);
            const uint32_t da = smem_u32(sA + s * kABytes);
            tma_load_4d(da, &mapA, fb, kc * kBK, tile.j0 + sx - 1, tile.i0 + r, tile.p);
            tma_load_4d(da + kAChunk, &mapA, fb, (kc + 1) * kBK, tile.j0 + sx - 1, tile.i0 + r, tile.p);
            tma_load_3d(smem_u32(sB + s * kBBytes), &mapB, fb, 0, n0, tap * cpt + kc);
          } else {
            tma_load_3d(smem_u32(sA + s * kABytes), &mapA, fb, 0, tile.m0, 2 * kb);
            tma_load_3d(smem_u32(sB + s * kBBytes), &mapB, fb, 0, n0, 2 * kb);
          }
        }
        __syncwarp();
      }
    }
    if (!ok || __any_sync(0xffffffffu, s_abort != 0)) {
      if (leader) s_abort = 1;
      // let the copies already in flight land before the CTA can exit
      for (int k = (kg > STAGES ? kg - STAGES : 0); k < kg; ++k)
        mbar_wait(smem_u32(&full[k % STAGES]), (k / STAGES) & 1, err, kErrWaitTmaFull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the loop so the descriptors stay warp-uniform; the
    // elected lane issues the MMAs and the commits (which track that lane's MMAs).
    const bool leader = elect_one();
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
    const uint64_t ad0 = sw128_kmajor_desc(smem_u32(sA));
    const uint64_t bd0 = sw128_kmajor_desc(smem_u32(sB));
    bool ok = true;
    int kg = 0, ti = 0;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++ti) {
      const int buf = ti & 1, use = ti >> 1;
      if (use > 0 && !mbar_wait_warp(smem_u32(&acc_empty[buf]), (use - 1) & 1, err, kErrWaitAccum)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d = tmem_d + buf * kCols;
      for (int kb = 0; kb < num_kb; ++kb, ++kg) {
        const int s = kg % STAGES, round = kg / STAGES;
        if (!mbar_wait_warp(smem_u32(&full[s]), round & 1, err, kErrWaitTmaFull)) { ok = false; break; }
        tc_fence_after();
        // operands: per-stage bases, compile-time offsets per K slice
        const uint64_t ad = ad0 + (uint64_t)s * (kABytes >> 4);
        const uint64_t bd = bd0 + (uint64_t)s * (kBBytes >> 4);
        const uint64_t ad1 = ad + (kAChunk >> 4), bd1 = bd + (kBChunk >> 4);
        if (leader) {
          umma_f16_ss(d, ad, bd, idesc, kb > 0);
#pragma unroll
          for (int kk = 1; kk < kBK / 16; ++kk) umma_f16_ss(d, ad + 2 * kk, bd + 2 * kk, idesc, 1);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) umma_f16_ss(d, ad1 + 2 * kk, bd1 + 2 * kk, idesc, 1);
          umma_commit(smem_u32(&empty[s]));
        }
        __syncwarp();
      }
      if (ok && leader) umma_commit(smem_u32(&acc_full[buf]));
      __syncwarp();
    }
    if (!ok && leader) s_abort = 1;
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    int ti = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++ti) {
      const int buf = ti & 1, use = ti >> 1;
      const TileInfo tile = tile_of(plan, t / n_tiles_n);
      const int n0 = (t % n_tiles_n) * BN;
      const long long gm = out_row(plan, epi, tile, row, true);
      uint4 res[BN / 8];
      prefetch_residual<BN>(epi, gm, n0, plan.N, res);
      const bool ready = mbar_wait(smem_u32(&acc_full[buf]), use & 1, err, kErrWaitAccum);
      tc_fence_after();
      epilogue_tile<BN>(plan, epi, ready && !s_abort ? gm : -1, n0,
                        tmem_d + buf * kCols + ((uint32_t)(sub * 32) << 16), res, sStage + sub * 128);
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[buf]));
      if (!ready) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, 2 * kCols);
  }
}

// CTA-pair variant (cluster of 2, cta_group::2): the pair computes 256 x BN tiles.  Each
// CTA loads its own 128 rows of A and half of B's BN rows into its own shared memory
// (plain TMA loads whose byte counts land on the leader's barrier), the leader's MMA warp
// issues M = 256 MMAs that read both CTAs' tiles, and each CTA's epilogue drains its own
// 128 x BN accumulator.  Per SM that is 128 + BN/2 operand rows per k-stage instead of
// 128 + BN: the loads, not the tensor core, bound the single-CTA kernel.
template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                    const TcGemmPlan plan, const Epilogue epi, int* err) {
  constexpr int BNH = BN / 2;                             // B rows held by this CTA
  constexpr uint32_t kAChunk = kBM * kBK * 2;
  constexpr uint32_t kBChunk = BNH * kBK * 2;
  constexpr uint32_t kABytes = 2 * kAChunk;
  constexpr uint32_t kBBytes = 2 * kBChunk;
  constexpr uint32_t kCols = TmemCols<BN>::v;            // one accumulator
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  uint4* sStage = reinterpret_cast<uint4*>(sB + STAGES * kBBytes);   // 4 epilogue warps x 2 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * kBBytes + kStageBytes);
  uint64_t* full = bars;                                 // leader's: both CTAs' loads
  uint64_t* empty = bars + STAGES;                       // each CTA's, from the leader's commits
  uint64_t* acc_full = bars + 2 * STAGES;                // [2] each CTA's
  uint64_t* acc_empty = bars + 2 * STAGES + 2;           // [2] leader's: one arrival per CTA
  uint64_t* exit_bar = bars + 2 * STAGES + 4;            // both CTAs arrive on both
  uint64_t* drain = bars + 2 * STAGES + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 6);
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_tiles_n = plan.N / BN;
  const int m_pairs = (plan.m_tiles + 1) / 2;
  const int n_tiles = m_pairs * n_tiles_n;
  const int cpt = plan.conv ? plan.Cin / kBK : 0;
  const int ppt = (cpt + 1) / 2;
  const int num_kb = plan.conv ? 9 * ppt : (plan.K / kBK + 1) / 2;
  const uint32_t a_box_bytes =
      plan.conv ? (uint32_t)(2 * plan.rows_tile * plan.cols_tile * kBK * 2) : kABytes;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) { mbar_init(smem_u32(&full[s]), 1); mbar_init(smem_u32(&empty[s]), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&acc_full[i]), 1); mbar_init(smem_u32(&acc_empty[i]), 2); }
    mbar_init(smem_u32(exit_bar), 2);
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 2 * kCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers exist before either touches the other's
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  wait_prior_grid();           // the set-up above touches no global memory
  allow_next_grid();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    const bool issuer = elect_one();
    if (issuer) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
    }
    int kg = 0;
    bool ok = true;
    for (int t = pair; ok && t < n_tiles; t += n_pairs) {
      const TileInfo tile = tile_of(plan, 2 * (t / n_tiles_n) + (int)rank);   // past the end: TMA zero fill
      const int n0 = (t % n_tiles_n) * BN + (int)rank * BNH;
      for (int kb = 0; kb < num_kb; ++kb, ++kg) {
        const int s = kg % STAGES, round = kg / STAGES;
        if (round > 0 && !__all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(&empty[s]), (round - 1) & 1, err,
                                                                   kErrWaitStageFree))) {
          ok = false;
          break;
        }
        if (__any_sync(0xffffffffu, s_abort != 0)) { ok = false; break; }
        const uint32_t fb = map_to_rank(smem_u32(&full[s]), 0);
        if (issuer) {
          if (lead) mbar_arrive_expect_tx(smem_u32(&full[s]), 2 * (a_box_bytes + kBBytes));
          if (plan.conv) {
            const int tap = kb / ppt, kc = 2 * (kb - tap * ppt);
            const int r = tap / 3, sx = tap - 3 * (tap / 3);
            const uint32_t da = smem_u32(sA + s * kABytes);
            tma_load_4d_pair(da, &mapA, fb, kc * kBK, tile.j0 + sx - 1, tile.i0 + r, tile.p);
            tma_load_4d_pair(da + kAChunk, &mapA, fb, (kc + 1) * kBK, tile.j0 + sx - 1, tile.i0 + r, tile.p);
            tma_load_3d_pair(smem_u32(sB + s * kBBytes), &mapB, fb, 0, n0, tap * cpt + kc);
          } else {
            tma_load_3d_pair(smem_u32(sA + s * kABytes), &mapA, fb, 0, tile.m0, 2 * kb);
            tma_load_3d_pair(smem_u32(sB + s * kBBytes), &mapB, fb, 0, n0, 2 * kb);
          }
        }
        __syncwarp();
      }
    }
    if (!ok || __any_sync(0xffffffffu, s_abort != 0)) {
      if (issuer) s_abort = 1;
      // the leader's barriers count both CTAs' copies: let those in flight land
      if (lead)
        for (int k = (kg > STAGES ? kg - STAGES : 0); k < kg; ++k)
          mbar_wait_cluster(smem_u32(&full[k % STAGES]), (k / STAGES) & 1, err, kErrWaitTmaFull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (lead) {
      const bool issuer = elect_one();
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, BN, false, false);
      const uint64_t ad0 = sw128_kmajor_desc(smem_u32(sA));
      const uint64_t bd0 = sw128_kmajor_desc(smem_u32(sB));
      bool ok = true;
      int kg = 0, ti = 0;
      for (int t = pair; ok && t < n_tiles; t += n_pairs, ++ti) {
        const int buf = ti & 1, use = ti >> 1;
        if (use > 0 && !__all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(&acc_empty[buf]), (use - 1) & 1, err,
                                                                   kErrWaitAccum))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_d + buf * kCols;
        for (int kb = 0; kb < num_kb; ++kb, ++kg) {
          const int s = kg % STAGES, round = kg / STAGES;
          if (!__all_sync(0xffffffffu, mbar_wait_cluster(smem_u32(&full[s]), round & 1, err, kErrWaitTmaFull))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = ad0 + (uint64_t)s * (kABytes >> 4);
          const uint64_t bd = bd0 + (uint64_t)s * (kBBytes >> 4);
          const uint64_t ad1 = ad + (kAChunk >> 4), bd1 = bd + (kBChunk >> 4);
          if (issuer) {
            umma_f16_ss_pair(d, ad, bd, idesc, kb > 0);
#pragma unroll
            for (int kk = 1; kk < kBK / 16; ++kk) umma_f16_ss_pair(d, ad + 2 * kk, bd + 2 * kk, idesc, 1);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) umma_f16_ss_pair(d, ad1 + 2 * kk, bd1 + 2 * kk, idesc, 1);
            umma_commit_pair(smem_u32(&empty[s]), 0x3);   // the stage is free in both CTAs
          }
          __syncwarp();
        }
        if (ok && issuer) umma_commit_pair(smem_u32(&acc_full[buf]), 0x3);
        __syncwarp();
      }
      if (!ok && issuer) s_abort = 1;
      // every MMA of this CTA pair completes before TMEM can be released
      if (issuer) umma_commit_pair(smem_u32(drain), 0x1);
      __syncwarp();
      mbar_wait(smem_u32(drain), 0, err, kErrWaitAccum);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    int ti = 0;
    for (int t = pair; t < n_tiles; t += n_pairs, ++ti) {
      const int buf = ti & 1, use = ti >> 1;
      const int m_tile = 2 * (t / n_tiles_n) + (int)rank;
      const TileInfo tile = tile_of(plan, m_tile);
      const int n0 = (t % n_tiles_n) * BN;
      const long long gm = out_row(plan, epi, tile, row, m_tile < plan.m_tiles);
      uint4 res[BN / 8];
      prefetch_residual<BN>(epi, gm, n0, plan.N, res);
      const bool ready = mbar_wait_cluster(smem_u32(&acc_full[buf]), use & 1, err, kErrWaitAccum);
      tc_fence_after();
      epilogue_tile<BN>(plan, epi, ready && !s_abort ? gm : -1, n0,
                        tmem_d + buf * kCols + ((uint32_t)(sub * 32) << 16), res, sStage + sub * 128);
      tc_fence_before();
      // the four epilogue warps of this CTA are done with the accumulator; they also agree
      // on giving up (a failed wait anywhere ends the loop for all of them)
      const bool give_up = named_bar_red_or(1, 128, !ready);
      if (threadIdx.x == 64) {
        if (lead) mbar_arrive(smem_u32(&acc_empty[buf]));
        else mbar_arrive_remote(map_to_rank(smem_u32(&acc_empty[buf]), 0));
      }
      if (give_up) break;
    }
  }

  // ---- exit: neither CTA leaves while the other may still reach into its shared memory
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive(smem_u32(exit_bar));
    mbar_arrive_remote(map_to_rank(smem_u32(exit_bar), rank ^ 1u));
    mbar_wait_cluster(smem_u32(exit_bar), 0, err, kErrWaitAccum);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, 2 * kCols);
  }
}

template <int BN, int STAGES>
cudaError_t launch_pair(const TcGemmPlan& plan, const CUtensorMap& mA, const CUtensorMap& mB,
                        const Epilogue& epi, int* err, cudaStream_t s) {
  const size_t smem = 1024 + (size_t)STAGES * 2 * (kBM * kBK * 2 + (BN / 2) * kBK * 2) + kStageBytes +
                      (2 * STAGES + 8) * 8 + 64;
  auto kern = tc_gemm_pair_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_tiles = ((plan.m_tiles + 1) / 2) * (plan.N / BN);
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;   // the occupancy query sees the cluster shape only
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // persistent: no more pairs than can be resident at once (a GPC with an odd number of
  // free SMs leaves one idle), so no pair waits for a second wave
  static int max_pairs = 0;
  if (!max_pairs) {
    cfg.gridDim = dim3(2 * (plan.sms / 2));
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess) return e;
    max_pairs = n > 0 ? n : 1;
  }
  const int pairs = n_tiles < max_pairs ? n_tiles : max_pairs;
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = plan.pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, mA, mB, plan, epi, err);
}

template <int BN, int STAGES>
cudaError_t launch_bn(const TcGemmPlan& plan, const CUtensorMap& mA, const CUtensorMap& mB,
                      const Epilogue& epi, int* err, cudaStream_t s) {
  const size_t smem = 1024 + (size_t)STAGES * 2 * (kBM * kBK * 2 + BN * kBK * 2) + kStageBytes +
                      (2 * STAGES + 6) * 8 + 64;
  auto kern = tc_gemm_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_tiles = plan.m_tiles * (plan.N / BN);
  const int grid = n_tiles < plan.sms ? n_tiles : plan.sms;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = plan.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, mA, mB, plan, epi, err);
}

}  // namespace

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

int gemm_m_tiles_plain(int M) { return (M + kBM - 1) / kBM; }

GemmChoice choose_gemm(int N, int m_tiles, int k_stages, int force_bn) {
  const int sms = sm_count();
  GemmChoice best{0, 0};
  long best_cost = 0;
  for (int pair = 1; pair >= 0; --pair) {
    for (int bn : {160, 128, 64}) {
      if (N % bn || (force_bn && bn != force_bn)) continue;
      if (pair && (bn == 64 || m_tiles < 2)) continue;
      if (pair) {
        // the pair's set-up (cluster sync, remote arrivals, exit handshake) and its
        // longer pipeline fill pay off with long tiles (K >= 1024) or many of them (measured on the
        // 64x64x640, 240x240x640 and SDXL-stage projections)
        const long ptiles = (long)((m_tiles + 1) / 2) * (N / bn);
        const long per_pair = (ptiles + sms / 2 - 1) / (sms / 2);
        if (k_stages < 8 && per_pair * k_stages < 64) continue;
      }
      // per SM and k-stage the loads move 128 + bn (single CTA) or 128 + bn/2 (CTA pair)
      // operand rows; that, times the waves, is the time
      const long units = pair ? (long)((m_tiles + 1) / 2) * (N / bn) : (long)m_tiles * (N / bn);
      const long slots = pair ? sms / 2 : sms;
      const long cost = ((units + slots - 1) / slots) * (pair ? 128 + bn / 2 : 128 + bn);
      if (!best.bn || cost < best_cost) { best = GemmChoice{bn, pair}; best_cost = cost; }
    }
  }
  if (!best.bn) best = GemmChoice{64, 0};
  return best;
}

cudaError_t launch_tc_gemm(const TcGemmPlan& plan_in, const CUtensorMap& mapA, const CUtensorMap& mapB,
                           const Epilogue& epi, int* err, cudaStream_t s) {
  TcGemmPlan plan = plan_in;
  // conv: tiles of patches [p0, p0 + P); plain: rows [m_base, M)
  plan.m_tiles = plan.conv ? plan.P * (plan.R / plan.rows_tile) * plan.tiles_per_row
                           : (plan.M - plan.m_base + kBM - 1) / kBM;
  if (plan.m_tiles <= 0) return cudaErrorInvalidValue;
  plan.sms = sm_count();
  // as many two-chunk stages as fit in ~220 KB of shared memory
  if (plan.pair) {
    switch (plan.bn) {
      case 128: return launch_pair<128, 4>(plan, mapA, mapB, epi, err, s);
      case 160: return launch_pair<160, 4>(plan, mapA, mapB, epi, err, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (plan.bn) {
    case 128: return launch_bn<128, 3>(plan, mapA, mapB, epi, err, s);
    case 160: return launch_bn<160, 3>(plan, mapA, mapB, epi, err, s);
    case 64: return launch_bn<64, 4>(plan, mapA, mapB, epi, err, s);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- TMA descriptors
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}
bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

bool encode_gemm_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
  // view [K/64 chunks][rows][64] of a row-major [rows][K] bf16 matrix; one box = two chunks
  const cuuint64_t dims[3] = {64, rows, (K + 63) / 64};
  const cuuint64_t strides[2] = {K * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, 2};
  return encode(m, base, 3, dims, strides, box);
}

bool encode_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t outer_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {outer_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  return encode(m, base, 2, dims, strides, box);
}
bool encode_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1, uint32_t b2) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  return encode(m, base, 3, dims, strides, box);
}
bool encode_tmap_5d(CUtensorMap* m, const void* base, const uint64_t dims[5],
                    const uint64_t strides_bytes[4], const uint32_t box[5]) {
  const cuuint64_t d[5] = {dims[0], dims[1], dims[2], dims[3], dims[4]};
  const cuuint64_t st[4] = {strides_bytes[0], strides_bytes[1], strides_bytes[2], strides_bytes[3]};
  const cuuint32_t b[5] = {box[0], box[1], box[2], box[3], box[4]};
  return encode(m, base, 5, d, st, b);
}
bool encode_tmap_4d(CUtensorMap* m, const void* base, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4]) {
  const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t st[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
  return encode(m, base, 4, d, st, b);
}

}  // namespace dfp
