// Displaced self-attention on tcgen05 / TMEM / TMA (sm_100a), bf16 operands, fp32
// softmax statistics and accumulation, head width 64.
//
// DistriSelfAttentionPP ("DistriFusion源码探秘" source walkthrough, Patch
// Parallelism section item 2): the queries of patch p attend to all L tokens; the
// K/V of its own rows are this step's, those of every other patch come from the
// previous step's cache (project README, Overview (c): activations of the
// previous step are reused).  The KV loop walks a list of segments:
//   sync       [0, L) fresh
//   displaced  own patch fresh, then [0, p*Lp) stale, then [(p+1)*Lp, L) stale
//   naive      own patch fresh only (the naive-patch baseline, README Overview (b))
// Segment ends need not be multiples of the 128-key tile: columns past a
// segment's end are masked.
//
// CTA layout (640 threads, five warpgroups): two softmax groups of 8 warps, each
// owning one 128-query tile.  Warps w and w+4 of a group read the same 32 TMEM
// lanes (query rows); the first takes key columns 0-63, the second 64-127, and
// they exchange their partial row maxima through shared memory -- at head width
// 64 the softmax work per tile is large next to the MMAs, and two threads per
// row double the latency hiding.  In the fifth warpgroup warp 16 issues TMA
// (both Q tiles once, K/V through 3-stage rings shared by the groups) and warp
// 17 issues the MMAs from one thread.  Per KV tile j and group g:
//   S_g = Q_g K_j^T            tcgen05.mma, A and B from shared memory, D in TMEM
//   P_g = exp2(S_g * c - m_g)  softmax threads, written back over S_g in TMEM as
//                              bf16 pairs (byte-permute truncation)
//   O_g += P_g [V_j | 1]       tcgen05.mma with A = P from TMEM; the ones block
//                              appended to V makes the tensor core produce the row
//                              sums of the same truncated P, so the truncation
//                              cancels in O / l
// The groups ping-pong: the MMAs of one group run while the other computes its
// softmax.  The running maximum is lazy: O and l are rescaled (in TMEM) only
// when a row's maximum grows by more than 2^8.  Part of the exponentials run as
// a polynomial on the FMA pipe (range reduction to 2^j * 2^f, |f| <= 1/2, with a
// degree-3 polynomial for 2^f fitted by weighted least squares on Chebyshev
// nodes, max relative error 7.5e-5) to offload the MUFU unit.
//
// Split-KV: with few query tiles per SM (small maps) the KV tile list of a Q-tile
// pair is split over `splits` CTAs; each writes its unnormalised O, m and l to a
// scratch buffer and the last CTA of the pair (arrival counter) merges them in
// split order, so the result is deterministic.
#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kThreads = 640;
constexpr int kSoftmaxThreads = 512;
constexpr int kWarpTma = 16, kWarpMma = 17;
constexpr int kTile = 128;
constexpr uint32_t kTileBytes = 128 * 64 * 2;   // one 128 x 64 bf16 tile
constexpr int kStages = 3;
constexpr int kOCols = 80;                      // 64 outputs + 16 row-sum columns
constexpr uint32_t kTmemCols = 512;             // S/P: [128g, 128g+128), O: [256+128g, +80)
constexpr float kRescale = 8.f;                 // lazy rescale threshold (log2 units)
constexpr int kPolyPer8 = 3;                    // of every 8 columns, this many use the polynomial

struct Segs {
  int n;
  int stale[3], start[3], len[3], tiles[3];
  int total;
};

__device__ __forceinline__ Segs make_segs(int mode, int p, int Lp, int L, int kv_len) {
  Segs s{};
  auto add = [&](int st, int b, int len) {
    if (len <= 0) return;
    s.stale[s.n] = st; s.start[s.n] = b; s.len[s.n] = len;
    s.tiles[s.n] = (len + kTile - 1) / kTile;
    s.total += s.tiles[s.n];
    ++s.n;
  };
  if (mode == kAttnSync) {
    add(0, 0, L);
  } else if (mode == kAttnCross) {
    add(0, 0, kv_len);        // the fixed context: same for every patch, never stale
  } else {
    add(0, p * Lp, Lp);
    if (mode == kAttnDisplaced) {
      add(1, 0, p * Lp);
      add(1, (p + 1) * Lp, L - (p + 1) * Lp);
    }
  }
  return s;
}

// tile j of the segment list -> (stale?, first key row, valid keys)
__device__ __forceinline__ void seg_tile(const Segs& s, int j, int& stale, int& row, int& valid) {
  int k = 0;
  while (k < s.n - 1 && j >= s.tiles[k]) { j -= s.tiles[k]; ++k; }
  stale = s.stale[k];
  row = s.start[k] + j * kTile;
  valid = min(kTile, s.len[k] - j * kTile);
}

__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- packed fp32x2 arithmetic (two lanes per 64-bit register pair)
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x for a pair on the FMA pipe, returned as a truncated bf16 pair (lo = first
// lane): x = j + f with j = rint(x) by magic-constant rounding (1.5 * 2^23 puts j
// in the low mantissa bits), 2^f by a degree-3 polynomial, 2^j added into the
// exponent field.  x is clamped to >= -125 so the exponent cannot wrap.
__device__ __forceinline__ uint32_t ex2_poly_pair_bf16(uint64_t x2) {
  float x0, x1;
  f2_split(x2, x0, x1);
  const uint64_t x = f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = add2(x, f2(12582912.f, 12582912.f));
  const uint64_t j = add2(t, f2(-12582912.f, -12582912.f));
  const uint64_t f = fma2(j, f2(-1.f, -1.f), x);
  uint64_t p = fma2(f2(0.0551716648f, 0.0551716648f), f, f2(0.242611125f, 0.242611125f));
  p = fma2(p, f, f2(0.693260968f, 0.693260968f));
  p = fma2(p, f, f2(0.999928057f, 0.999928057f));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  const uint32_t r0 = __float_as_uint(p0) + (__float_as_uint(t0) << 23);
  const uint32_t r1 = __float_as_uint(p1) + (__float_as_uint(t1) << 23);
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(r0), "r"(r1));
  return r;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// upper halves of two fp32 words -> one bf16 pair (lo = a, hi = b): truncation
__device__ __forceinline__ uint32_t pack_trunc(float a, float b) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(__float_as_uint(a)), "r"(__float_as_uint(b)));
  return r;
}

__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Named barrier that also ORs a predicate over the participating threads: every
// thread leaves with the same answer, so a group can give up collectively.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(n) : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
tc_attention_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mkf,
                    const __grid_constant__ CUtensorMap mvf, const __grid_constant__ CUtensorMap mks,
                    const __grid_constant__ CUtensorMap mvs, const TcAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                          // 2 x 16 KB
  uint8_t* sK = sQ + 2 * kTileBytes;           // kStages x 16 KB
  uint8_t* sV = sK + kStages * kTileBytes;     // kStages x 16 KB
  uint8_t* sOnes = sV + kStages * kTileBytes;  // 16 KB of bf16 1.0 (the row-sum columns of B)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOnes + kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* v_full = k_empty + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_full = v_empty + kStages;        // [2]
  uint64_t* p_full = s_full + 2;               // [2]
  uint64_t* o_done = p_full + 2;               // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 2);
  __shared__ volatile int s_abort;
  __shared__ int s_last;
  __shared__ Segs s_segs;
  __shared__ float s_rowmax[2][2][2][128];   // [tile parity][group][half][row]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int splits = a.splits;
  const int split = blockIdx.x % splits, pair = blockIdx.x / splits;
  const int p = blockIdx.y, head = blockIdx.z;
  const int qt0 = 2 * pair;
  const bool activeB = qt0 + 1 < a.n_qtiles;
  const Segs& segs = s_segs;   // the KV segment list lives in shared memory (registers are precious)
  int* err = a.err;

  if (threadIdx.x == 0) {
    s_segs = make_segs(a.mode, p, a.Lp, a.L, a.kv_len);
    s_abort = 0;
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1); mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1); mbar_init(smem_u32(&v_empty[i]), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(smem_u32(&s_full[g]), 1);
      mbar_init(smem_u32(&p_full[g]), 256);
      mbar_init(smem_u32(&o_done[g]), 1);
    }
    fence_mbar_init();
  }
  {
    uint4* ones = reinterpret_cast<uint4*>(sOnes);
    for (int i = threadIdx.x; i < (int)(kTileBytes / 16); i += kThreads)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int j0 = split * segs.total / splits;
  const int nt = (split + 1) * segs.total / splits - j0;

  if (warp >= kWarpTma) {
   if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mq);
      const int qrow = p * a.Lp + qt0 * kTile;
      mbar_arrive_expect_tx(smem_u32(q_full), activeB ? 2 * kTileBytes : kTileBytes);
      tma_load_3d(smem_u32(sQ), &mq, smem_u32(q_full), 0, qrow, head);
      if (activeB) tma_load_3d(smem_u32(sQ + kTileBytes), &mq, smem_u32(q_full), 0, qrow + kTile, head);
      int issued = 0;
      for (int jj = 0; jj < nt; ++jj) {
        const int s = jj % kStages, round = jj / kStages;
        int stale, row, valid;
        seg_tile(segs, j0 + jj, stale, row, valid);
        if (round > 0 && !mbar_wait(smem_u32(&k_empty[s]), (round - 1) & 1, err, kErrWaitStageFree)) { s_abort = 1; break; }
        mbar_arrive_expect_tx(smem_u32(&k_full[s]), kTileBytes);
        tma_load_3d(smem_u32(sK + s * kTileBytes), stale ? &mks : &mkf, smem_u32(&k_full[s]), 0, row, head);
        if (round > 0 && !mbar_wait(smem_u32(&v_empty[s]), (round - 1) & 1, err, kErrWaitStageFree)) {
          s_abort = 1;
          mbar_arrive_expect_tx(smem_u32(&v_full[s]), 0);
          ++issued;
          break;
        }
        mbar_arrive_expect_tx(smem_u32(&v_full[s]), kTileBytes);
        tma_load_3d(smem_u32(sV + s * kTileBytes), stale ? &mvs : &mvf, smem_u32(&v_full[s]), 0, row, head);
        ++issued;
      }
      if (s_abort) {
        for (int jj = (issued > kStages ? issued - kStages : 0); jj < issued; ++jj) {
          mbar_wait(smem_u32(&k_full[jj % kStages]), (jj / kStages) & 1, err, kErrWaitTmaFull);
          mbar_wait(smem_u32(&v_full[jj % kStages]), (jj / kStages) & 1, err, kErrWaitTmaFull);
        }
      }
    }
   } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Per MMA, every operand is a per-tile base plus a compile-time offset (the two
      // groups and the K slices are unrolled): runtime arithmetic between
      // tcgen05.mma instructions stalls their issue.
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTile, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, kOCols, false, true);
      constexpr uint64_t kTileDesc = kTileBytes >> 4;            // one tile in descriptor address units
      const uint64_t qd0 = sw128_kmajor_desc(smem_u32(sQ));
      const uint64_t kd0 = sw128_kmajor_desc(smem_u32(sK));
      // V stage 0 with the ones block as its second 64-column atom (leading byte offset);
      // stage st: start address + st tiles, leading byte offset - st tiles
      uint64_t vd0 = sw128_mnmajor_desc(smem_u32(sV));
      vd0 = (vd0 & ~(uint64_t(0x3FFF) << 16)) |
            (uint64_t(((smem_u32(sOnes) - smem_u32(sV)) >> 4) & 0x3FFF) << 16);
      const bool two = activeB;
      bool ok = mbar_wait(smem_u32(q_full), 0, err, kErrWaitTmaFull);
      // S_g = Q_g K^T, K tile at descriptor kd
#define DFP_ISSUE_S(G, KD)                                                   \
      do {                                                                   \
        const uint64_t qd = qd0 + (uint64_t)(G) * kTileDesc;                 \
        umma_f16_ss(tmem + 128 * (G), qd, (KD), idesc_s, 0);                 \
        umma_f16_ss(tmem + 128 * (G), qd + 2, (KD) + 2, idesc_s, 1);         \
        umma_f16_ss(tmem + 128 * (G), qd + 4, (KD) + 4, idesc_s, 1);         \
        umma_f16_ss(tmem + 128 * (G), qd + 6, (KD) + 6, idesc_s, 1);         \
        umma_commit(smem_u32(&s_full[G]));                                   \
      } while (0)
      // O_g += P_g [V | 1], V tile at descriptor vd (P read from TMEM over S_g)
#define DFP_ISSUE_PV(G, VD, ACC0)                                                                \
      do {                                                                                       \
        umma_f16_ts(tmem + 256 + 128 * (G), tmem + 128 * (G), (VD), idesc_o, (ACC0));            \
        _Pragma("unroll") for (int kk = 1; kk < 8; ++kk)                                         \
          umma_f16_ts(tmem + 256 + 128 * (G), tmem + 128 * (G) + kk * 8, (VD) + (uint64_t)kk * 128, idesc_o, 1); \
        umma_commit(smem_u32(&o_done[G]));                                                       \
      } while (0)
      if (ok && !mbar_wait(smem_u32(&k_full[0]), 0, err, kErrWaitTmaFull)) ok = false;
      if (ok) {
        tc_fence_after();
        DFP_ISSUE_S(0, kd0);
        if (two) DFP_ISSUE_S(1, kd0);
        umma_commit(smem_u32(&k_empty[0]));
      }
      for (int jj = 0; ok && jj < nt; ++jj) {
        const int st = jj % kStages, st1 = (jj + 1) % kStages;
        const uint32_t par = (uint32_t)(jj / kStages) & 1u, par1 = (uint32_t)((jj + 1) / kStages) & 1u;
        const bool more = jj + 1 < nt;
        const uint32_t acc0 = jj > 0;
        const uint64_t vd = vd0 + (uint64_t)st * (kTileDesc - (kTileDesc << 16));
        const uint64_t kd1 = kd0 + (uint64_t)st1 * kTileDesc;
        if (!mbar_wait(smem_u32(&v_full[st]), par, err, kErrWaitTmaFull)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&p_full[0]), (uint32_t)jj & 1u, err, kErrWaitAttnP)) { ok = false; break; }
        tc_fence_after();
        DFP_ISSUE_PV(0, vd, acc0);
        if (more) {
          if (!mbar_wait(smem_u32(&k_full[st1]), par1, err, kErrWaitTmaFull)) { ok = false; break; }
          tc_fence_after();
          DFP_ISSUE_S(0, kd1);
        }
        if (two) {
          if (!mbar_wait(smem_u32(&p_full[1]), (uint32_t)jj & 1u, err, kErrWaitAttnP)) { ok = false; break; }
          tc_fence_after();
          DFP_ISSUE_PV(1, vd, acc0);
          if (more) DFP_ISSUE_S(1, kd1);
        }
        umma_commit(smem_u32(&v_empty[st]));
        if (more) umma_commit(smem_u32(&k_empty[st1]));
      }
#undef DFP_ISSUE_S
#undef DFP_ISSUE_PV
      if (!ok) s_abort = 1;
    }
   }
  } else {
    // ------------------------------------------------------------ softmax groups (warps 0..15)
    const int g = warp >> 3;                    // query tile of this warp
    const int half = (warp >> 2) & 1;           // key columns [64 half, 64 half + 64)
    const int sub = warp & 3;                   // TMEM lane quadrant
    const int row = sub * 32 + lane;
    const bool active = g == 0 || activeB;
    const uint32_t lane_off = (uint32_t)(sub * 32) << 16;
    const uint32_t tS = tmem + 128 * g + lane_off;
    const uint32_t tO = tmem + 256 + 128 * g + lane_off;
    const float sl2 = 0.125f * 1.4426950408889634f;   // (1/sqrt(64)) * log2(e)
    float m_used = -INFINITY;
    bool ok = active;
    // A failed wait only marks the thread; the group leaves the loop together at the
    // next max-exchange barrier (bar.red.or), so no thread is left waiting there.
    bool carry = false;                         // a failed wait of the previous tile
    for (int jj = 0; ok && jj < nt; ++jj) {
      int stale, krow, valid;
      seg_tile(segs, j0 + jj, stale, krow, valid);
      bool bad = !mbar_wait(smem_u32(&s_full[g]), jj & 1, err, kErrWaitAttnS) || carry;
      tc_fence_after();
      float sc[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + half * 64 + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) sc[c * 32 + i] = __uint_as_float(r[i]);
      }
      tmem_wait_ld();
      const int vcols = valid - half * 64;     // valid columns of this half (may be <= 0 or >= 64)
      const bool full_tile = valid == kTile;
      if (!full_tile) {
#pragma unroll
        for (int i = 0; i < 64; ++i) sc[i] = i < vcols ? sc[i] : -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = max3(sc[i], sc[8 + i], sc[16 + i]);
#pragma unroll
      for (int i = 24; i < 64; i += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], sc[i + k], i + 8 + k < 64 ? sc[i + 8 + k] : mx[k]);
      }
      const float mhalf = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      // exchange with the other half of the row (double-buffered by tile parity)
      s_rowmax[jj & 1][g][half][row] = mhalf;
      if (named_bar_or(2 + g, 256, bad)) { ok = false; s_abort = 1; break; }
      const float mrow = fmaxf(mhalf, s_rowmax[jj & 1][g][half ^ 1][row]) * sl2;
      if (jj == 0) {
        m_used = mrow;
      } else {
        const bool need = mrow > m_used + kRescale;
        if (__any_sync(0xffffffffu, need)) {
          // both halves of a row see the same mrow, so they agree on every decision
          const float m_new = need ? mrow : m_used;
          const float alpha = ex2_mufu(m_used - m_new);
          if (!mbar_wait(smem_u32(&o_done[g]), (jj - 1) & 1, err, kErrWaitAttnO)) carry = true;
          tc_fence_after();
          // O (64 columns) and its row sums (16): half 0 rescales columns 0-39, half 1 40-79
#pragma unroll
          for (int c = 0; c < 5; ++c) {
            uint32_t r8[8];
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                         : "=r"(r8[0]), "=r"(r8[1]), "=r"(r8[2]), "=r"(r8[3]), "=r"(r8[4]), "=r"(r8[5]),
                           "=r"(r8[6]), "=r"(r8[7])
                         : "r"(tO + half * 40 + c * 8));
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i) r8[i] = __float_as_uint(__uint_as_float(r8[i]) * alpha);
            asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                         ::"r"(tO + half * 40 + c * 8), "r"(r8[0]), "r"(r8[1]), "r"(r8[2]), "r"(r8[3]),
                           "r"(r8[4]), "r"(r8[5]), "r"(r8[6]), "r"(r8[7])
                         : "memory");
          }
          tmem_wait_st();
          m_used = m_new;
        }
      }
      const float nm = -m_used;
      if (full_tile) {
        // x = s * c - m on pairs (fp32x2); a fixed share of the pairs through the
        // polynomial on the FMA pipe, the rest through the MUFU
        const uint64_t sl2x2 = f2(sl2, sl2), nmx2 = f2(nm, nm);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t x2 = fma2(f2(sc[c * 32 + e], sc[c * 32 + e + 1]), sl2x2, nmx2);
            if (((e >> 1) & 7) < kPolyPer8) {
              pk[e >> 1] = ex2_poly_pair_bf16(x2);
            } else {
              float x0, x1;
              f2_split(x2, x0, x1);
              pk[e >> 1] = pack_trunc(ex2_mufu(x0), ex2_mufu(x1));
            }
          }
          tmem_st16(tS + half * 32 + c * 16, pk);
        }
      } else {
        // partial tile: masked columns are -inf, which only the MUFU maps to exactly 0
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pk[e >> 1] = pack_trunc(ex2_mufu(fmaf(sc[c * 32 + e], sl2, nm)),
                                    ex2_mufu(fmaf(sc[c * 32 + e + 1], sl2, nm)));
          tmem_st16(tS + half * 32 + c * 16, pk);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[g]));
    }
    // every active thread of the group reaches this barrier exactly once
    if (active && named_bar_or(2 + g, 256, carry || !ok)) { ok = false; s_abort = 1; }
    // ---- epilogue: this half's 32 output columns and the row sum
    float o[32], l = 1.f;
    bool have = false;
    if (ok && !s_abort) {
      if (mbar_wait(smem_u32(&o_done[g]), (nt - 1) & 1, err, kErrWaitAttnO)) {
        tc_fence_after();
        uint32_t r[32], r16[16];
        tmem_ld32(tO + half * 32, r);
        tmem_ld16(tO + 64, r16);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(r[i]);
        l = __uint_as_float(r16[0]);
        have = true;
      } else {
        s_abort = 1;
      }
    }
    const int q_local = (qt0 + g) * kTile + row;
    const bool row_ok = have && q_local < a.Lp;
    __nv_bfloat16* out_row = static_cast<__nv_bfloat16*>(a.o) + (size_t)(p * a.Lp + q_local) * a.C + head * 64 + half * 32;
    if (splits == 1) {
      if (row_ok) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(out_row);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float w8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) w8[e] = o[c * 8 + e] * inv;
          dst[c] = pack16(w8);
        }
      }
    } else {
      // partial results of this split, then the last CTA of the pair merges them
      const size_t grp = ((size_t)head * a.N + p) * ((a.n_qtiles + 1) / 2) + pair;
      const size_t slot = (grp * splits + split) * 256 + g * 128 + row;
      if (have) {
        float4* po = reinterpret_cast<float4*>(a.part_o + slot * 64 + half * 32);
#pragma unroll
        for (int c = 0; c < 8; ++c) po[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        if (half == 0) reinterpret_cast<float2*>(a.part_ml)[slot] = make_float2(m_used, l);
      }
      __threadfence();
      named_bar(1, kSoftmaxThreads);
      if (threadIdx.x == 0) s_last = atomicAdd(a.counters + grp, 1u) == (unsigned)(splits - 1);
      named_bar(1, kSoftmaxThreads);
      if (s_last) {
        __threadfence();
        if (row_ok) {
          float mm = -INFINITY;
          for (int s2 = 0; s2 < splits; ++s2)
            mm = fmaxf(mm, __ldcg(reinterpret_cast<const float2*>(a.part_ml) + (grp * splits + s2) * 256 + g * 128 + row).x);
          float acc[32], lsum = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.f;
          for (int s2 = 0; s2 < splits; ++s2) {
            const size_t sl = (grp * splits + s2) * 256 + g * 128 + row;
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + sl);
            const float w = ex2_mufu(ml.x - mm);
            lsum = fmaf(ml.y, w, lsum);
            const float4* po = reinterpret_cast<const float4*>(a.part_o + sl * 64 + half * 32);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 v = __ldcg(po + c);
              acc[4 * c] = fmaf(v.x, w, acc[4 * c]);
              acc[4 * c + 1] = fmaf(v.y, w, acc[4 * c + 1]);
              acc[4 * c + 2] = fmaf(v.z, w, acc[4 * c + 2]);
              acc[4 * c + 3] = fmaf(v.w, w, acc[4 * c + 3]);
            }
          }
          const float inv = 1.f / lsum;
          uint4* dst = reinterpret_cast<uint4*>(out_row);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w8[e] = acc[c * 8 + e] * inv;
            dst[c] = pack16(w8);
          }
        }
        if (threadIdx.x == 0) a.counters[grp] = 0u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int attention_splits(int L, int Lp, int N, int heads, int mode_min_tiles) {
  const int n_qt = (Lp + kTile - 1) / kTile;
  const int groups = ((n_qt + 1) / 2) * N * heads;
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 4; ++s) {
    if (s > 1 && mode_min_tiles / s < 2) break;
    const long items = (long)groups * s;
    const long waves = (items + 147) / 148;
    const double eff = (double)items / (double)(waves * 148);
    if (eff > best_eff + 0.03) { best_eff = eff; best = s; }
    if (eff >= 0.7) break;   // each split adds a CTA prologue and a merge: stop early
  }
  return best;
}

cudaError_t launch_tc_attention(const TcAttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mkf,
                                const CUtensorMap& mvf, const CUtensorMap& mks,
                                const CUtensorMap& mvs, cudaStream_t s) {
  const size_t smem = 1024 + (2 + 2 * kStages + 1) * (size_t)kTileBytes + (4 * kStages + 8) * 8 + 64;
  cudaError_t e = cudaFuncSetAttribute(tc_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_qt = (a.Lp + kTile - 1) / kTile;
  dim3 grid(((n_qt + 1) / 2) * a.splits, a.N, a.heads);
  tc_attention_kernel<<<grid, kThreads, smem, s>>>(mq, mkf, mvf, mks, mvs, a);
  return cudaGetLastError();
}

}  // namespace dfp
