// Displaced self-attention on tcgen05 / TMEM / TMA (sm_100a), bf16 operands, fp32
// softmax and accumulation, head width 64.
//
// DistriSelfAttentionPP ("DistriFusion源码探秘" source walkthrough, Patch
// Parallelism section item 2): the queries of patch p attend to all L tokens; the
// K/V of its own rows are this step's, those of every other patch come from the
// previous step's cache (project README, Overview (c): activations of the
// previous step are reused).  The KV loop walks a list of segments:
//   sync       [0, L) fresh
//   displaced  own patch fresh, then [0, p*Lp) stale, then [(p+1)*Lp, L) stale
//   naive      own patch fresh only (the naive-patch baseline, README Overview (b))
// Segment boundaries need not be multiples of the 128-key tile: columns past a
// segment's end are masked to -inf.
//
// One CTA = one (128-query tile, head).  Warp 0: TMA (Q once, K/V two-stage
// rings), warp 1: one thread issues S = Q K^T (M=128, N=128, K=64) into TMEM and
// O_j = P_j V_j (M=128, N=64, K=128; V read MN-major) into a second TMEM region,
// warps 2-5: one thread per query row reads S from TMEM, runs the online softmax
// (exp2 on the MUFU), writes P (bf16) to shared memory in the 128-byte swizzle
// layout the MMA reads, and accumulates O = alpha * O + O_j in registers.
#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kThreads = 192;
constexpr int kTileQ = 128;
constexpr int kTileK = 128;
constexpr uint32_t kTileBytes = 128 * 64 * 2;   // one 128 x 64 bf16 tile
constexpr uint32_t kTmemCols = 256;             // S: cols [0,128), O_j: cols [128,192)

struct Segs {
  int n;
  int stale[3], start[3], len[3], tiles[3];
  int total;
};

__device__ __forceinline__ Segs make_segs(int mode, int p, int Lp, int L) {
  Segs s{};
  auto add = [&](int st, int b, int len) {
    if (len <= 0) return;
    s.stale[s.n] = st; s.start[s.n] = b; s.len[s.n] = len;
    s.tiles[s.n] = (len + kTileK - 1) / kTileK;
    s.total += s.tiles[s.n];
    ++s.n;
  };
  if (mode == kAttnSync) {
    add(0, 0, L);
  } else {
    add(0, p * Lp, Lp);
    if (mode == kAttnDisplaced) {
      add(1, 0, p * Lp);
      add(1, (p + 1) * Lp, L - (p + 1) * Lp);
    }
  }
  return s;
}

// tile j -> (stale?, first key row, valid keys)
__device__ __forceinline__ void seg_tile(const Segs& s, int j, int& stale, int& row, int& valid) {
  int k = 0;
  while (k < s.n - 1 && j >= s.tiles[k]) { j -= s.tiles[k]; ++k; }
  stale = s.stale[k];
  row = s.start[k] + j * kTileK;
  valid = min(kTileK, s.len[k] - j * kTileK);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_attention_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mkf,
                    const __grid_constant__ CUtensorMap mvf, const __grid_constant__ CUtensorMap mks,
                    const __grid_constant__ CUtensorMap mvs, const TcAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // 16 KB
  uint8_t* sK = sQ + kTileBytes;            // 2 x 16 KB
  uint8_t* sV = sK + 2 * kTileBytes;        // 2 x 16 KB
  uint8_t* sP = sV + 2 * kTileBytes;        // 32 KB: keys [0,64) then [64,128), each 128 rows x 128 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;
  uint64_t* p_full = bars + 10;
  uint64_t* o_full = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  __shared__ volatile int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.z, p = blockIdx.y;
  const int q_local0 = blockIdx.x * kTileQ;
  const int q_row0 = p * a.Lp + q_local0;
  const Segs segs = make_segs(a.mode, p, a.Lp, a.L);
  const int nt = segs.total;
  int* err = a.err;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1); mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1); mbar_init(smem_u32(&v_empty[i]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(p_full), 128);
    mbar_init(smem_u32(o_full), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem, tmem_o = tmem + 128;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mq);
      mbar_arrive_expect_tx(smem_u32(q_full), kTileBytes);
      tma_load_3d(smem_u32(sQ), &mq, smem_u32(q_full), 0, q_row0, head);
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j & 1, round = j >> 1;
        int stale, row, valid;
        seg_tile(segs, j, stale, row, valid);
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
        for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) {
          mbar_wait(smem_u32(&k_full[j & 1]), (j >> 1) & 1, err, kErrWaitTmaFull);
          mbar_wait(smem_u32(&v_full[j & 1]), (j >> 1) & 1, err, kErrWaitTmaFull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTileK, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 64, false, true);
      bool ok = mbar_wait(smem_u32(q_full), 0, err, kErrWaitTmaFull);
      const uint64_t qd = sw128_kmajor_desc(smem_u32(sQ));
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j & 1, round = j >> 1;
        if (!mbar_wait(smem_u32(&k_full[s]), round & 1, err, kErrWaitTmaFull)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kd = sw128_kmajor_desc(smem_u32(sK + s * kTileBytes));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_f16_ss(tmem_s, qd + 2 * kk, kd + 2 * kk, idesc_s, kk != 0);
        umma_commit(smem_u32(&k_empty[s]));
        umma_commit(smem_u32(s_full));
        if (!mbar_wait(smem_u32(p_full), j & 1, err, kErrWaitAttnP)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&v_full[s]), round & 1, err, kErrWaitTmaFull)) { ok = false; break; }
        tc_fence_after();
        const uint64_t vd = sw128_mnmajor_desc(smem_u32(sV + s * kTileBytes));
        const uint64_t pd0 = sw128_kmajor_desc(smem_u32(sP));
        const uint64_t pd1 = sw128_kmajor_desc(smem_u32(sP + kTileBytes));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = (kk < 4 ? pd0 : pd1) + 2 * (kk & 3);
          const uint64_t bd = vd + (uint64_t)((kk * 16 * 128) >> 4);   // 16 keys = 16 rows of 128 B
          umma_f16_ss(tmem_o, ad, bd, idesc_o, kk != 0);
        }
        umma_commit(smem_u32(&v_empty[s]));
        umma_commit(smem_u32(o_full));
      }
      if (!ok) s_abort = 1;
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 2..5)
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const uint32_t lane_off = (uint32_t)(sub * 32) << 16;
    const float sl2 = 0.125f * 1.4426950408889634f;   // (1/sqrt(64)) * log2(e)
    float m_run = -INFINITY, l_run = 0.f;
    float oacc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) oacc[i] = 0.f;
    uint8_t* prow = sP + row * 128;
    const int sw = row & 7;
    for (int j = 0; j < nt; ++j) {
      int stale, krow, valid;
      seg_tile(segs, j, stale, krow, valid);
      if (!mbar_wait(smem_u32(s_full), j & 1, err, kErrWaitAttnS)) { s_abort = 1; break; }
      tc_fence_after();
      float sc[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_s + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sc[c * 32 + i] = __uint_as_float(r[i]);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        sc[i] = i < valid ? sc[i] * sl2 : -INFINITY;
        mx = fmaxf(mx, sc[i]);
      }
      const float m_new = fmaxf(m_run, mx);
      const float alpha = ex2(m_run - m_new);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { pv[e] = ex2(sc[c * 8 + e] - m_new); rs += pv[e]; }
        const int blk = c >> 3, chunk = c & 7;
        *reinterpret_cast<uint4*>(prow + blk * kTileBytes + ((chunk ^ sw) << 4)) = pack16(pv);
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
      if (!mbar_wait(smem_u32(o_full), j & 1, err, kErrWaitAttnO)) { s_abort = 1; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_o + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) oacc[c * 32 + i] = fmaf(oacc[c * 32 + i], alpha, __uint_as_float(r[i]));
      }
      tc_fence_before();
    }
    if (!s_abort && q_local0 + row < a.Lp) {
      const float inv = 1.f / l_run;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) +
                                            (size_t)(q_row0 + row) * a.C + head * 64);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = oacc[c * 8 + e] * inv;
        dst[c] = pack16(w8);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_tc_attention(const TcAttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mkf,
                                const CUtensorMap& mvf, const CUtensorMap& mks,
                                const CUtensorMap& mvs, cudaStream_t s) {
  const size_t smem = 1024 + 7 * (size_t)kTileBytes + 13 * 8 + 64;
  cudaError_t e = cudaFuncSetAttribute(tc_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.Lp + kTileQ - 1) / kTileQ, a.N, a.heads);
  tc_attention_kernel<<<grid, kThreads, smem, s>>>(mq, mkf, mvf, mks, mvs, a);
  return cudaGetLastError();
}

}  // namespace dfp
