// Tensor-core (tcgen05 / TMEM / TMA) GEMM for sm_100a, bf16 operands, fp32 accumulate.
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

template <int BN> struct TmemCols { static constexpr uint32_t v = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256; };

struct TileInfo {
  int p, i0, j0, m0;  // conv: patch, patch-local first row, first column; plain: first row
};

__device__ __forceinline__ TileInfo tile_of(const TcGemmPlan& pl, int m_tile) {
  TileInfo t{};
  if (pl.conv) {
    const int per_patch = (pl.R / pl.rows_tile) * pl.tiles_per_row;
    t.p = m_tile / per_patch;
    const int rem = m_tile - t.p * per_patch;
    const int it = rem / pl.tiles_per_row;
    const int jt = rem - it * pl.tiles_per_row;
    t.i0 = it * pl.rows_tile;
    t.j0 = jt * pl.cols_tile;
  } else {
    t.m0 = m_tile * kBM;
  }
  return t;
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
               const TcGemmPlan plan, const Epilogue epi, int* err) {
  constexpr uint32_t kABytes = kBM * kBK * 2;
  constexpr uint32_t kBBytes = BN * kBK * 2;
  constexpr uint32_t kCols = TmemCols<BN>::v;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * kBBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* accum = bars + 2 * STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const TileInfo tile = tile_of(plan, blockIdx.y);
  const int num_kb = plan.K / kBK;
  const uint32_t a_box_bytes =
      plan.conv ? (uint32_t)(plan.rows_tile * plan.cols_tile * kBK * 2) : kABytes;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) { mbar_init(smem_u32(&full[s]), 1); mbar_init(smem_u32(&empty[s]), 1); }
    mbar_init(smem_u32(accum), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mapA);
      tma_prefetch_desc(&mapB);
      const int kc_per_tap = plan.conv ? plan.Cin / kBK : 1;
      int issued = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % STAGES, round = kb / STAGES;
        if (round > 0 && !mbar_wait(smem_u32(&empty[s]), (round - 1) & 1, err, kErrWaitStageFree)) {
          s_abort = 1;
          break;
        }
        const uint32_t fb = smem_u32(&full[s]);
        mbar_arrive_expect_tx(fb, a_box_bytes + kBBytes);
        if (plan.conv) {
          const int tap = kb / kc_per_tap, kc = kb - tap * kc_per_tap;
          const int r = tap / 3, sx = tap - 3 * (tap / 3);
          tma_load_4d(smem_u32(sA + s * kABytes), &mapA, fb, kc * kBK, tile.j0 + sx - 1, tile.i0 + r, tile.p);
        } else {
          tma_load_2d(smem_u32(sA + s * kABytes), &mapA, fb, kb * kBK, tile.m0);
        }
        tma_load_2d(smem_u32(sB + s * kBBytes), &mapB, fb, kb * kBK, n0);
        ++issued;
      }
      if (s_abort) {
        // let the copies already in flight land before the CTA can exit
        for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
          mbar_wait(smem_u32(&full[kb % STAGES]), (kb / STAGES) & 1, err, kErrWaitTmaFull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // The stage ring is unrolled so that every MMA operand is a hoisted descriptor
      // plus a compile-time offset: runtime arithmetic between tcgen05.mma
      // instructions stalls their issue.
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
      const uint64_t ad0 = sw128_kmajor_desc(smem_u32(sA));
      const uint64_t bd0 = sw128_kmajor_desc(smem_u32(sB));
      bool ok = true;
      for (int kb0 = 0; ok && kb0 < num_kb; kb0 += STAGES) {
        const uint32_t par = (uint32_t)(kb0 / STAGES) & 1u;
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
          const int kb = kb0 + s;
          if (kb >= num_kb) break;
          if (!mbar_wait(smem_u32(&full[s]), par, err, kErrWaitTmaFull)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = ad0 + (uint64_t)((s * kABytes) >> 4);
          const uint64_t bd = bd0 + (uint64_t)((s * kBBytes) >> 4);
          umma_f16_ss(tmem_d, ad, bd, idesc, kb > 0);
#pragma unroll
          for (int kk = 1; kk < kBK / 16; ++kk) umma_f16_ss(tmem_d, ad + 2 * kk, bd + 2 * kk, idesc, 1);
          umma_commit(smem_u32(&empty[s]));
        }
      }
      if (!ok) s_abort = 1;
      umma_commit(smem_u32(accum));
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const bool ready = mbar_wait(smem_u32(accum), 0, err, kErrWaitAccum);
    tc_fence_after();
    long long gm = -1;
    if (plan.conv) {
      const int rr = row / plan.cols_tile, jj = row - rr * plan.cols_tile;
      if (rr < plan.rows_tile && tile.j0 + jj < plan.W)
        gm = ((long long)tile.p * plan.R + tile.i0 + rr) * plan.W + tile.j0 + jj;
    } else if (tile.m0 + row < plan.M) {
      gm = tile.m0 + row;
    }
    if (!ready || s_abort) gm = -1;
    const uint32_t taddr = tmem_d + ((uint32_t)(sub * 32) << 16);
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
          const float a = __uint_as_float(rv[i]) + __ldg(epi.bias + nv + i);
          const float g = __uint_as_float(rg[i]) + __ldg(epi.bias + ng + i);
          w[i] = a * (0.5f * g * (1.f + erff(g * 0.70710678118654752f)));
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
    } else
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_wait_ld();
      const int n = n0 + c * 32;
      if (gm < 0 || n >= plan.N) continue;
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
          const uint4* r4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(epi.residual) + gm * epi.ldo + n);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float rr[8];
            unpack16(r4[i], rr);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[i * 8 + e] += rr[e];
          }
        }
        dst = static_cast<__nv_bfloat16*>(epi.out) + gm * epi.ldo + n;
      } else {
        const int which = n / epi.C, cc = n - which * epi.C;
        const int head = cc >> 6, d0 = cc & 63;
        void* base = which == 0 ? epi.q : (which == 1 ? epi.k : epi.v);
        dst = static_cast<__nv_bfloat16*>(base) + ((long long)head * epi.L + gm) * 64 + d0;
      }
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = v[i * 8 + e];
        d4[i] = pack16(w8);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, kCols);
  }
}

template <int BN, int STAGES>
cudaError_t launch_bn(const TcGemmPlan& plan, const CUtensorMap& mA, const CUtensorMap& mB,
                      const Epilogue& epi, int* err, cudaStream_t s) {
  const size_t smem = 1024 + (size_t)STAGES * (kBM * kBK * 2 + BN * kBK * 2) + (2 * STAGES + 2) * 8 + 64;
  auto kern = tc_gemm_kernel<BN, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int m_tiles;
  if (plan.conv)
    m_tiles = plan.P * (plan.R / plan.rows_tile) * plan.tiles_per_row;
  else
    m_tiles = (plan.M + kBM - 1) / kBM;
  dim3 grid(plan.N / BN, m_tiles);
  kern<<<grid, kThreads, smem, s>>>(mA, mB, plan, epi, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm(const TcGemmPlan& plan, const CUtensorMap& mapA, const CUtensorMap& mapB,
                           const Epilogue& epi, int* err, cudaStream_t s) {
  switch (plan.bn) {
    case 128: return launch_bn<128, 4>(plan, mapA, mapB, epi, err, s);
    case 160: return launch_bn<160, 4>(plan, mapA, mapB, epi, err, s);
    case 64: return launch_bn<64, 6>(plan, mapA, mapB, epi, err, s);
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
bool encode_tmap_4d(CUtensorMap* m, const void* base, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4]) {
  const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
  const cuuint64_t st[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
  return encode(m, base, 4, d, st, b);
}

}  // namespace dfp
