// GroupNorm over row patches with stale cross-patch statistics, and the halo
// refresh of the conv input cache.  All three kernels are HBM-bandwidth bound.
//
// DistriGroupNorm ("DistriFusion源码探秘" source walkthrough, Patch Parallelism
// section, item 3) with the "corrected asynchronous" default of the --sync_mode
// flag (DistriFusion project README, Benchmarks).  Per (patch p, group g) the
// step's moments m_p = (E[x], E[x^2]) are merged with the previous step's:
//   sync       est_p = mean_j m_j(t)                      (exact full-map GroupNorm)
//   corrected  est_p = mean_j m_j(t-1) + (m_p(t) - m_p(t-1))
//   stale-oth. est_p = (m_p(t) + sum_{j != p} m_j(t-1)) / N
//   naive      est_p = m_p(t)                             (no cross-patch context)
//   mean = est.E[x], var = max(est.E[x^2] - mean^2, 0), rstd = 1 / sqrt(var + eps).
// The reductions are deterministic: per-thread sums in a fixed pixel order, a
// fixed-order shared-memory tree, and a last-block merge over the chunk partials
// in a fixed order (no floating-point atomics).
#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kGnThreads = 512;

template <typename T>
__global__ void __launch_bounds__(kGnThreads)
gn_stats_merge_kernel(GnArgs a, int n_chunks, int pix_per_chunk) {
  constexpr int VEC = VecTraits<T>::kN;
  extern __shared__ float sh[];                 // [2][PL][C] per-thread-row channel sums
  __shared__ float s_mom[256 * 2];              // merged fresh moments  [N*G][2]
  __shared__ float s_mr[256 * 2];               // (mean, rstd)          [N*G][2]
  __shared__ int s_last;
  const int C = a.C, G = a.G, N = a.N;
  const int V = C / VEC;
  const int PL = kGnThreads / V;                // pixel lanes
  const int tid = threadIdx.x;
  const int vc = tid % V, pl = tid / V;
  const int p = blockIdx.y, chunk = blockIdx.x;

  // ---- phase 1: per-channel partial sums of this chunk of patch p
  float s1[VEC], s2[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) s1[i] = s2[i] = 0.f;
  if (pl < PL) {
    const int pix0 = chunk * pix_per_chunk;
    const int pix1 = min(pix0 + pix_per_chunk, a.pix_per_patch);
    const T* base = static_cast<const T*>(a.x) + (size_t)p * a.pix_per_patch * C + vc * VEC;
    int pix = pix0 + pl;
    for (; pix + 3 * PL < pix1; pix += 4 * PL) {
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) u[j] = ld_nc16(base + (size_t)(pix + j * PL) * C);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v[VEC];
        unpack16(u[j], v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) { s1[i] += v[i]; s2[i] = fmaf(v[i], v[i], s2[i]); }
      }
    }
    for (; pix < pix1; pix += PL) {
      float v[VEC];
      unpack16(ld_nc16(base + (size_t)pix * C), v);
#pragma unroll
      for (int i = 0; i < VEC; ++i) { s1[i] += v[i]; s2[i] = fmaf(v[i], v[i], s2[i]); }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      sh[pl * C + vc * VEC + i] = s1[i];
      sh[PL * C + pl * C + vc * VEC + i] = s2[i];
    }
  }
  __syncthreads();
  const int cg = C / G;
  for (int g = tid; g < G; g += kGnThreads) {
    float t1 = 0.f, t2 = 0.f;
    for (int c = g * cg; c < (g + 1) * cg; ++c)
      for (int l = 0; l < PL; ++l) { t1 += sh[l * C + c]; t2 += sh[PL * C + l * C + c]; }
    float2* dst = reinterpret_cast<float2*>(a.part) + ((size_t)p * n_chunks + chunk) * G + g;
    *dst = make_float2(t1, t2);
  }

  // ---- phase 2: the last block to finish merges every partial in a fixed order
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counter, 1u) == gridDim.x * gridDim.y - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int NG = N * G;                         // <= 256 (checked on the host)
  const int S = kGnThreads / NG;                // threads per (patch, group)
  float* red = sh;                              // [S][NG][2] reuse
  if (tid < S * NG) {
    const int item = tid % NG, part_id = tid / NG;
    const int pp = item / G, gg = item % G;
    const float2* src = reinterpret_cast<const float2*>(a.part) + (size_t)pp * n_chunks * G + gg;
    float t1 = 0.f, t2 = 0.f;
    for (int c = part_id; c < n_chunks; c += S) {
      const float2 v = __ldcg(src + (size_t)c * G);
      t1 += v.x; t2 += v.y;
    }
    red[(part_id * NG + item) * 2 + 0] = t1;
    red[(part_id * NG + item) * 2 + 1] = t2;
  }
  __syncthreads();
  const float inv_n = 1.f / ((float)a.pix_per_patch * (float)cg);
  if (tid < NG) {
    float t1 = 0.f, t2 = 0.f;
    for (int s = 0; s < S; ++s) { t1 += red[(s * NG + tid) * 2]; t2 += red[(s * NG + tid) * 2 + 1]; }
    s_mom[tid * 2] = t1 * inv_n;
    s_mom[tid * 2 + 1] = t2 * inv_n;
    a.fresh_out[tid * 2] = s_mom[tid * 2];
    a.fresh_out[tid * 2 + 1] = s_mom[tid * 2 + 1];
  }
  __syncthreads();
  if (tid < NG) {
    const int pp = tid / G, gg = tid % G;
    float e1, e2;
    if (a.naive) {
      e1 = s_mom[tid * 2]; e2 = s_mom[tid * 2 + 1];
    } else if (a.is_sync) {
      e1 = 0.f; e2 = 0.f;
      for (int j = 0; j < N; ++j) { e1 += s_mom[(j * G + gg) * 2]; e2 += s_mom[(j * G + gg) * 2 + 1]; }
      e1 /= (float)N; e2 /= (float)N;
    } else {
      float st1 = 0.f, st2 = 0.f;
      for (int j = 0; j < N; ++j) { st1 += a.stale[(j * G + gg) * 2]; st2 += a.stale[(j * G + gg) * 2 + 1]; }
      const float own1 = a.stale[(pp * G + gg) * 2], own2 = a.stale[(pp * G + gg) * 2 + 1];
      if (a.mode == 0) {        // corrected
        e1 = st1 / (float)N + (s_mom[tid * 2] - own1);
        e2 = st2 / (float)N + (s_mom[tid * 2 + 1] - own2);
      } else {                  // stale others
        e1 = (s_mom[tid * 2] + (st1 - own1)) / (float)N;
        e2 = (s_mom[tid * 2 + 1] + (st2 - own2)) / (float)N;
      }
    }
    const float var = fmaxf(e2 - e1 * e1, 0.f);
    const float rstd = 1.f / sqrtf(var + a.eps);
    s_mr[tid * 2] = e1;
    s_mr[tid * 2 + 1] = rstd;
    a.dbg[tid * 2] = e1;
    a.dbg[tid * 2 + 1] = rstd;
  }
  __syncthreads();
  for (int i = tid; i < N * C; i += kGnThreads) {
    const int pp = i / C, c = i % C, gg = c / cg;
    const float mean = s_mr[(pp * G + gg) * 2], rstd = s_mr[(pp * G + gg) * 2 + 1];
    const float sc = a.gamma[c] * rstd;
    reinterpret_cast<float2*>(a.coef)[i] = make_float2(sc, a.beta[c] - mean * sc);
  }
  if (tid == 0) *a.counter = 0u;
}

__device__ __forceinline__ float silu_f(float y) { return y / (1.f + expf(-y)); }

template <typename T, bool SILU>
__global__ void __launch_bounds__(kGnThreads)
gn_apply_kernel(const T* __restrict__ x, T* __restrict__ out, const float* __restrict__ coef,
                int pix_per_patch, int C, long long out_patch_stride, long long out_off,
                int pix_per_chunk) {
  constexpr int VEC = VecTraits<T>::kN;
  const int V = C / VEC;
  const int PL = kGnThreads / V;
  const int vc = threadIdx.x % V, pl = threadIdx.x / V;
  if (pl >= PL) return;
  const int p = blockIdx.y, chunk = blockIdx.x;
  float sc[VEC], sf[VEC];
  const float2* cf = reinterpret_cast<const float2*>(coef) + (size_t)p * C + vc * VEC;
#pragma unroll
  for (int i = 0; i < VEC; ++i) { const float2 t = cf[i]; sc[i] = t.x; sf[i] = t.y; }
  const int pix0 = chunk * pix_per_chunk;
  const int pix1 = min(pix0 + pix_per_chunk, pix_per_patch);
  const T* src = x + (size_t)p * pix_per_patch * C + vc * VEC;
  T* dst = out + ((size_t)p * out_patch_stride + out_off) * C + vc * VEC;
  int pix = pix0 + pl;
  for (; pix + PL < pix1; pix += 2 * PL) {
    uint4 u0 = ld_nc16(src + (size_t)pix * C);
    uint4 u1 = ld_nc16(src + (size_t)(pix + PL) * C);
    float v0[VEC], v1[VEC];
    unpack16(u0, v0);
    unpack16(u1, v1);
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      v0[i] = fmaf(v0[i], sc[i], sf[i]);
      v1[i] = fmaf(v1[i], sc[i], sf[i]);
      if (SILU) { v0[i] = silu_f(v0[i]); v1[i] = silu_f(v1[i]); }
    }
    *reinterpret_cast<uint4*>(dst + (size_t)pix * C) = pack16(v0);
    *reinterpret_cast<uint4*>(dst + (size_t)(pix + PL) * C) = pack16(v1);
  }
  for (; pix < pix1; pix += PL) {
    float v[VEC];
    unpack16(ld_nc16(src + (size_t)pix * C), v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      v[i] = fmaf(v[i], sc[i], sf[i]);
      if (SILU) v[i] = silu_f(v[i]);
    }
    *reinterpret_cast<uint4*>(dst + (size_t)pix * C) = pack16(v);
  }
}

template <typename T>
__global__ void halo_refresh_kernel(const T* __restrict__ src, T* __restrict__ dst, int R, int W, int C) {
  constexpr int VEC = VecTraits<T>::kN;
  const int b = blockIdx.y >> 1, dir = blockIdx.y & 1;
  const size_t row = (size_t)W * C;
  const size_t slab = (size_t)(R + 2) * row;
  // dir 0: top halo of patch b+1 <- last interior row of patch b
  // dir 1: bottom halo of patch b <- first interior row of patch b+1
  const T* s = dir == 0 ? src + b * slab + (size_t)R * row : src + (b + 1) * slab + row;
  T* d = dir == 0 ? dst + (b + 1) * slab : dst + b * slab + (size_t)(R + 1) * row;
  const int nvec = (int)(row / VEC);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += gridDim.x * blockDim.x)
    reinterpret_cast<uint4*>(d)[i] = ld_nc16(reinterpret_cast<const uint4*>(s) + i);
}

int chunk_pixels(int N, int pix_per_patch) {
  // about two resident 512-thread blocks per SM over the whole map
  const int target_blocks = 296;
  int per = (N * pix_per_patch + target_blocks - 1) / target_blocks;
  if (per < 16) per = 16;
  return per;
}

}  // namespace

int gn_stats_chunks(int N, int pix_per_patch) {
  const int per = chunk_pixels(N, pix_per_patch);
  return (pix_per_patch + per - 1) / per;
}

template <typename T>
cudaError_t launch_gn_stats_merge(const GnArgs& a, cudaStream_t s) {
  constexpr int VEC = VecTraits<T>::kN;
  const int per = chunk_pixels(a.N, a.pix_per_patch);
  const int n_chunks = (a.pix_per_patch + per - 1) / per;
  const int V = a.C / VEC;
  const int PL = kGnThreads / V;
  size_t smem = (size_t)2 * PL * a.C * sizeof(float);
  const size_t red = (size_t)kGnThreads * 2 * sizeof(float);
  if (smem < red) smem = red;
  dim3 grid(n_chunks, a.N);
  gn_stats_merge_kernel<T><<<grid, kGnThreads, smem, s>>>(a, n_chunks, per);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gn_apply(const T* x, T* out, const float* coef, int N, int pix_per_patch, int C,
                            long long out_patch_stride_pix, long long out_pix_off, bool silu,
                            cudaStream_t s) {
  const int per = chunk_pixels(N, pix_per_patch);
  dim3 grid((pix_per_patch + per - 1) / per, N);
  if (silu)
    gn_apply_kernel<T, true><<<grid, kGnThreads, 0, s>>>(x, out, coef, pix_per_patch, C,
                                                         out_patch_stride_pix, out_pix_off, per);
  else
    gn_apply_kernel<T, false><<<grid, kGnThreads, 0, s>>>(x, out, coef, pix_per_patch, C,
                                                          out_patch_stride_pix, out_pix_off, per);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_halo_refresh(const T* src_slab, T* dst_slab, int N, int R, int W, int C,
                                cudaStream_t s) {
  if (N < 2) return cudaSuccess;
  constexpr int VEC = VecTraits<T>::kN;
  const int nvec = W * C / VEC;
  const int threads = 256;
  int bx = (nvec + threads - 1) / threads;
  if (bx > 64) bx = 64;
  dim3 grid(bx, 2 * (N - 1));
  halo_refresh_kernel<T><<<grid, threads, 0, s>>>(src_slab, dst_slab, R, W, C);
  return cudaGetLastError();
}

template cudaError_t launch_gn_stats_merge<float>(const GnArgs&, cudaStream_t);
template cudaError_t launch_gn_stats_merge<__nv_bfloat16>(const GnArgs&, cudaStream_t);
template cudaError_t launch_gn_apply<float>(const float*, float*, const float*, int, int, int,
                                            long long, long long, bool, cudaStream_t);
template cudaError_t launch_gn_apply<__nv_bfloat16>(const __nv_bfloat16*, __nv_bfloat16*,
                                                    const float*, int, int, int, long long,
                                                    long long, bool, cudaStream_t);
template cudaError_t launch_halo_refresh<float>(const float*, float*, int, int, int, int,
                                                cudaStream_t);
template cudaError_t launch_halo_refresh<__nv_bfloat16>(const __nv_bfloat16*, __nv_bfloat16*, int,
                                                        int, int, int, cudaStream_t);

}  // namespace dfp
