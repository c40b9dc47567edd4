// GroupNorm over row patches with stale cross-patch statistics (writing the conv input
// slab with its halo rows), and the per-token LayerNorm of the transformer stage.  All of
// them move whole feature maps once or twice: HBM (and at small sizes latency) bound.
//
// DistriGroupNorm ("DistriFusion源码探秘" source walkthrough, Patch Parallelism
// section, item 3) with the "corrected asynchronous" default of the --sync_mode
// flag (DistriFusion project README, Benchmarks).  Per (patch p, group g) the
// step's moments (E[x], E[x^2]) are merged with the previous step's:
//   sync       est_p = mean_j m_j(t)                      (exact full-map GroupNorm)
//   corrected  est_p = mean_j m_j(t-1) + (m_p(t) - m_p(t-1))
//   stale-oth. est_p = (m_p(t) + sum_{j != p} m_j(t-1)) / N
//   naive      est_p = m_p(t)                             (no cross-patch context)
// The GroupNorm-only variants of --sync_mode apply the sync rule (mode "sync") or the
// naive rule (mode "separate") on displaced steps too, the other layers staying displaced.
//   mean = est.E[x], var = max(est.E[x^2] - mean^2, 0), rstd = 1 / sqrt(var + eps).
// j runs over the N patches of the same image: a batch of images (the guidance
// batch) is images x N patches, numbered image-major, with nothing shared across images.
//
// Numerics.  In fp32, E[x^2] - mean^2 loses every digit of the variance when the mean
// is large next to the spread (at mean 30 and unit variance E[x^2] ~ 901 has an ulp of
// 6e-5).  So the kernels never form E[x^2]: each (patch, group) is summed as x - K with
// K the patch's first pixel in the group's first channel (one shift for every chunk and
// channel of the group, so the shifted sums still add across them), and the moments
// kept per (patch, group) are (mean, variance) = (K + S1/n, S2/n - (S1/n)^2).  Every merge
// rule above is a mixture of per-patch distributions, and is evaluated in that central
// form, which is the same value in exact arithmetic without the cancellation:
//   sync       mean = avg_j m_j, var = avg_j v_j + avg_j (m_j - mean)^2
//   corrected  with M, V the previous step's moments, d = m_p - M_p, M~ = avg_j M_j:
//              mean = M~ + d, var = avg_j V_j + (v_p - V_p) + avg_j (M_j - M~)^2 + 2 d (M_p - M~)
//   stale-oth. the components (m_p, v_p) and (M_j, V_j) for j != p:
//              mean = avg c, var = avg w + avg (c - mean)^2
// The reductions are deterministic: per-thread sums in a fixed pixel order, a
// fixed-order shared-memory tree, and a merge over the chunk partials in a fixed order
// (no floating-point atomics).
#include <algorithm>

#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kGnThreads = 512;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float load_f32(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_f32(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// The shift of (patch p, group g): the patch's first pixel in the group's first channel.
template <typename T>
__device__ __forceinline__ float gn_shift(const void* x, int p, int pix_per_patch, int C, int g, int cg) {
  return load_f32(static_cast<const T*>(x) + (size_t)p * pix_per_patch * C + (size_t)g * cg);
}

// Shifts of one thread's VEC channels c0 .. c0+VEC-1 (each the shift of its group).
template <typename T, int VEC>
__device__ __forceinline__ void gn_thread_shifts(const void* x, int p, int pix_per_patch, int C, int c0, int cg,
                                                 float (&k)[VEC]) {
#pragma unroll
  for (int i = 0; i < VEC; ++i) k[i] = gn_shift<T>(x, p, pix_per_patch, C, (c0 + i) / cg, cg);
}

// Merge rules of DistriGroupNorm on per-patch (mean, var) moments (see the file header).
enum GnRule : int { kGnNaive = 0, kGnSync = 1, kGnCorrected = 2, kGnStaleOthers = 3 };
// a.mode is the dfp_gn_mode: 0 corrected, 1 stale-others, 2 sync, 3 separate (the last two
// are GroupNorm-only variants: every step this step's full-map / patch-local statistics)
__device__ __forceinline__ int gn_rule(const GnArgs& a) {
  if (a.naive) return kGnNaive;
  if (a.is_sync) return kGnSync;
  switch (a.mode) {
    case 0: return kGnCorrected;
    case 1: return kGnStaleOthers;
    case 2: return kGnSync;
    default: return kGnNaive;
  }
}
// own: this step's moments of patch pi (of NI in its image); img: moments (mean, var) of
// the image's patches (this step's for kGnSync, the previous step's otherwise), patch j's
// pair at img[2 j stride] (scalar reads: no alignment assumed).  Returns (mean, var) of
// the estimate, var clamped at 0.
__device__ __forceinline__ float2 mom_at(const float* img, int j, int stride) {
  return make_float2(img[2 * j * stride], img[2 * j * stride + 1]);
}
__device__ __forceinline__ float2 gn_estimate(int rule, int NI, int pi, float2 own, const float* img, int stride) {
  const float inv = 1.f / (float)NI;
  float mu, var;
  if (rule == kGnNaive) {
    mu = own.x;
    var = own.y;
  } else if (rule == kGnCorrected) {
    float sm = 0.f, sv = 0.f;
    for (int j = 0; j < NI; ++j) { const float2 q = mom_at(img, j, stride); sm += q.x; sv += q.y; }
    const float mb = sm * inv;
    float ss = 0.f;
    for (int j = 0; j < NI; ++j) { const float e = mom_at(img, j, stride).x - mb; ss = fmaf(e, e, ss); }
    const float2 st = mom_at(img, pi, stride);
    const float d = own.x - st.x;
    mu = mb + d;
    var = sv * inv + (own.y - st.y) + ss * inv + 2.f * d * (st.x - mb);
  } else {
    // sync: every component is this step's; stale-others: all but patch pi are the previous step's
    float sm = 0.f, sv = 0.f;
    for (int j = 0; j < NI; ++j) {
      const float2 q = (rule == kGnStaleOthers && j == pi) ? own : mom_at(img, j, stride);
      sm += q.x; sv += q.y;
    }
    mu = sm * inv;
    float ss = 0.f;
    for (int j = 0; j < NI; ++j) {
      const float e = ((rule == kGnStaleOthers && j == pi) ? own : mom_at(img, j, stride)).x - mu;
      ss = fmaf(e, e, ss);
    }
    var = sv * inv + ss * inv;
  }
  return make_float2(mu, fmaxf(var, 0.f));
}

template <typename T>
__global__ void __launch_bounds__(kGnThreads)
gn_stats_merge_kernel(GnArgs a, int n_chunks, int pix_per_chunk) {
  constexpr int VEC = VecTraits<T>::kN;
  extern __shared__ float sh[];                 // [2][PL][C] lane sums, then [2][C] channel sums
  __shared__ __align__(16) float s_mom[512 * 2];   // fresh moments (mean, var) [N*G][2]
  __shared__ int s_last;
  const int C = a.C, G = a.G, N = a.N;
  const int V = C / VEC;
  const int PL = kGnThreads / V;                // pixel lanes
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vc = tid % V, pl = tid / V;
  const int p = blockIdx.y, chunk = blockIdx.x;
  float* chan = sh + 2 * PL * C;

  // ---- phase 1: per-channel partial sums of x - K (K: the group's shift) over this chunk
  // of patch p (8 loads in flight)
  float s1[VEC], s2[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) s1[i] = s2[i] = 0.f;
  if (pl < PL) {
    float k[VEC];
    gn_thread_shifts<T, VEC>(a.x, p, a.pix_per_patch, C, vc * VEC, C / G, k);
    const int pix0 = chunk * pix_per_chunk;
    const int pix1 = min(pix0 + pix_per_chunk, a.pix_per_patch);
    const T* base = static_cast<const T*>(a.x) + (size_t)p * a.pix_per_patch * C + vc * VEC;
    // eight predicated loads in flight per thread, then accumulate in pixel order
    for (int pix = pix0 + pl; pix < pix1; pix += 8 * PL) {
      uint4 u[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        u[j] = pix + j * PL < pix1 ? ld_nc16(base + (size_t)(pix + j * PL) * C) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (pix + j * PL >= pix1) break;   // past the chunk: a zero would add -K, K^2 to the sums
        float v[VEC];
        unpack16(u[j], v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          const float d = v[i] - k[i];
          s1[i] += d;
          s2[i] = fmaf(d, d, s2[i]);
        }
      }
    }
    float4* d1 = reinterpret_cast<float4*>(sh + pl * C + vc * VEC);
    float4* d2 = reinterpret_cast<float4*>(sh + PL * C + pl * C + vc * VEC);
#pragma unroll
    for (int i = 0; i < VEC / 4; ++i) {
      d1[i] = make_float4(s1[4 * i], s1[4 * i + 1], s1[4 * i + 2], s1[4 * i + 3]);
      d2[i] = make_float4(s2[4 * i], s2[4 * i + 1], s2[4 * i + 2], s2[4 * i + 3]);
    }
  }
  __syncthreads();
  for (int c = tid; c < C; c += kGnThreads) {
    float t1 = 0.f, t2 = 0.f;
    for (int l = 0; l < PL; ++l) { t1 += sh[l * C + c]; t2 += sh[PL * C + l * C + c]; }
    chan[c] = t1;
    chan[C + c] = t2;
  }
  __syncthreads();
  const int cg = C / G;
  for (int g = warp; g < G; g += kGnThreads / 32) {
    float t1 = 0.f, t2 = 0.f;
    for (int c = lane; c < cg; c += 32) { t1 += chan[g * cg + c]; t2 += chan[C + g * cg + c]; }
    t1 = warp_sum(t1);
    t2 = warp_sum(t2);
    if (lane == 0) {
      reinterpret_cast<float2*>(a.part)[((size_t)p * n_chunks + chunk) * G + g] = make_float2(t1, t2);
      __threadfence();                          // only the writers need to publish
    }
  }

  // ---- phase 2: the last block to finish merges every partial in a fixed order
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counter, 1u) == gridDim.x * gridDim.y - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int NG = N * G;                         // <= 512 (checked on the host)
  const int S = kGnThreads / NG;                // threads per (patch, group), >= 1
  float* red = sh;                              // [S][NG][2]
  if (tid < S * NG) {
    const int item = tid % NG, part_id = tid / NG;
    const int pp = item / G, gg = item % G;
    const float2* src = reinterpret_cast<const float2*>(a.part) + (size_t)pp * n_chunks * G + gg;
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    for (int c = part_id; c < n_chunks; c += 4 * S) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int cc = c + u * S;
        if (cc < n_chunks) {
          const float2 v = __ldcg(src + (size_t)cc * G);
          acc[u].x += v.x; acc[u].y += v.y;
        }
      }
    }
    red[(part_id * NG + item) * 2 + 0] = (acc[0].x + acc[1].x) + (acc[2].x + acc[3].x);
    red[(part_id * NG + item) * 2 + 1] = (acc[0].y + acc[1].y) + (acc[2].y + acc[3].y);
  }
  __syncthreads();
  const float inv_n = 1.f / ((float)a.pix_per_patch * (float)cg);
  if (tid < NG) {
    float t1 = 0.f, t2 = 0.f;
    for (int s = 0; s < S; ++s) { t1 += red[(s * NG + tid) * 2]; t2 += red[(s * NG + tid) * 2 + 1]; }
    // (mean, var) of patch tid / G, group tid % G from the shifted sums
    const float m1 = t1 * inv_n;
    const float mean = gn_shift<T>(a.x, tid / G, a.pix_per_patch, C, tid % G, cg) + m1;
    const float var = fmaxf(fmaf(-m1, m1, t2 * inv_n), 0.f);
    s_mom[tid * 2] = mean;
    s_mom[tid * 2 + 1] = var;
    a.fresh_out[tid * 2] = mean;
    a.fresh_out[tid * 2 + 1] = var;
  }
  __syncthreads();
  if (tid < NG) {
    const int pp = tid / G, gg = tid % G;
    const int NI = a.per_image, j0 = pp / NI * NI;   // the patches of pp's image
    const int rule = gn_rule(a);
    const float* img = (rule == kGnSync ? s_mom : a.stale) + 2 * (j0 * G + gg);
    const float2 e = gn_estimate(rule, NI, pp - j0, make_float2(s_mom[tid * 2], s_mom[tid * 2 + 1]), img, G);
    a.mean_rstd[tid * 2] = e.x;
    a.mean_rstd[tid * 2 + 1] = 1.f / sqrtf(e.y + a.eps);
  }
  if (tid == 0) *a.counter = 0u;
}

__device__ __forceinline__ float silu_f(float y) { return y / (1.f + expf(-y)); }
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Normalise (+SiLU) one chunk of patch p.  With halo_mode != 0 the output is the
// haloed slab and the kernel also fills the neighbours' halo rows: a patch's
// first row goes to the bottom halo of patch p-1, its last row to the top halo
// of patch p+1 -- this step's values on sync steps (halo_mode 1), the previous
// step's values of the same rows, read from prev_slab, on displaced steps
// (halo_mode 2).  Halo rows at the image top and bottom stay zero.
template <typename T>
__device__ __forceinline__ void write_halos(T* out, const T* prev_slab, const uint4& o, int p, int q,
                                            int pix_per_patch, int last_row0, int W, int C, int c0,
                                            long long stride, long long off, bool top_src, bool bot_src,
                                            int halo_mode) {
  const bool first = top_src && q < W;
  const bool last = bot_src && q >= last_row0;
  if (!first && !last) return;
  const uint4 hv = halo_mode == 1 ? o : ld_nc16(prev_slab + ((size_t)p * stride + off + q) * C + c0);
  if (first)   // bottom halo row (slab row R+1) of patch p-1
    *reinterpret_cast<uint4*>(out + ((size_t)(p - 1) * stride + off + pix_per_patch + q) * C + c0) = hv;
  if (last)    // top halo row (slab row 0) of patch p+1
    *reinterpret_cast<uint4*>(out + ((size_t)(p + 1) * stride + (q - last_row0)) * C + c0) = hv;
}

template <typename T, bool SILU>
__global__ void __launch_bounds__(kGnThreads)
gn_apply_kernel(const T* __restrict__ x, T* __restrict__ out, const T* __restrict__ prev_slab,
                const float* __restrict__ mean_rstd, const float* __restrict__ gamma,
                const float* __restrict__ beta, int G, int pix_per_patch, int C, long long out_patch_stride,
                long long out_off, int pix_per_chunk, int W, int per_image, int halo_mode) {
  constexpr int VEC = VecTraits<T>::kN;
  const int V = C / VEC;
  const int PL = kGnThreads / V;
  const int vc = threadIdx.x % V, pl = threadIdx.x / V;
  if (pl >= PL) return;
  const int p = blockIdx.y, chunk = blockIdx.x;
  // per-channel scale and shift of this thread's channels from the group (mean, rstd)
  float sc[VEC], sf[VEC];
  const int cg = C / G;
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    const int c = vc * VEC + i;
    const float2 mr = reinterpret_cast<const float2*>(mean_rstd)[p * G + c / cg];
    sc[i] = __ldg(gamma + c) * mr.y;
    sf[i] = __ldg(beta + c) - mr.x * sc[i];
  }
  const int pix0 = chunk * pix_per_chunk;
  const int pix1 = min(pix0 + pix_per_chunk, pix_per_patch);
  const T* src = x + (size_t)p * pix_per_patch * C + vc * VEC;
  T* dst = out + ((size_t)p * out_patch_stride + out_off) * C + vc * VEC;
  const int last_row0 = pix_per_patch - W;
  const int pi = p % per_image;                          // patch within its image
  const bool top_src = halo_mode != 0 && pi > 0;         // my first row feeds patch p-1
  const bool bot_src = halo_mode != 0 && pi < per_image - 1;   // my last row feeds patch p+1
  for (int pix = pix0 + pl; pix < pix1; pix += 4 * PL) {
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      u[j] = pix + j * PL < pix1 ? ld_nc16(src + (size_t)(pix + j * PL) * C) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int q = pix + j * PL;
      if (q >= pix1) break;
      float v[VEC];
      unpack16(u[j], v);
#pragma unroll
      for (int i = 0; i < VEC; ++i) {
        v[i] = fmaf(v[i], sc[i], sf[i]);
        if (SILU) v[i] = silu_f(v[i]);
      }
      const uint4 o = pack16(v);
      *reinterpret_cast<uint4*>(dst + (size_t)q * C) = o;
      if (halo_mode != 0) write_halos(out, prev_slab, o, p, q, pix_per_patch, last_row0, W, C, vc * VEC,
                                      out_patch_stride, out_off, top_src, bot_src, halo_mode);
    }
  }
}

// ---------------------------------------------------------------- fused GroupNorm
// Statistics, merge and apply in one cooperative launch (every block resident): each
// block sums its chunk, all blocks meet at a grid barrier, then every block reduces
// the chunk partials of the patches it needs (its own; all of them on sync steps) in
// a fixed order, applies the same merge rule as above and normalises its chunk (the
// map was just read, so the second read is served by L2).  Block (0, p) publishes
// patch p's fresh moments and (mean, rstd).  counter[0] counts arrivals at the
// barrier and counter[1] departures; the last block to leave zeroes both.

// Arrive at the grid barrier: once every thread of the block has finished the writes the
// barrier publishes (the block barrier orders them before thread 0), thread 0 counts the
// block in with a release reduction at GPU scope.  grid_wait() then waits for all blocks
// (an acquire load, so the other blocks' published writes are visible after the block
// barrier); work in between overlaps the wait.
__device__ __forceinline__ void grid_arrive(unsigned* count) {
  __syncthreads();
  if (threadIdx.x == 0) red_release_gpu_add(count, 1u);
}
__device__ __forceinline__ bool grid_wait(unsigned* count, unsigned total, int* err) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire_gpu(count) < total) {
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicCAS(err, 0, kErrGridSync);
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

template <typename T, bool SILU>
__global__ void __launch_bounds__(kGnThreads, 1)
gn_fused_kernel(GnArgs a, GnOut o, int n_chunks, int pix_per_chunk, int* err) {
  constexpr int VEC = VecTraits<T>::kN;
  extern __shared__ float sh[];                 // [2][PL][C] lane sums, then [2][C] channel sums
  __shared__ __align__(16) float s_mr[256 * 2];    // (mean, rstd) of this patch's groups
  __shared__ __align__(16) float s_mom[256 * 2];   // fresh moments (mean, var) of the patches needed
  const int C = a.C, G = a.G;
  const int V = C / VEC;
  const int PL = kGnThreads / V;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vc = tid % V, pl = tid / V;
  const int lp = blockIdx.y, p = a.p0 + lp, chunk = blockIdx.x;   // lp: place in the computed range
  const int pix0 = chunk * pix_per_chunk;
  const int pix1 = min(pix0 + pix_per_chunk, a.pix_per_patch);
  const T* base = static_cast<const T*>(a.x) + (size_t)p * a.pix_per_patch * C + vc * VEC;
  float* chan = sh + 2 * PL * C;
  wait_prior_grid();            // everything below reads or writes buffers of other launches
  allow_next_grid();

  const int last_row0 = a.pix_per_patch - o.W;
  const int NI = a.per_image, pi = p % NI;                 // patch within its image
  const bool top_src = o.halo_mode != 0 && pi > 0;         // my first row feeds patch p-1
  const bool bot_src = o.halo_mode != 0 && pi < NI - 1;    // my last row feeds patch p+1
  // ---- phase 1: per-channel partial sums of x - K (K: the group's shift) over this chunk
  // (8 loads in flight)
  {
    float s1[VEC], s2[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) s1[i] = s2[i] = 0.f;
    if (pl < PL) {
      float k[VEC];
      gn_thread_shifts<T, VEC>(a.x, p, a.pix_per_patch, C, vc * VEC, C / G, k);
      // the chunk is read again after the barrier: ask L2 to keep it; sixteen loads in flight
      // per thread (one block per SM: the map's first read is DRAM latency bound)
      const uint64_t keep = l2_evict_last_policy();
      for (int pix = pix0 + pl; pix < pix1; pix += 16 * PL) {
        uint4 u[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          u[j] = pix + j * PL < pix1 ? ld_nc16_policy(base + (size_t)(pix + j * PL) * C, keep) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (pix + j * PL >= pix1) break;   // past the chunk: a zero would add -K, K^2 to the sums
          float v[VEC];
          unpack16(u[j], v);
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            const float d = v[i] - k[i];
            s1[i] += d;
            s2[i] = fmaf(d, d, s2[i]);
          }
        }
      }
      float4* d1 = reinterpret_cast<float4*>(sh + pl * C + vc * VEC);
      float4* d2 = reinterpret_cast<float4*>(sh + PL * C + pl * C + vc * VEC);
#pragma unroll
      for (int i = 0; i < VEC / 4; ++i) {
        d1[i] = make_float4(s1[4 * i], s1[4 * i + 1], s1[4 * i + 2], s1[4 * i + 3]);
        d2[i] = make_float4(s2[4 * i], s2[4 * i + 1], s2[4 * i + 2], s2[4 * i + 3]);
      }
    }
  }
  __syncthreads();
  for (int c = tid; c < C; c += kGnThreads) {
    float t1 = 0.f, t2 = 0.f;
    for (int l = 0; l < PL; ++l) { t1 += sh[l * C + c]; t2 += sh[PL * C + l * C + c]; }
    chan[c] = t1;
    chan[C + c] = t2;
  }
  __syncthreads();
  const int cg = C / G;
  for (int g = warp; g < G; g += kGnThreads / 32) {
    float t1 = 0.f, t2 = 0.f;
    for (int c = lane; c < cg; c += 32) { t1 += chan[g * cg + c]; t2 += chan[C + g * cg + c]; }
    t1 = warp_sum(t1);
    t2 = warp_sum(t2);
    if (lane == 0) reinterpret_cast<float2*>(a.part)[((size_t)lp * n_chunks + chunk) * G + g] = make_float2(t1, t2);
  }

  // ---- grid barrier: every chunk partial is written
  const unsigned total = gridDim.x * gridDim.y;
  grid_arrive(a.counter);
  // displaced steps: the halo rows are last step's values, final already -- copy them
  // while the other blocks reach the barrier (eight 16-byte loads in flight per thread;
  // only the blocks whose chunk holds a patch's first or last row have any)
  if (o.halo_mode == 2 && pl < PL && ((top_src && pix0 < o.W) || (bot_src && pix1 > last_row0))) {
    T* outp = static_cast<T*>(o.out);
    const T* prev = static_cast<const T*>(o.prev_slab);
    for (int q0 = pix0 + pl; q0 < pix1; q0 += 8 * PL) {
      uint4 hv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = q0 + j * PL;
        const bool need = q < pix1 && ((top_src && q < o.W) || (bot_src && q >= last_row0));
        hv[j] = need ? ld_nc16(prev + ((size_t)p * o.out_patch_stride + o.out_off + q) * C + vc * VEC)
                     : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = q0 + j * PL;
        if (q >= pix1) break;
        if (top_src && q < o.W)   // bottom halo row (slab row R+1) of patch p-1
          *reinterpret_cast<uint4*>(outp + ((size_t)(p - 1) * o.out_patch_stride + o.out_off + a.pix_per_patch + q) *
                                               C + vc * VEC) = hv[j];
        if (bot_src && q >= last_row0)   // top halo row (slab row 0) of patch p+1
          *reinterpret_cast<uint4*>(outp + ((size_t)(p + 1) * o.out_patch_stride + (q - last_row0)) * C + vc * VEC) =
              hv[j];
      }
    }
  }
  if (!grid_wait(a.counter, total, err)) return;

  // ---- phase 2: fresh moments of the patches needed, in a fixed order
  const bool all = gn_rule(a) == kGnSync;       // the sync rule merges the image's fresh moments
  const int p_lo = all ? p - pi : p, np = all ? NI : 1;
  const int items = np * G;                     // <= 256
  const int S = kGnThreads / items;             // threads per item, >= 2
  float* red = sh;                              // [S][items][2]
  if (tid < S * items) {
    const int item = tid % items, part_id = tid / items;
    const int pp = p_lo + item / G - a.p0, gg = item % G;   // place in the computed range
    const float2* src = reinterpret_cast<const float2*>(a.part) + (size_t)pp * n_chunks * G + gg;
    // chunks part_id, part_id + S, ... summed in that order, eight loads in flight (the
    // zeros past the end leave the sum unchanged)
    float2 acc = make_float2(0.f, 0.f);
    for (int c = part_id; c < n_chunks; c += 8 * S) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = c + u * S < n_chunks ? __ldcg(src + (size_t)(c + u * S) * G) : make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) { acc.x += v[u].x; acc.y += v[u].y; }
    }
    red[(part_id * items + item) * 2 + 0] = acc.x;
    red[(part_id * items + item) * 2 + 1] = acc.y;
  }
  __syncthreads();
  const float inv_n = 1.f / ((float)a.pix_per_patch * (float)cg);
  if (tid < items) {
    float t1 = 0.f, t2 = 0.f;
    for (int s2 = 0; s2 < S; ++s2) { t1 += red[(s2 * items + tid) * 2]; t2 += red[(s2 * items + tid) * 2 + 1]; }
    // (mean, var) of patch p_lo + tid / G, group tid % G from the shifted sums
    const float m1 = t1 * inv_n;
    s_mom[tid * 2] = gn_shift<T>(a.x, p_lo + tid / G, a.pix_per_patch, C, tid % G, cg) + m1;
    s_mom[tid * 2 + 1] = fmaxf(fmaf(-m1, m1, t2 * inv_n), 0.f);
  }
  __syncthreads();
  if (tid < G) {
    const int gg = tid;
    const int own = (all ? pi : 0) * G + gg;    // this patch's entry in s_mom
    const float2 mo = make_float2(s_mom[own * 2], s_mom[own * 2 + 1]);
    const int rule = gn_rule(a);
    const float* img = rule == kGnSync ? s_mom + 2 * gg : a.stale + 2 * ((p - pi) * G + gg);
    const float2 e = gn_estimate(rule, NI, pi, mo, img, G);
    const float rstd = 1.f / sqrtf(e.y + a.eps);
    s_mr[gg * 2] = e.x;
    s_mr[gg * 2 + 1] = rstd;
    if (chunk == 0) {
      a.fresh_out[(p * G + gg) * 2] = mo.x;
      a.fresh_out[(p * G + gg) * 2 + 1] = mo.y;
      a.mean_rstd[(p * G + gg) * 2] = e.x;
      a.mean_rstd[(p * G + gg) * 2 + 1] = rstd;
    }
  }
  __syncthreads();

  // ---- phase 3: normalise (+SiLU) this chunk, with the halo rows
  if (pl < PL) {
    float sc[VEC], sf[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      const int c = vc * VEC + i;
      sc[i] = __ldg(a.gamma + c) * s_mr[(c / cg) * 2 + 1];
      sf[i] = __ldg(a.beta + c) - s_mr[(c / cg) * 2] * sc[i];
    }
    T* outp = static_cast<T*>(o.out);
    T* dst = outp + ((size_t)p * o.out_patch_stride + o.out_off) * C + vc * VEC;
    // the last read of the chunk: let L2 drop it first (the output is what the next kernel reads)
    const uint64_t drop = l2_evict_first_policy();
    auto load8 = [&](uint4 (&u)[8], int pix) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        u[j] = pix + j * PL < pix1 ? ld_nc16_policy(base + (size_t)(pix + j * PL) * C, drop) : make_uint4(0, 0, 0, 0);
    };
    auto apply8 = [&](const uint4 (&u)[8], int pix) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = pix + j * PL;
        if (q >= pix1) break;
        float v[VEC];
        unpack16(u[j], v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          v[i] = fmaf(v[i], sc[i], sf[i]);
          // SiLU as v/2 (1 + tanh(v/2)): one MUFU operation for a bf16 output (the approximate
          // tanh, relative error below 2^-10, is finer than the output's rounding); exact for fp32
          if (SILU) {
            if (sizeof(T) == 2) {
              const float hv = 0.5f * v[i];
              v[i] = fmaf(hv, tanh_approx(hv), hv);
            } else {
              v[i] = silu_f(v[i]);
            }
          }
        }
        const uint4 ov = pack16(v);
        *reinterpret_cast<uint4*>(dst + (size_t)q * C) = ov;
        if (o.halo_mode == 1)   // sync steps: this step's boundary rows (displaced: copied above)
          write_halos(outp, static_cast<const T*>(o.prev_slab), ov, p, q, a.pix_per_patch, last_row0, o.W, C,
                      vc * VEC, o.out_patch_stride, o.out_off, top_src, bot_src, o.halo_mode);
      }
    };
    // two batches of eight in flight: the next batch loads while this one is written
    uint4 ua[8], ub[8];
    load8(ua, pix0 + pl);
    for (int pix = pix0 + pl; pix < pix1; pix += 16 * PL) {
      load8(ub, pix + 8 * PL);
      apply8(ua, pix);
      load8(ua, pix + 16 * PL);
      apply8(ub, pix + 8 * PL);
    }
  }
  // ---- departure: the last block out re-arms the barrier for the next launch
  if (tid == 0 && atomicAdd(a.counter + 1, 1u) == total - 1) {
    a.counter[0] = 0u;
    a.counter[1] = 0u;
  }
}

// ---------------------------------------------------------------- streamed GroupNorm (bf16)
// The fused GroupNorm with its two passes over the chunk moved by the copy engine.  A copy
// warp streams the chunk (contiguous: pixels [pix0, pix1) of patch p, all channels) through
// a ring of kGsStages shared-memory stages with untiled bulk copies completing on `full`
// mbarriers; the 16 compute warps only read shared memory and release each stage with one
// arrival per warp on its `empty` mbarrier, so neither side waits for the other except on
// the stage it needs.  Statistics pass: the stages are summed as in gn_fused_kernel (the
// same shifts, the same fixed per-thread pixel order, so the same partial sums).  Apply
// pass: the copy warp requests its first stages as soon as first-pass slots free up (the
// reads do not depend on the grid barrier); the compute warps normalise each stage in place,
// and the copy warp writes it back with a bulk store (plus, on sync steps, the rows that are a
// neighbour's halo) before it reuses the slot.  The first pass's copies ask L2 to keep the
// lines (the chunk is read again), the second's to drop them first.
constexpr int kGsStages = 4;
constexpr int kGsStageBytes = 40960;
constexpr int kGsThreads = kGnThreads + 32;   // 16 compute warps and the copy warp

// stage size: kGsStageBytes, less for very wide maps so that the ring and the partial sums
// stay within 192 KB of dynamic shared memory
size_t gs_sums_bytes(int C) { return (size_t)(2 * (kGnThreads / (C / 8)) + 2) * C * sizeof(float); }
int gs_stage_pixels(int C) {
  const long long room = (196608ll - (long long)gs_sums_bytes(C)) / kGsStages;
  return (int)std::max(1ll, std::min<long long>(kGsStageBytes, room) / (C * 2));
}
size_t gs_smem_bytes(int C) { return (size_t)kGsStages * gs_stage_pixels(C) * C * 2 + gs_sums_bytes(C); }

// barrier over the compute warps only (the copy warp runs its own loop)
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kGnThreads) : "memory"); }
__device__ __forceinline__ void grid_arrive_c(unsigned* count) {
  compute_sync();
  if (threadIdx.x == 0) red_release_gpu_add(count, 1u);
}
__device__ __forceinline__ bool grid_wait_c(unsigned* count, unsigned total, int* err) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    int ok = 1;
    const long long t0 = clock64();
    while (ld_acquire_gpu(count) < total) {
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicCAS(err, 0, kErrGridSync);
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    s_ok = ok;
  }
  compute_sync();
  return s_ok != 0;
}

template <bool SILU>
__global__ void __launch_bounds__(kGsThreads, 1)
gn_stream_kernel(GnArgs a, GnOut o, int n_chunks, int pix_per_chunk, int stage_pix, int* err) {
  using T = __nv_bfloat16;
  constexpr int VEC = 8;
  constexpr int S = kGsStages;
  extern __shared__ __align__(128) uint8_t gs_smem[];
  __shared__ __align__(8) uint64_t full[S], empty[S];
  __shared__ __align__(16) float s_mr[256 * 2];    // (mean, rstd) of this patch's groups
  __shared__ __align__(16) float s_mom[256 * 2];   // fresh moments (mean, var) of the patches needed
  __shared__ float s_shift[256];                   // their shifts K
  __shared__ __align__(16) float s_stale[256 * 2]; // previous step's moments of the image's patches
  const int C = a.C, G = a.G;
  const int V = C / VEC;
  const int PL = kGnThreads / V;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vc = tid % V, pl = tid / V;
  const int lp = blockIdx.y, p = a.p0 + lp, chunk = blockIdx.x;
  const int pix0 = chunk * pix_per_chunk;
  const int pix1 = min(pix0 + pix_per_chunk, a.pix_per_patch);
  const int nst = (pix1 - pix0 + stage_pix - 1) / stage_pix;   // stages of the chunk
  const size_t stage_elems = (size_t)stage_pix * C;
  T* ring = reinterpret_cast<T*>(gs_smem);
  float* sh = reinterpret_cast<float*>(gs_smem + (size_t)S * stage_elems * sizeof(T));
  float* chan = sh + 2 * PL * C;
  const T* src = static_cast<const T*>(a.x) + (size_t)p * a.pix_per_patch * C;
  const int last_row0 = a.pix_per_patch - o.W;
  const int NI = a.per_image, pi = p % NI;                 // patch within its image
  const bool top_src = o.halo_mode != 0 && pi > 0;         // my first row feeds patch p-1
  const bool bot_src = o.halo_mode != 0 && pi < NI - 1;    // my last row feeds patch p+1

  if (tid == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), kGnThreads / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  wait_prior_grid();            // everything below reads or writes buffers of other launches
  allow_next_grid();

  if (warp == kGnThreads / 32) {
    // ------------------------------------------------------------ copy warp
    if (lane == 0) {
      const uint64_t keep = l2_evict_last_policy(), drop = l2_evict_first_policy();
      T* outp = static_cast<T*>(o.out);
      // load number L: stage L of the first pass, stage L - nst of the second, into slot L % S
      auto issue = [&](int L) {
        const int k = L < nst ? L : L - nst;
        const int s0 = pix0 + k * stage_pix, n = min(stage_pix, pix1 - s0);
        const uint32_t bytes = (uint32_t)n * C * 2, bar = smem_u32(&full[L % S]);
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load_policy(smem_u32(ring + (size_t)(L % S) * stage_elems), src + (size_t)s0 * C, bytes, bar,
                         L < nst ? keep : drop);
      };
      // the normalised second-pass stage of load L back to the output (and the halo rows)
      auto store = [&](int L) {
        const int k = L - nst;
        const int s0 = pix0 + k * stage_pix, n = min(stage_pix, pix1 - s0);
        const uint32_t sa = smem_u32(ring + (size_t)(L % S) * stage_elems);
        bulk_store(outp + ((size_t)p * o.out_patch_stride + o.out_off + s0) * C, sa, (uint32_t)n * C * 2);
        if (o.halo_mode == 1) {
          // sync steps: this step's boundary rows are also the neighbours' halo rows
          if (top_src && s0 < o.W) {
            const int e = min(s0 + n, o.W);
            bulk_store(outp + ((size_t)(p - 1) * o.out_patch_stride + o.out_off + a.pix_per_patch + s0) * C, sa,
                       (uint32_t)(e - s0) * C * 2);
          }
          if (bot_src && s0 + n > last_row0) {
            const int b = max(s0, last_row0);
            bulk_store(outp + ((size_t)(p + 1) * o.out_patch_stride + (b - last_row0)) * C,
                       sa + (uint32_t)(b - s0) * C * 2, (uint32_t)(s0 + n - b) * C * 2);
          }
        }
        bulk_commit();
      };
      // the slot of load L is free once its previous occupant (load L - S) is released by the
      // compute warps and, for a second-pass stage, stored and read out by the copy engine
      bool ok = true;
      int issued = 0;
      for (int L = 0; L < 2 * nst; ++L) {
        if (L >= S) {
          const int occ = L - S;
          ok = mbar_wait(smem_u32(&empty[occ % S]), (uint32_t)(occ / S) & 1u, err, kErrWaitStageFree);
          if (!ok) break;
          if (occ >= nst) {
            store(occ);
            bulk_wait_read_all();
          }
        }
        issue(L);
        issued = L + 1;
      }
      // the second-pass stages no later load displaces
      for (int occ = max(nst, 2 * nst - S); ok && occ < 2 * nst; ++occ) {
        ok = mbar_wait(smem_u32(&empty[occ % S]), (uint32_t)(occ / S) & 1u, err, kErrWaitStageFree);
        if (ok) store(occ);
      }
      // the block's shared memory must outlive the stores' reads of it; their writes complete
      // with the grid, before any later launch that waits for it reads them
      bulk_wait_read_all();
      if (!ok) {
        // a wait gave up: let the loads still in flight land before the block exits (the last
        // load issued into each slot; the earlier ones of a slot completed before it)
        for (int L = max(0, issued - S); L < issued; ++L)
          mbar_wait(smem_u32(&full[L % S]), (uint32_t)(L / S) & 1u, err, kErrWaitTmaFull);
      }
    }
    return;
  }

  // ------------------------------------------------------------ compute warps (512 threads)
  // a failed wait ends this thread's work (the code is in err); arrivals continue, so the
  // copy warp is never left waiting on a warp that gave up
  auto ready = [&](int L) { return mbar_wait(smem_u32(&full[L % S]), (uint32_t)(L / S) & 1u, err, kErrWaitTmaFull); };
  auto release = [&](int L) {
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[L % S]));
  };
  bool ok = true;
  // ---- pass 1: per-channel partial sums of x - K (K: the group's shift) over this chunk
  {
    float s1[VEC], s2[VEC], k[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) s1[i] = s2[i] = 0.f;
    if (pl < PL) gn_thread_shifts<T, VEC>(a.x, p, a.pix_per_patch, C, vc * VEC, C / G, k);
    for (int L = 0; L < nst; ++L) {
      ok = ok && ready(L);
      const T* st = ring + (size_t)(L % S) * stage_elems;
      const int n = min(stage_pix, pix1 - (pix0 + L * stage_pix));
      if (ok && pl < PL) {
        for (int q = pl; q < n; q += PL) {
          float v[VEC];
          unpack16(*reinterpret_cast<const uint4*>(st + (size_t)q * C + vc * VEC), v);
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            const float d = v[i] - k[i];
            s1[i] += d;
            s2[i] = fmaf(d, d, s2[i]);
          }
        }
      }
      release(L);
    }
    if (pl < PL) {
      float4* d1 = reinterpret_cast<float4*>(sh + pl * C + vc * VEC);
      float4* d2 = reinterpret_cast<float4*>(sh + PL * C + pl * C + vc * VEC);
#pragma unroll
      for (int i = 0; i < VEC / 4; ++i) {
        d1[i] = make_float4(s1[4 * i], s1[4 * i + 1], s1[4 * i + 2], s1[4 * i + 3]);
        d2[i] = make_float4(s2[4 * i], s2[4 * i + 1], s2[4 * i + 2], s2[4 * i + 3]);
      }
    }
  }
  compute_sync();
  for (int c = tid; c < C; c += kGnThreads) {
    float t1 = 0.f, t2 = 0.f;
    for (int l = 0; l < PL; ++l) { t1 += sh[l * C + c]; t2 += sh[PL * C + l * C + c]; }
    chan[c] = t1;
    chan[C + c] = t2;
  }
  compute_sync();
  const int cg = C / G;
  for (int g = warp; g < G; g += kGnThreads / 32) {
    float t1 = 0.f, t2 = 0.f;
    for (int c = lane; c < cg; c += 32) { t1 += chan[g * cg + c]; t2 += chan[C + g * cg + c]; }
    t1 = warp_sum(t1);
    t2 = warp_sum(t2);
    if (lane == 0) reinterpret_cast<float2*>(a.part)[((size_t)lp * n_chunks + chunk) * G + g] = make_float2(t1, t2);
  }
  // this thread's gamma and beta (read while the other blocks finish)
  float gm[VEC], bt[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    gm[i] = pl < PL ? __ldg(a.gamma + vc * VEC + i) : 0.f;
    bt[i] = pl < PL ? __ldg(a.beta + vc * VEC + i) : 0.f;
  }
  const int rule = gn_rule(a);
  const bool all = rule == kGnSync;             // the sync rule merges the image's fresh moments
  const int p_lo = all ? p - pi : p, np = all ? NI : 1;
  const int items = np * G;                     // <= 256

  // ---- grid barrier: every chunk partial is written
  const unsigned total = gridDim.x * gridDim.y;
  grid_arrive_c(a.counter);
  // the merge's other inputs, read while the other blocks reach the barrier
  if (tid < items) s_shift[tid] = gn_shift<T>(a.x, p_lo + tid / G, a.pix_per_patch, C, tid % G, cg);
  if (rule == kGnCorrected || rule == kGnStaleOthers)
    for (int i = tid; i < NI * G * 2; i += kGnThreads) s_stale[i] = a.stale[(size_t)(p - pi) * G * 2 + i];
  // displaced steps: the halo rows are last step's values, final already -- copy them
  // while the other blocks reach the barrier
  if (o.halo_mode == 2 && pl < PL && ((top_src && pix0 < o.W) || (bot_src && pix1 > last_row0))) {
    T* outp = static_cast<T*>(o.out);
    const T* prev = static_cast<const T*>(o.prev_slab);
    for (int q0 = pix0 + pl; q0 < pix1; q0 += 8 * PL) {
      uint4 hv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = q0 + j * PL;
        const bool need = q < pix1 && ((top_src && q < o.W) || (bot_src && q >= last_row0));
        hv[j] = need ? ld_nc16(prev + ((size_t)p * o.out_patch_stride + o.out_off + q) * C + vc * VEC)
                     : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int q = q0 + j * PL;
        if (q >= pix1) break;
        if (top_src && q < o.W)
          *reinterpret_cast<uint4*>(outp + ((size_t)(p - 1) * o.out_patch_stride + o.out_off + a.pix_per_patch + q) *
                                               C + vc * VEC) = hv[j];
        if (bot_src && q >= last_row0)
          *reinterpret_cast<uint4*>(outp + ((size_t)(p + 1) * o.out_patch_stride + (q - last_row0)) * C + vc * VEC) =
              hv[j];
      }
    }
  }
  if (!grid_wait_c(a.counter, total, err)) ok = false;

  // ---- merge: fresh moments of the patches needed, in a fixed order
  const int SP = kGnThreads / items;            // threads per item, >= 2
  float* red = sh;                              // [SP][items][2]
  if (ok && tid < SP * items) {
    const int item = tid % items, part_id = tid / items;
    const int pp = p_lo + item / G - a.p0, gg = item % G;
    const float2* srcp = reinterpret_cast<const float2*>(a.part) + (size_t)pp * n_chunks * G + gg;
    float2 acc = make_float2(0.f, 0.f);
    for (int c = part_id; c < n_chunks; c += 8 * SP) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = c + u * SP < n_chunks ? __ldcg(srcp + (size_t)(c + u * SP) * G) : make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) { acc.x += v[u].x; acc.y += v[u].y; }
    }
    red[(part_id * items + item) * 2 + 0] = acc.x;
    red[(part_id * items + item) * 2 + 1] = acc.y;
  }
  compute_sync();
  const float inv_n = 1.f / ((float)a.pix_per_patch * (float)cg);
  if (ok && tid < items) {
    float t1 = 0.f, t2 = 0.f;
    for (int s2 = 0; s2 < SP; ++s2) { t1 += red[(s2 * items + tid) * 2]; t2 += red[(s2 * items + tid) * 2 + 1]; }
    const float m1 = t1 * inv_n;
    s_mom[tid * 2] = s_shift[tid] + m1;
    s_mom[tid * 2 + 1] = fmaxf(fmaf(-m1, m1, t2 * inv_n), 0.f);
  }
  compute_sync();
  if (ok && tid < G) {
    const int gg = tid;
    const int own = (all ? pi : 0) * G + gg;
    const float2 mo = make_float2(s_mom[own * 2], s_mom[own * 2 + 1]);
    const float* img = (rule == kGnSync ? s_mom : s_stale) + 2 * gg;
    const float2 e = gn_estimate(rule, NI, pi, mo, img, G);
    const float rstd = 1.f / sqrtf(e.y + a.eps);
    s_mr[gg * 2] = e.x;
    s_mr[gg * 2 + 1] = rstd;
    if (chunk == 0) {
      a.fresh_out[(p * G + gg) * 2] = mo.x;
      a.fresh_out[(p * G + gg) * 2 + 1] = mo.y;
      a.mean_rstd[(p * G + gg) * 2] = e.x;
      a.mean_rstd[(p * G + gg) * 2 + 1] = rstd;
    }
  }
  compute_sync();

  // ---- pass 2: normalise (+SiLU) each stage in place; the copy warp stores it back
  float scl[VEC], sft[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    const int c = vc * VEC + i;
    scl[i] = gm[i] * s_mr[(c / cg) * 2 + 1];
    sft[i] = bt[i] - s_mr[(c / cg) * 2] * scl[i];
  }
  for (int k = 0; k < nst; ++k) {
    const int L = nst + k;
    ok = ok && ready(L);
    T* st = ring + (size_t)(L % S) * stage_elems;
    const int n = min(stage_pix, pix1 - (pix0 + k * stage_pix));
    if (ok && pl < PL) {
      for (int q = pl; q < n; q += PL) {
        uint4* cell = reinterpret_cast<uint4*>(st + (size_t)q * C + vc * VEC);
        float v[VEC];
        unpack16(*cell, v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
          v[i] = fmaf(v[i], scl[i], sft[i]);
          if (SILU) {
            // SiLU as v/2 (1 + tanh(v/2)): one MUFU operation (the approximate tanh, relative
            // error below 2^-10, is finer than the bf16 output's rounding)
            const float hv = 0.5f * v[i];
            v[i] = fmaf(hv, tanh_approx(hv), hv);
          }
        }
        *cell = pack16(v);
      }
    }
    fence_proxy_async_smem();   // this thread's writes, before the copy engine reads them
    release(L);
  }
  // ---- departure: the last block out re-arms the barrier for the next launch
  if (tid == 0 && atomicAdd(a.counter + 1, 1u) == total - 1) {
    a.counter[0] = 0u;
    a.counter[1] = 0u;
  }
}

// Pixels per block: one wave of 512-thread blocks over the whole map.
// Per-token LayerNorm (transformer blocks of the SDXL-style stage): one warp per
// token, the token's C channels held in registers (NV 16-byte vectors per lane, NV
// fixed at compile time so nothing is masked), mean and biased variance by warp
// butterflies (deterministic, two passes over the registers), fp32 math, bf16 in/out.
template <int NV>
__global__ void __launch_bounds__(256)
layernorm_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                 const float* __restrict__ gamma, const float* __restrict__ beta, int L, int C, float eps) {
  const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  wait_prior_grid();
  allow_next_grid();
  if (tok >= L) return;
  const int nvec = C / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)tok * C);
  uint4 u[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = lane + 32 * k;
    u[k] = i < nvec ? ld_nc16(src + i) : make_uint4(0, 0, 0, 0);
  }
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    float v[8];
    unpack16(u[k], v);
#pragma unroll
    for (int e = 0; e < 8; ++e) s += v[e];
  }
  const float mean = warp_sum(s) / (float)C;
  float q = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    if (lane + 32 * k < nvec) {
      float v[8];
      unpack16(u[k], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) { const float d = v[e] - mean; q = fmaf(d, d, q); }
    }
  }
  const float rstd = 1.f / sqrtf(warp_sum(q) / (float)C + eps);
  uint4* dst = reinterpret_cast<uint4*>(y + (size_t)tok * C);
  const float4* g4 = reinterpret_cast<const float4*>(gamma);
  const float4* b4 = reinterpret_cast<const float4*>(beta);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = lane + 32 * k;
    if (i < nvec) {
      float v[8];
      unpack16(u[k], v);
      const float4 ga = __ldg(g4 + 2 * i), gb = __ldg(g4 + 2 * i + 1);
      const float4 ba = __ldg(b4 + 2 * i), bb = __ldg(b4 + 2 * i + 1);
      const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
      const float bt[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = fmaf((v[e] - mean) * rstd, gg[e], bt[e]);
      dst[i] = pack16(o);
    }
  }
}

int chunk_pixels(int N, int pix_per_patch) {
  const int target_blocks = 148;
  int per = (N * pix_per_patch + target_blocks - 1) / target_blocks;
  if (per < 16) per = 16;
  return per;
}

}  // namespace

int gn_stats_chunks(int N, int pix_per_patch) {
  const int per = chunk_pixels(N, pix_per_patch);
  return (pix_per_patch + per - 1) / per;
}

size_t gn_part_floats(int N, int pix_per_patch, int G) {
  size_t most = 0;
  for (int n = 1; n <= N; ++n) most = std::max(most, (size_t)n * gn_stats_chunks(n, pix_per_patch));
  return most * G * 2;
}

template <typename T>
cudaError_t launch_gn_stats_merge(const GnArgs& a, cudaStream_t s) {
  constexpr int VEC = VecTraits<T>::kN;
  const int per = chunk_pixels(a.N, a.pix_per_patch);
  const int n_chunks = (a.pix_per_patch + per - 1) / per;
  const int V = a.C / VEC;
  const int PL = kGnThreads / V;
  size_t smem = (size_t)(2 * PL + 2) * a.C * sizeof(float);
  const size_t red = (size_t)kGnThreads * 2 * sizeof(float);
  if (smem < red) smem = red;
  dim3 grid(n_chunks, a.N);
  // wide maps (bf16 C > 3072: one pixel lane of 16 C floats) need more than the default 48 KiB
  cudaError_t e = cudaFuncSetAttribute(gn_stats_merge_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gn_stats_merge_kernel<T><<<grid, kGnThreads, smem, s>>>(a, n_chunks, per);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gn_apply(const T* x, T* out, const T* prev_slab, const float* mean_rstd, const float* gamma,
                            const float* beta, int G, int N, int per_image, int pix_per_patch, int C, int W,
                            long long out_patch_stride_pix, long long out_pix_off, bool silu, int halo_mode,
                            cudaStream_t s) {
  const int per = chunk_pixels(N, pix_per_patch);
  dim3 grid((pix_per_patch + per - 1) / per, N);
  if (silu)
    gn_apply_kernel<T, true><<<grid, kGnThreads, 0, s>>>(x, out, prev_slab, mean_rstd, gamma, beta, G,
                                                         pix_per_patch, C, out_patch_stride_pix, out_pix_off,
                                                         per, W, per_image, halo_mode);
  else
    gn_apply_kernel<T, false><<<grid, kGnThreads, 0, s>>>(x, out, prev_slab, mean_rstd, gamma, beta, G,
                                                          pix_per_patch, C, out_patch_stride_pix, out_pix_off,
                                                          per, W, per_image, halo_mode);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gn_fused(const GnArgs& a, const GnOut& o, bool silu, int* err, cudaStream_t s) {
  constexpr int VEC = VecTraits<T>::kN;
  constexpr bool kStream = sizeof(T) == 2;   // bf16: the streamed kernel
  const int V = a.C / VEC;
  const int PL = kGnThreads / V;
  size_t smem = kStream ? gs_smem_bytes(a.C) : (size_t)(2 * PL + 2) * a.C * sizeof(float);
  const size_t red = (size_t)kGnThreads * 2 * sizeof(float);
  if (smem < red) smem = red;
  using Kern = void (*)(GnArgs, GnOut, int, int, int*);
  using SKern = void (*)(GnArgs, GnOut, int, int, int, int*);
  // bf16 takes the streamed kernel, fp32 the register-streaming one (only one is instantiated)
  Kern kern = nullptr;
  SKern skern = nullptr;
  if constexpr (kStream) skern = silu ? gn_stream_kernel<true> : gn_stream_kernel<false>;
  else kern = silu ? gn_fused_kernel<T, true> : gn_fused_kernel<T, false>;
  const void* kfn = kStream ? reinterpret_cast<const void*>(skern) : reinterpret_cast<const void*>(kern);
  // every block must be resident at once (the grid barrier): at most the occupancy
  // limit, and no more chunks than the partial-sum scratch holds
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  const int threads = kStream ? kGsThreads : kGnThreads;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, threads, smem);
  if (e != cudaSuccess) return e;
  const int max_blocks = per_sm * sm_count();
  const int n_run = a.n_run > 0 ? a.n_run : a.N;   // patches computed
  if (a.p0 < 0 || a.p0 + n_run > a.N) return cudaErrorInvalidValue;
  // the sync rule merges every patch of an image from this launch's partial sums
  const bool all = !a.naive && (a.is_sync || a.mode == 2);
  if (all && n_run != a.N) return cudaErrorInvalidValue;
  if (n_run > max_blocks) return cudaErrorCooperativeLaunchTooLarge;
  int n_chunks = std::min(gn_stats_chunks(n_run, a.pix_per_patch), max_blocks / n_run);
  const int per = (a.pix_per_patch + n_chunks - 1) / n_chunks;
  n_chunks = (a.pix_per_patch + per - 1) / per;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n_chunks, n_run);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;   // every block resident: the grid barrier cannot starve
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  const int stage_pix = gs_stage_pixels(a.C);
  auto go = [&]() {
    if constexpr (kStream) return cudaLaunchKernelEx(&cfg, skern, a, o, n_chunks, per, stage_pix, err);
    else return cudaLaunchKernelEx(&cfg, kern, a, o, n_chunks, per, err);
  };
  e = go();
  if (e != cudaSuccess && a.pdl) {
    // a runtime that does not take both attributes together: launch it plainly
    cudaGetLastError();
    cfg.numAttrs = 1;
    e = go();
  }
  return e;
}


cudaError_t launch_layernorm(const void* x, void* y, const float* gamma, const float* beta, int L, int C,
                             float eps, bool pdl, cudaStream_t s) {
  if (C % 8 || C > 2048) return cudaErrorInvalidValue;
  const auto* xi = static_cast<const __nv_bfloat16*>(x);
  auto* yo = static_cast<__nv_bfloat16*>(y);
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((L + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  switch ((C / 8 + 31) / 32) {   // 16-byte vectors per lane
    case 1: return cudaLaunchKernelEx(&cfg, layernorm_kernel<1>, xi, yo, gamma, beta, L, C, eps);
    case 2: return cudaLaunchKernelEx(&cfg, layernorm_kernel<2>, xi, yo, gamma, beta, L, C, eps);
    case 3: return cudaLaunchKernelEx(&cfg, layernorm_kernel<3>, xi, yo, gamma, beta, L, C, eps);
    case 4: return cudaLaunchKernelEx(&cfg, layernorm_kernel<4>, xi, yo, gamma, beta, L, C, eps);
    case 5: return cudaLaunchKernelEx(&cfg, layernorm_kernel<5>, xi, yo, gamma, beta, L, C, eps);
    case 6: return cudaLaunchKernelEx(&cfg, layernorm_kernel<6>, xi, yo, gamma, beta, L, C, eps);
    case 7: return cudaLaunchKernelEx(&cfg, layernorm_kernel<7>, xi, yo, gamma, beta, L, C, eps);
    default: return cudaLaunchKernelEx(&cfg, layernorm_kernel<8>, xi, yo, gamma, beta, L, C, eps);
  }
}

template cudaError_t launch_gn_stats_merge<float>(const GnArgs&, cudaStream_t);
template cudaError_t launch_gn_stats_merge<__nv_bfloat16>(const GnArgs&, cudaStream_t);
template cudaError_t launch_gn_apply<float>(const float*, float*, const float*, const float*, const float*,
                                            const float*, int, int, int, int, int, int, long long,
                                            long long, bool, int, cudaStream_t);
template cudaError_t launch_gn_apply<__nv_bfloat16>(const __nv_bfloat16*, __nv_bfloat16*,
                                                    const __nv_bfloat16*, const float*, const float*,
                                                    const float*, int, int, int, int, int, int,
                                                    long long, long long, bool, int, cudaStream_t);
template cudaError_t launch_gn_fused<float>(const GnArgs&, const GnOut&, bool, int*, cudaStream_t);
template cudaError_t launch_gn_fused<__nv_bfloat16>(const GnArgs&, const GnOut&, bool, int*, cudaStream_t);

}  // namespace dfp
