// Small kernels of the multi-level UNet (DFP_BLOCK_UNET): the haloed conv input slab
// filled from a map (plain or upsampled x2), channel concatenation of the skips, the
// timestep MLP and the DDIM update.  All move little data next to the convolutions and
// attention of a UNet evaluation; they are plain vectorised CUDA-core kernels.
#include <cuda_bf16.h>

#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

using bf = __nv_bfloat16;

// One 16-byte vector (8 channels from c8) of pixel (row, col) of the source map, as the
// conv input sees it: the map itself, or (up) the map at half resolution repeated 2 x 2;
// channels at or past src_C read as zero (a narrow input padded to the conv's width).
__device__ __forceinline__ uint4 src_vec(const bf* src, int src_C, int W, int row, int col, int c8, bool up) {
  const int sw = up ? W / 2 : W;
  const long long pix = up ? (long long)(row / 2) * sw + col / 2 : (long long)row * sw + col;
  const bf* p = src + pix * src_C + c8;
  if (c8 + 8 <= src_C && (src_C % 8) == 0) return ld_nc16(p);
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = c8 + e < src_C ? __bfloat162float(p[e]) : 0.f;
  return pack16(v);
}

// slab [N][R+2][W][C] (one halo row above and below each patch).  Interior rows come from
// the source map; halo rows (halo_mode 1: this step's neighbour rows from the source;
// 2: the previous step's, from the neighbour's interior rows of prev_slab; 0: none) are
// written for patches with a neighbour, image-edge halos keep their zeros.
template <bool UP>
__global__ void slab_fill_kernel(const bf* __restrict__ src, int src_C, bf* __restrict__ slab,
                                 const bf* __restrict__ prev_slab, int C, int N, int R, int W, int halo_mode) {
  wait_prior_grid();
  allow_next_grid();
  const int V = C / 8;
  const long long total = (long long)N * (R + 2) * W * V;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int v = (int)(i % V);
    long long t = i / V;
    const int col = (int)(t % W);
    t /= W;
    const int sr = (int)(t % (R + 2));     // slab row of patch p
    const int p = (int)(t / (R + 2));
    uint4 val;
    if (sr >= 1 && sr <= R) {
      val = src_vec(src, src_C, W, p * R + sr - 1, col, 8 * v, UP);
    } else {
      const bool top = sr == 0;
      if (halo_mode == 0 || (top && p == 0) || (!top && p == N - 1)) continue;
      if (halo_mode == 1) {
        val = src_vec(src, src_C, W, top ? p * R - 1 : (p + 1) * R, col, 8 * v, UP);
      } else {
        // the neighbour's boundary row of the previous step: last row of p-1 / first row of p+1
        const long long nr = top ? (long long)(p - 1) * (R + 2) + R : (long long)(p + 1) * (R + 2) + 1;
        val = ld_nc16(prev_slab + (nr * W + col) * C + 8 * v);
      }
    }
    *reinterpret_cast<uint4*>(slab + (((long long)p * (R + 2) + sr) * W + col) * C + 8 * v) = val;
  }
}

// out[l] = [a[l] | b[l]]  (channels of a, then of b)
__global__ void concat_kernel(const bf* __restrict__ a, int Ca, const bf* __restrict__ b, int Cb,
                              bf* __restrict__ out, long long L) {
  wait_prior_grid();
  allow_next_grid();
  const int Va = Ca / 8, V = (Ca + Cb) / 8;
  const long long total = L * V;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long l = i / V;
    const int v = (int)(i - l * V);
    const uint4 x = v < Va ? ld_nc16(a + l * Ca + 8 * v) : ld_nc16(b + l * Cb + 8 * (v - Va));
    *reinterpret_cast<uint4*>(out + l * (Ca + Cb) + 8 * v) = x;
  }
}

__device__ __forceinline__ float silu_exact(float y) { return y / (1.f + expf(-y)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// y[r] = act(W[r] . x + b[r] (+ add[r])), one warp per output row; fp32 weights [rows][cols].
// x_tau >= 0: x is the sinusoidal embedding of the timestep, [cos(tau f_k), sin(tau f_k)],
// f_k = 10000^(-k / (cols/2)), computed here instead of read.
__device__ __forceinline__ float gemv_x(const float* x, float x_tau, int c, int half) {
  if (x_tau < 0.f) return x[c];
  const int k = c < half ? c : c - half;
  const float f = expf(-9.210340371976184f * (float)k / (float)half);   // ln(10000) = 9.2103...
  return c < half ? cosf(x_tau * f) : sinf(x_tau * f);
}

// VEC4: cols % 4 == 0 and 16-byte aligned rows: each lane reads 16-byte vectors of the row,
// four of them in flight (a row of 1280 weights is ten vectors a lane).
template <bool VEC4>
__global__ void gemv_kernel(const float* __restrict__ Wt, const float* __restrict__ b,
                            const float* __restrict__ add, const float* __restrict__ x, float x_tau,
                            float* __restrict__ y, int rows, int cols, int silu_out) {
  wait_prior_grid();
  allow_next_grid();
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float* w = Wt + (size_t)r * cols;
  const int half = cols / 2;
  float s = 0.f;
  if (VEC4) {
    const float4* w4 = reinterpret_cast<const float4*>(w);
    const int n4 = cols / 4;
#pragma unroll 4
    for (int c4 = lane; c4 < n4; c4 += 32) {
      const float4 wv = __ldg(w4 + c4);
      const int c = 4 * c4;
      s = fmaf(wv.x, gemv_x(x, x_tau, c, half), s);
      s = fmaf(wv.y, gemv_x(x, x_tau, c + 1, half), s);
      s = fmaf(wv.z, gemv_x(x, x_tau, c + 2, half), s);
      s = fmaf(wv.w, gemv_x(x, x_tau, c + 3, half), s);
    }
  } else {
    for (int c = lane; c < cols; c += 32) s = fmaf(__ldg(w + c), gemv_x(x, x_tau, c, half), s);
  }
  s = warp_sum(s);
  if (lane == 0) {
    float v = s + b[r] + (add ? add[r] : 0.f);
    y[r] = silu_out ? silu_exact(v) : v;
  }
}

// Several y_s = W_s x + b_s (+ add_s) over the same x in one launch (the ResNets' time
// projections): the warps of the grid take the segments' rows one after another.
__global__ void gemv_multi_kernel(const GemvBatch batch, const float* __restrict__ x, int cols) {
  wait_prior_grid();
  allow_next_grid();
  int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  int sgi = 0;
  while (sgi < batch.n && r >= batch.seg[sgi].rows) r -= batch.seg[sgi++].rows;
  if (sgi >= batch.n) return;
  const GemvSeg& sg = batch.seg[sgi];
  const float4* w4 = reinterpret_cast<const float4*>(sg.W + (size_t)r * cols);
  const float4* x4 = reinterpret_cast<const float4*>(x);
  float s = 0.f;
#pragma unroll 4
  for (int c4 = lane; c4 < cols / 4; c4 += 32) {
    const float4 wv = __ldg(w4 + c4), xv = __ldg(x4 + c4);
    s = fmaf(wv.x, xv.x, s);
    s = fmaf(wv.y, xv.y, s);
    s = fmaf(wv.z, xv.z, s);
    s = fmaf(wv.w, xv.w, s);
  }
  s = warp_sum(s);
  if (lane == 0) sg.y[r] = s + sg.b[r] + (sg.add ? sg.add[r] : 0.f);
}

// DDIM (eta = 0): lat = c1 * lat + c2 * eps over [L][4]; x_bf = bf16(lat) for the next UNet.
__global__ void ddim_update_kernel(float* __restrict__ lat, const bf* __restrict__ eps, bf* __restrict__ x_bf,
                                   long long n, float c1, float c2) {
  wait_prior_grid();
  allow_next_grid();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = fmaf(c1, lat[i], c2 * __bfloat162float(eps[i]));
    lat[i] = v;
    x_bf[i] = __float2bfloat16_rn(v);
  }
}

__global__ void to_bf16_kernel(const float* __restrict__ a, bf* __restrict__ b, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    b[i] = __float2bfloat16_rn(a[i]);
}

template <typename K, typename... Args>
cudaError_t launch_pdl(K kern, int blocks, int threads, bool pdl, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

int grid_for(long long items) {
  const long long b = (items + 255) / 256;
  return (int)(b < 8 * 148 ? (b < 1 ? 1 : b) : 8 * 148);
}

}  // namespace

cudaError_t launch_slab_fill(const void* src, int src_C, void* slab, const void* prev_slab, int C, int N, int R,
                             int W, int halo_mode, bool upsample, bool pdl, cudaStream_t s) {
  if (C % 8) return cudaErrorInvalidValue;
  const long long items = (long long)N * (R + 2) * W * (C / 8);
  auto k = upsample ? slab_fill_kernel<true> : slab_fill_kernel<false>;
  return launch_pdl(k, grid_for(items), 256, pdl, s, static_cast<const bf*>(src), src_C, static_cast<bf*>(slab),
                    static_cast<const bf*>(prev_slab), C, N, R, W, halo_mode);
}

cudaError_t launch_concat(const void* a, int Ca, const void* b, int Cb, void* out, long long L, bool pdl,
                          cudaStream_t s) {
  if (Ca % 8 || Cb % 8) return cudaErrorInvalidValue;
  return launch_pdl(concat_kernel, grid_for(L * ((Ca + Cb) / 8)), 256, pdl, s, static_cast<const bf*>(a), Ca,
                    static_cast<const bf*>(b), Cb, static_cast<bf*>(out), L);
}

cudaError_t launch_gemv(const float* W, const float* b, const float* add, const float* x, float x_tau, float* y,
                        int rows, int cols, bool silu_out, bool pdl, cudaStream_t s) {
  const bool vec4 = cols % 4 == 0 && reinterpret_cast<uintptr_t>(W) % 16 == 0;
  return launch_pdl(vec4 ? gemv_kernel<true> : gemv_kernel<false>, (rows * 32 + 255) / 256, 256, pdl, s, W, b, add,
                    x, x_tau, y, rows, cols, silu_out ? 1 : 0);
}

cudaError_t launch_gemv_multi(const GemvBatch& batch, const float* x, int cols, bool pdl, cudaStream_t s) {
  if (cols % 4 || reinterpret_cast<uintptr_t>(x) % 16 || batch.n < 1 || batch.n > kGemvSegs) return cudaErrorInvalidValue;
  int rows = 0;
  for (int i = 0; i < batch.n; ++i) {
    if (reinterpret_cast<uintptr_t>(batch.seg[i].W) % 16) return cudaErrorInvalidValue;
    rows += batch.seg[i].rows;
  }
  return launch_pdl(gemv_multi_kernel, (rows * 32 + 255) / 256, 256, pdl, s, batch, x, cols);
}

cudaError_t launch_ddim_update(float* lat, const void* eps, void* x_bf, long long n, float c1, float c2, bool pdl,
                               cudaStream_t s) {
  return launch_pdl(ddim_update_kernel, grid_for(n), 256, pdl, s, lat, static_cast<const bf*>(eps),
                    static_cast<bf*>(x_bf), n, c1, c2);
}

cudaError_t launch_to_bf16(const float* a, void* b, long long n, cudaStream_t s) {
  to_bf16_kernel<<<grid_for(n), 256, 0, s>>>(a, static_cast<bf*>(b), n);
  return cudaGetLastError();
}

}  // namespace dfp
