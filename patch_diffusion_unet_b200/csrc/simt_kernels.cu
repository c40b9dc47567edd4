// CUDA-core (SIMT) contractions of the layer step: the implicit-GEMM conv3x3 /
// projection GEMM and the displaced self-attention.  fp32 FMA throughout, so the
// fp32 configuration meets its 1e-5 relative-L2 bar (tcgen05 has no fp32 MMA);
// for bf16 storage they serve as an independent on-GPU cross-check of the
// tensor-core kernels.
//
// Displaced conv (DistriConv2dPP, "DistriFusion源码探秘" source walkthrough, Patch
// Parallelism section item 1): the A operand is read from the haloed per-patch
// slab, whose halo rows hold the previous step's neighbour rows on displaced
// steps.  Displaced attention (DistriSelfAttentionPP, same section item 2): the
// queries of patch p walk their own fresh K/V, then the other patches' K/V of
// the previous step (project README, Overview (c)).
#include "dfp_common.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kTm = 64, kTn = 64, kTk = 16;

template <typename T, bool CONV>
__device__ __forceinline__ float load_a(const T* A, const ConvA& cv, int m, int k, int K) {
  if (!CONV) return to_f32(A[(size_t)m * K + k]);
  const int tap = k / cv.Cin, ci = k - tap * cv.Cin;
  const int r = tap / 3, s = tap - 3 * (tap / 3);
  const int ppix = cv.R * cv.W;
  const int p = m / ppix, rem = m - p * ppix;
  const int i = rem / cv.W, j = rem - i * cv.W;
  const int jj = j + s - 1;
  if (jj < 0 || jj >= cv.W) return 0.f;
  const T* slab = static_cast<const T*>(cv.slab);
  return to_f32(slab[(((size_t)p * (cv.R + 2) + i + r) * cv.W + jj) * cv.Cin + ci]);
}

template <typename T>
__device__ __forceinline__ void store_epi(const Epilogue& e, int m, int n, float acc) {
  if (e.kind == 0) {
    if (e.bias) acc += e.bias[n];
    static_cast<T*>(e.out)[(size_t)m * e.ldo + n] = from_f32<T>(acc);
  } else {
    const int which = n / e.C, c = n - which * e.C;
    const int head = c >> 6, d = c & 63;
    T* dst = static_cast<T*>(which == 0 ? e.q : (which == 1 ? e.k : e.v));
    dst[((size_t)head * e.L + m) * 64 + d] = from_f32<T>(acc);
  }
}

// C[m, n] = sum_k A(m, k) * B[n, k]   (B is [N, K] row-major, i.e. PyTorch Linear weight)
template <typename T, bool CONV>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(const T* __restrict__ A, ConvA cv, const T* __restrict__ B, int M, int N, int K,
                 Epilogue epi) {
  __shared__ float As[kTk][kTm + 4];
  __shared__ float Bs[kTk][kTn + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kTm, n0 = blockIdx.x * kTn;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kTk) {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int e = tid + it * 256;
      const int row = e / kTk, kk = e % kTk;
      const int m = m0 + row, n = n0 + row, k = k0 + kk;
      As[kk][row] = (m < M && k < K) ? load_a<T, CONV>(A, cv, m, k, K) : 0.f;
      Bs[kk][row] = (n < N && k < K) ? to_f32(B[(size_t)n * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTk; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (m < M && n < N) store_epi<T>(epi, m, n, acc[i][j]);
    }
}

constexpr int kAq = 64;   // queries per block (one per thread)
constexpr int kAk = 32;   // keys staged per shared-memory tile

// One thread per query row, head width 64, online softmax in fp32.  blockIdx.y runs
// over images x N patches; q, k, v are [heads][images * L][64] and o [images * L][C],
// and a patch reads the keys of its own image only.
template <typename T>
__global__ void __launch_bounds__(kAq)
simt_attention_kernel(const T* __restrict__ q, const T* __restrict__ kf, const T* __restrict__ vf,
                      const T* __restrict__ ks, const T* __restrict__ vs, T* __restrict__ o, int L,
                      int Lp, int N, int images, int C, int mode) {
  __shared__ float Ksh[kAk][64];
  __shared__ float Vsh[kAk][64];
  const int head = blockIdx.z, pg = blockIdx.y, p = pg % N, img = pg / N;
  const size_t LT = (size_t)images * L;    // rows per head
  const int local = blockIdx.x * kAq + threadIdx.x;
  const bool valid = local < Lp;
  const int qi = pg * Lp + (valid ? local : 0);
  const float scale = 0.125f;  // 1 / sqrt(64)
  float qv[64], acc[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    qv[j] = to_f32(q[((size_t)head * LT + qi) * 64 + j]) * scale;
    acc[j] = 0.f;
  }
  float mrun = -INFINITY, lrun = 0.f;

  // key segments: (use_stale, start, length)
  int seg_n = 0, seg_st[3], seg_b[3], seg_len[3];
  if (mode == kAttnSync) {
    seg_st[0] = 0; seg_b[0] = 0; seg_len[0] = L; seg_n = 1;
  } else {
    seg_st[0] = 0; seg_b[0] = p * Lp; seg_len[0] = Lp; seg_n = 1;   // own patch, fresh
    if (mode == kAttnDisplaced) {
      if (p > 0) { seg_st[seg_n] = 1; seg_b[seg_n] = 0; seg_len[seg_n] = p * Lp; ++seg_n; }
      if ((p + 1) * Lp < L) {
        seg_st[seg_n] = 1; seg_b[seg_n] = (p + 1) * Lp; seg_len[seg_n] = L - (p + 1) * Lp; ++seg_n;
      }
    }
  }
  for (int sg = 0; sg < seg_n; ++sg) {
    const T* Kb = seg_st[sg] ? ks : kf;
    const T* Vb = seg_st[sg] ? vs : vf;
    for (int t0 = 0; t0 < seg_len[sg]; t0 += kAk) {
      const int nk = min(kAk, seg_len[sg] - t0);
      for (int e = threadIdx.x; e < kAk * 64; e += kAq) {
        const int kk = e >> 6, j = e & 63;
        const size_t row = (size_t)head * LT + (size_t)img * L + seg_b[sg] + t0 + kk;
        Ksh[kk][j] = kk < nk ? to_f32(Kb[row * 64 + j]) : 0.f;
        Vsh[kk][j] = kk < nk ? to_f32(Vb[row * 64 + j]) : 0.f;
      }
      __syncthreads();
      for (int kk = 0; kk < nk; ++kk) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) s = fmaf(qv[j], Ksh[kk][j], s);
        if (s > mrun) {
          const float alpha = expf(mrun - s);
          lrun *= alpha;
#pragma unroll
          for (int j = 0; j < 64; ++j) acc[j] *= alpha;
          mrun = s;
        }
        const float pe = expf(s - mrun);
        lrun += pe;
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] = fmaf(pe, Vsh[kk][j], acc[j]);
      }
      __syncthreads();
    }
  }
  if (valid) {
    const float inv = 1.f / lrun;
#pragma unroll
    for (int j = 0; j < 64; ++j) o[(size_t)qi * C + head * 64 + j] = from_f32<T>(acc[j] * inv);
  }
}

}  // namespace

template <typename T>
cudaError_t launch_simt_gemm(const T* A, const ConvA* conv, const T* B, int M, int N, int K,
                             const Epilogue& epi, cudaStream_t s) {
  dim3 grid((N + kTn - 1) / kTn, (M + kTm - 1) / kTm);
  if (conv)
    simt_gemm_kernel<T, true><<<grid, 256, 0, s>>>(A, *conv, B, M, N, K, epi);
  else
    simt_gemm_kernel<T, false><<<grid, 256, 0, s>>>(A, ConvA{}, B, M, N, K, epi);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_simt_attention(const T* q, const T* kf, const T* vf, const T* ks, const T* vs,
                                  T* o, int L, int Lp, int N, int images, int heads, int C, int mode,
                                  cudaStream_t s) {
  dim3 grid((Lp + kAq - 1) / kAq, N * images, heads);
  simt_attention_kernel<T><<<grid, kAq, 0, s>>>(q, kf, vf, ks, vs, o, L, Lp, N, images, C, mode);
  return cudaGetLastError();
}

template cudaError_t launch_simt_gemm<float>(const float*, const ConvA*, const float*, int, int,
                                             int, const Epilogue&, cudaStream_t);
template cudaError_t launch_simt_gemm<__nv_bfloat16>(const __nv_bfloat16*, const ConvA*,
                                                     const __nv_bfloat16*, int, int, int,
                                                     const Epilogue&, cudaStream_t);
template cudaError_t launch_simt_attention<float>(const float*, const float*, const float*,
                                                  const float*, const float*, float*, int, int,
                                                  int, int, int, int, int, cudaStream_t);
template cudaError_t launch_simt_attention<__nv_bfloat16>(
    const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
    const __nv_bfloat16*, __nv_bfloat16*, int, int, int, int, int, int, int, cudaStream_t);

}  // namespace dfp
