// dfp_group_norm_noalloc: the displaced-patch GroupNorm (statistics, stale/fresh
// merge, normalise, optional SiLU) as a standalone call that allocates nothing.
//
// Some callers cannot allocate device memory at the moment they need the op: an
// engine that owns a fixed memory pool and forbids the CUDA allocator, code that
// runs where allocation is not allowed (inside a memory-capped or pre-planned
// region), or a host that must not take the allocator's locks on its critical
// path.  The regular path (dfp_create / dfp_step) allocates its scratch when the
// handle is made; this entry point instead takes its scratch -- the per-block
// partial sums, the block-arrival counter and, when the caller does not want them,
// the per-(patch, group) mean / rstd -- from one fixed array compiled into the
// library.  The caller passes only inputs and outputs.
//
// The array (g_noalloc_scratch below) is file-scope device memory: every GPU that
// loads the library holds its 256 KiB until the process exits.  Its host-side name
// is only a stand-in, so the device address is looked up with
// cudaGetSymbolAddress, once per device, by the first call made with that device
// current; make that first call before any stream capture begins.  All calls on a
// device share the array and it keeps the last call's contents: the counter that
// must start at zero is cleared by every call, and calls whose work overlaps on
// the GPU (different streams without ordering) race on the array.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>

#include <cuda_bf16.h>

#include "../../include/dfp.h"
#include "kernels.h"

namespace {

// Layout of the scratch, in floats.
constexpr size_t kCounterFloats = 64;                 // arrival counter (first word), padded
constexpr size_t kPartFloats = 64960;                 // per-block partial (sum x, sum x^2)
constexpr size_t kStatFloats = 512;                   // (mean, rstd) per (patch, group), N*G <= 256
constexpr size_t kScratchFloats = kCounterFloats + kPartFloats + kStatFloats;   // 256 KiB

static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_ptr[kMaxDevices] = {};

thread_local std::string g_noalloc_error;

// Byte ranges [a, a + na) and [b, b + nb) share at least one byte.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

dfp_status fail(dfp_status s, const std::string& m) {
  g_noalloc_error = m;
  return s;
}

}  // namespace

extern "C" DFP_API const char* dfp_group_norm_noalloc_error(void) { return g_noalloc_error.c_str(); }

extern "C" DFP_API dfp_status dfp_group_norm_noalloc(const void* x, void* y, dfp_dtype dtype, int H, int W,
                                                     int C, int n_patches, int groups, float eps,
                                                     const float* gamma, const float* beta,
                                                     const float* stale_moments, dfp_gn_mode mode,
                                                     int apply_silu, float* fresh_moments, float* mean_rstd,
                                                     void* cuda_stream) {
  // ---- argument checks (host only, before anything reaches the GPU)
  if (!x || !y || !gamma || !beta || !fresh_moments) return fail(DFP_E_ARG, "x, y, gamma, beta and fresh_moments must be non-NULL");
  if (dtype != DFP_F32 && dtype != DFP_BF16) return fail(DFP_E_ARG, "unknown dtype");
  if (H <= 0 || W <= 0 || C <= 0 || n_patches <= 0 || groups <= 0) return fail(DFP_E_ARG, "sizes must be positive");
  if (H % n_patches) return fail(DFP_E_ARG, "H must be a multiple of n_patches");
  if (C % groups) return fail(DFP_E_ARG, "C must be a multiple of groups");
  const int vec = dtype == DFP_BF16 ? 8 : 4;
  if (C % vec || C / vec > 512) return fail(DFP_E_ARG, "C must be a multiple of 16 bytes of elements and C/vector <= 512");
  if (n_patches * groups > 256) return fail(DFP_E_ARG, "n_patches * groups must be <= 256");
  if (mode < DFP_GN_CORRECTED || mode > DFP_GN_SEPARATE) return fail(DFP_E_ARG, "unknown gn mode");
  if (!(eps >= 0.f)) return fail(DFP_E_ARG, "eps must be >= 0");
  if ((long long)H * W * C >= (1ll << 31)) return fail(DFP_E_ARG, "feature map too large");
  // the kernels read x while writing y, and read stale_moments after writing fresh_moments
  // (and before writing mean_rstd): no two of these may share memory
  const size_t map_bytes = (size_t)H * W * C * (dtype == DFP_BF16 ? 2 : 4);
  const size_t mom_bytes = (size_t)n_patches * groups * 2 * sizeof(float);
  if (overlaps(x, map_bytes, y, map_bytes)) return fail(DFP_E_ARG, "x and y overlap (the op does not run in place)");
  if (stale_moments && overlaps(stale_moments, mom_bytes, fresh_moments, mom_bytes))
    return fail(DFP_E_ARG, "stale_moments and fresh_moments overlap: alternate two buffers between calls");
  if (mean_rstd && overlaps(mean_rstd, mom_bytes, fresh_moments, mom_bytes))
    return fail(DFP_E_ARG, "mean_rstd and fresh_moments overlap");
  if (mean_rstd && stale_moments && overlaps(mean_rstd, mom_bytes, stale_moments, mom_bytes))
    return fail(DFP_E_ARG, "mean_rstd and stale_moments overlap");
  const int pix_per_patch = (H / n_patches) * W;
  const int n_chunks = dfp::gn_stats_chunks(n_patches, pix_per_patch);
  const size_t part_need = (size_t)n_patches * n_chunks * groups * 2;
  if (part_need > kPartFloats)
    return fail(DFP_E_ARG, "too many (patch, group, block) partials for the fixed scratch (" +
                               std::to_string(part_need) + " > " + std::to_string(kPartFloats) + " floats)");

  // ---- once per device: the device address of the scratch array
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DFP_E_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(DFP_E_UNSUPPORTED, "device ordinal out of range");
  float* base;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return fail(DFP_E_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_ptr[dev] = static_cast<float*>(p);
    }
    base = g_ptr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  unsigned* counter = reinterpret_cast<unsigned*>(base);
  float* part = base + kCounterFloats;
  float* stats = part + kPartFloats;

  // the arrival counter must start at zero (the kernel also leaves it at zero)
  e = cudaMemsetAsync(counter, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return fail(DFP_E_CUDA, std::string("counter clear: ") + cudaGetErrorString(e));

  dfp::GnArgs a{};
  a.x = x; a.N = n_patches; a.per_image = n_patches; a.pix_per_patch = pix_per_patch; a.C = C; a.G = groups; a.eps = eps;
  a.part = part; a.counter = counter;
  a.fresh_out = fresh_moments; a.stale = stale_moments ? stale_moments : fresh_moments;
  a.gamma = gamma; a.beta = beta;
  float* mr = mean_rstd ? mean_rstd : stats;  // the (mean, rstd) the apply step reads
  a.mean_rstd = mr;
  a.is_sync = stale_moments ? 0 : 1; a.mode = (int)mode; a.naive = 0;
  if (dtype == DFP_BF16) {
    e = dfp::launch_gn_stats_merge<__nv_bfloat16>(a, s);
    if (e == cudaSuccess)
      e = dfp::launch_gn_apply<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y),
                                              nullptr, mr, gamma, beta, groups, n_patches, n_patches, pix_per_patch, C, W,
                                              pix_per_patch, 0,
                                              apply_silu != 0, 0, s);
  } else {
    e = dfp::launch_gn_stats_merge<float>(a, s);
    if (e == cudaSuccess)
      e = dfp::launch_gn_apply<float>(static_cast<const float*>(x), static_cast<float*>(y), nullptr, mr, gamma,
                                      beta, groups, n_patches, n_patches, pix_per_patch, C, W, pix_per_patch, 0,
                                      apply_silu != 0, 0, s);
  }
  if (e != cudaSuccess) return fail(DFP_E_CUDA, std::string("launch: ") + cudaGetErrorString(e));
  return DFP_OK;
}
