// Internal: the handle behind dfp_handle, shared by the C-ABI file and the stage
// scheduler.  Not part of the public interface.
#pragma once
#include <cuda_bf16.h>

#include <set>
#include <string>
#include <vector>

#include "../../include/dfp.h"
#include "kernels.h"

namespace dfp {
struct Stage;
void delete_stage(Stage* s);
struct Unet;
void delete_unet(Unet* u);
size_t dtype_size(dfp_dtype d);
// Host-side fault injection for allocation failure: while the environment variable
// DFP_FAULT_ALLOC_AFTER=k is set, the first k device allocations the library attempts
// succeed and every later one fails as if the device were out of memory (the count
// restarts when the variable is unset).  Returns true if this attempt must fail.
bool alloc_fault_injected();
}  // namespace dfp

struct dfp_ctx {
  dfp_config cfg{};
  cudaStream_t stream = nullptr;
  // dfp_step_host_async: copy streams, double-buffered device input and output staging,
  // and the events that order them against the compute stream (created on first use)
  cudaStream_t s_in = nullptr, s_out = nullptr;
  void* xin2[2] = {nullptr, nullptr};
  void* ystage[2] = {nullptr, nullptr};
  cudaEvent_t ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};
  long long n_async = 0;       // asynchronous host steps issued so far
  bool async_ready = false;    // the streams, events and buffers above are all set up
  std::string err;
  int R = 0, L = 0, Lp = 0, family = 0;
  int B = 1;                   // images per step (the guidance batch); L, Lp are per image
  bool overlap = true;         // programmatic dependent launch between the step's kernels
  long long attn_kv_budget = 0;   // attention whole-unit rounds above this many K/V bytes (0: default)
  size_t esz = 4;
  // weights
  void* w_conv = nullptr;   // [C][9][C]
  float* b_conv = nullptr;
  void* w_qkv = nullptr;    // [3C][C]
  void* w_o = nullptr;      // [C][C]
  float* b_o = nullptr;
  float *gn1_g = nullptr, *gn1_b = nullptr, *gn2_g = nullptr, *gn2_b = nullptr;
  std::set<std::string> loaded;
  std::vector<std::string> spec_names;   // storage behind the names of the stage's weight specs
  // activations and caches
  void* slab[2] = {nullptr, nullptr};
  void *h = nullptr, *t = nullptr, *q = nullptr, *o = nullptr, *y = nullptr, *xin = nullptr;
  void* kb[2] = {nullptr, nullptr};
  void* vb[2] = {nullptr, nullptr};
  float *mom1[2] = {nullptr, nullptr}, *mom2[2] = {nullptr, nullptr};
  float *mr1 = nullptr, *mr2 = nullptr, *part = nullptr;   // mr = (mean, rstd) per (patch, group)
  unsigned* counter = nullptr;
  int* dev_err = nullptr;
  // split-KV attention scratch
  int attn_ctas = 0;
  float *attn_part_o = nullptr, *attn_part_ml = nullptr;
  unsigned* attn_flags = nullptr;
  std::vector<void*> allocs;
  int last_step = -1;
  int launches = 0;
  // per-launch timing (dfp_set_profiling)
  static constexpr int kMaxEv = 128;
  bool profiling = false;
  cudaEvent_t ev[kMaxEv] = {};
  const char* ev_name[kMaxEv] = {};
  int n_ev = 0;
  // TMA descriptors (bf16 only)
  CUtensorMap m_slab[2], m_wconv, m_t, m_wqkv, m_o, m_wo, m_q, m_k[2], m_v[2];
  dfp::TcGemmPlan conv_plan{}, qkv_plan{}, out_plan{};
  // the SDXL-style stage (DFP_BLOCK_SDXL_STAGE): its own buffers and weights
  dfp::Stage* stage = nullptr;
  // the multi-level UNet (DFP_BLOCK_UNET)
  dfp::Unet* unet = nullptr;

  dfp_status fail(dfp_status s, const std::string& msg) {
    err = msg;
    return s;
  }
  dfp_status cuda_fail(cudaError_t e, const char* where) {
    err = std::string(where) + ": " + cudaGetErrorString(e);
    return DFP_E_CUDA;
  }
  bool alloc(void** p, size_t bytes) {
    if (dfp::alloc_fault_injected() || cudaMalloc(p, bytes) != cudaSuccess) { *p = nullptr; return false; }
    allocs.push_back(*p);
    return true;
  }
  // Free one allocation made by alloc() (and forget it).
  void release(void*& p) {
    if (!p) return;
    for (size_t i = 0; i < allocs.size(); ++i)
      if (allocs[i] == p) { allocs.erase(allocs.begin() + i); break; }
    cudaFree(p);
    p = nullptr;
  }
};


// Record an event before a launch when profiling, launch, check, count.
#define DFP_LAUNCH(call, what)                                   \
  do {                                                           \
    if (h->profiling && launches + 1 < dfp_ctx::kMaxEv) {        \
      cudaEventRecord(h->ev[launches], s);                       \
      h->ev_name[launches] = what;                               \
    }                                                            \
    e = (call);                                                  \
    if (e != cudaSuccess) return h->cuda_fail(e, what);          \
    ++launches;                                                  \
  } while (0)
#define DFP_LAUNCH_END()                                         \
  do {                                                           \
    if (h->profiling && launches < dfp_ctx::kMaxEv) {            \
      cudaEventRecord(h->ev[launches], s);                       \
      h->n_ev = launches + 1;                                    \
    } else if (h->profiling) {                                   \
      h->n_ev = 0;  /* more launches than events: no timing */   \
    }                                                            \
    h->launches = launches;                                      \
  } while (0)

namespace dfp {
// SDXL-style stage (csrc/stage.cu)
struct WeightSpec {
  const char* name;
  std::vector<long long> shape;
};
std::vector<WeightSpec> stage_weight_specs(const dfp_config& c, std::vector<std::string>& names);
dfp_status stage_create(dfp_ctx* h);
// Store one named weight (values as float); returns false if the name is not a stage weight.
bool stage_load_weight(dfp_ctx* h, const std::string& name, const std::vector<float>& v, dfp_status& st);
dfp_status stage_finish_load(dfp_ctx* h);
dfp_status stage_step(dfp_ctx* h, const void* x, int step, int is_sync);
bool stage_buffer(dfp_ctx* h, const std::string& name, const void** ptr, long long* bytes);
// multi-level UNet (csrc/unet.cu)
dfp_status unet_create(dfp_ctx* h);
std::vector<WeightSpec> unet_weight_specs(dfp_ctx* h);
bool unet_load_weight(dfp_ctx* h, const std::string& name, const std::vector<float>& v, dfp_status& st);
dfp_status unet_finish_load(dfp_ctx* h);
dfp_status unet_step(dfp_ctx* h, const void* x, int step, int is_sync);
void unet_set_timestep(dfp_ctx* h, float tau);
dfp_status unet_ddim(dfp_ctx* h, const float* x_T, int n_steps, int n_sync, int n_train, float beta_start,
                     float beta_end, float* x_out, dfp_status (*step_fn)(dfp_ctx*, const void*, int, int));
bool unet_buffer(dfp_ctx* h, const std::string& name, const void** ptr, long long* bytes);
}  // namespace dfp
