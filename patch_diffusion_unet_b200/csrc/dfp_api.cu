// libdfp host side: the C ABI of include/dfp.h, the handle with its device
// buffers, weight re-layout, and the fixed launch sequence of one layer step.
//
// Device memory of a handle (row-major; B images of L = H*W tokens, one after another,
// each split into N row patches -- patch index b*N + p):
//   slab[2]     [B*N][R+2][W][C] GN1+SiLU output with one halo row above/below each
//                                patch; two buffers alternate by step parity, the other
//                                one holds the previous step's map (stale context)
//   h, t        [B*H*W][C]       conv output, GN2 output
//   q           [heads][B*L][64] this step's queries
//   k[2], v[2]  [heads][B*L][64] keys / values, alternating by step parity
//   o, y        [B*L][C]         attention output, block output
//   mom1/2[2]   [B*N][G][2] fp32 per-(patch, group) (mean, variance) of GN1 / GN2, alternating
//   part        fp32 scratch     per-chunk partial sums of the GroupNorm statistics
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <new>
#include <set>
#include <string>
#include <vector>

#include <cuda_bf16.h>

#include "../../include/dfp.h"
#include "handle.h"
#include "kernels.h"

using namespace dfp;

namespace dfp {
size_t dtype_size(dfp_dtype d) { return d == DFP_BF16 ? 2 : 4; }

bool alloc_fault_injected() {
  static std::atomic<long long> attempts{0};
  const char* v = std::getenv("DFP_FAULT_ALLOC_AFTER");
  if (!v || !*v) {
    attempts.store(0);
    return false;
  }
  const long long k = std::atoll(v);
  return attempts.fetch_add(1) >= k;
}
}  // namespace dfp

namespace {

thread_local std::string g_create_error;


float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
uint16_t f32_to_bf16_bits(float f) {
  // round to nearest even (the inputs handed in are finite)
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t rounding = 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)((u + rounding) >> 16);
}

}  // namespace

namespace {

dfp_status check_config(const dfp_config* c, std::string& why) {
  auto bad = [&](const char* m) { why = m; return DFP_E_ARG; };
  if (c->H <= 0 || c->W <= 0 || c->C <= 0 || c->n_patches <= 0) return bad("H, W, C, n_patches must be positive");
  if (c->H % c->n_patches) return bad("H must be a multiple of n_patches");
  if (c->gn_groups <= 0 || c->C % c->gn_groups) return bad("C must be a multiple of gn_groups");
  if (c->n_patches * c->gn_groups > 256) return bad("n_patches * gn_groups must be <= 256");
  if (c->batch < 0 || c->batch > 8) return bad("batch must be 0..8 (0 counts as 1)");
  const long long B = c->batch > 1 ? c->batch : 1;
  if (c->dtype == DFP_F32 && B * c->n_patches * c->gn_groups > 512)
    return bad("batch * n_patches * gn_groups must be <= 512 for the SIMT kernels (fp32)");
  if (c->head_dim != 64) return bad("head_dim must be 64");
  if (c->heads * c->head_dim != c->C) return bad("heads * head_dim must equal C");
  if (c->C % 64) return bad("C must be a multiple of 64");
  if (c->C > 4096) return bad("C must be <= 4096");
  if (c->dtype != DFP_F32 && c->dtype != DFP_BF16) return bad("unknown dtype");
  if (c->gn_mode < DFP_GN_CORRECTED || c->gn_mode > DFP_GN_SEPARATE) return bad("unknown gn_mode");
  if (c->context != DFP_CTX_DISPLACED && c->context != DFP_CTX_NAIVE) return bad("unknown context");
  if (!(c->gn_eps >= 0.f)) return bad("gn_eps must be >= 0");
  const long long Lp = (long long)(c->H / c->n_patches) * c->W;
  if (Lp % 8) return bad("(H / n_patches) * W must be a multiple of 8");
  if (B * c->H * c->W * c->C > (1ll << 31)) return bad("feature map too large (batch*H*W*C >= 2^31)");
  if (c->block == DFP_BLOCK_SDXL_STAGE) {
    if (c->dtype != DFP_BF16) { why = "the transformer stage is built for bf16 storage only"; return DFP_E_UNSUPPORTED; }
    if (c->n_xformer < 1 || c->n_xformer > 2) return bad("n_xformer must be 1 or 2");
    if (c->ffn_inner <= 0 || c->ffn_inner % 64) return bad("ffn_inner must be a positive multiple of 64");
    if (c->ctx_len <= 0 || c->ctx_dim <= 0 || c->ctx_dim % 8) return bad("ctx_len > 0 and ctx_dim a positive multiple of 8");
    if (c->C > 2048) return bad("C must be <= 2048 for the transformer stage");
  } else if (c->block == DFP_BLOCK_UNET) {
    if (c->dtype != DFP_BF16) { why = "the UNet is built for bf16 storage only"; return DFP_E_UNSUPPORTED; }
    if (B != 1) { why = "the UNet runs one image per handle"; return DFP_E_UNSUPPORTED; }
    if (c->H % (4 * c->n_patches) || c->W % 4) return bad("the UNet needs H a multiple of 4 n_patches and W of 4");
    const long long R1 = c->H / c->n_patches / 2, R2 = R1 / 2;
    if ((R1 * (c->W / 2)) % 8 || (R2 * (c->W / 4)) % 8)
      return bad("the UNet's lower levels need a multiple of 8 tokens per patch");
    if (6 * c->C > 4096) return bad("the UNet needs 6 C <= 4096 (its widest concatenation)");
    if (c->ctx_len <= 0 || c->ctx_dim <= 0 || c->ctx_dim % 8) return bad("ctx_len > 0 and ctx_dim a positive multiple of 8");
  } else if (c->block != DFP_BLOCK_RES_ATTN) {
    return bad("unknown block type");
  }
  return DFP_OK;
}

// Conv tile geometry of the implicit GEMM: 128 output pixels = rows_tile x cols_tile.
void conv_tiles(int R, int W, int& cols_tile, int& rows_tile, int& tiles_per_row) {
  cols_tile = W < 128 ? W : 128;
  tiles_per_row = (W + cols_tile - 1) / cols_tile;
  rows_tile = 128 / cols_tile;
  if (rows_tile < 1) rows_tile = 1;
  while (R % rows_tile) --rows_tile;
}

dfp_status build_tmaps(dfp_ctx* h) {
  const dfp_config& c = h->cfg;
  // the batch is B * N patches and B * L tokens: every map and plan spans all images
  const int C = c.C, W = c.W, N = h->B * c.n_patches, R = h->R, L = h->B * h->L;
  bool ok = true;
  int cols_tile, rows_tile, tpr;
  conv_tiles(R, W, cols_tile, rows_tile, tpr);
  for (int i = 0; i < 2; ++i) {
    const uint64_t dims[4] = {(uint64_t)C, (uint64_t)W, (uint64_t)(R + 2), (uint64_t)N};
    const uint64_t str[3] = {(uint64_t)C * 2, (uint64_t)W * C * 2, (uint64_t)(R + 2) * W * C * 2};
    const uint32_t box[4] = {64, (uint32_t)cols_tile, (uint32_t)rows_tile, 1};
    ok &= encode_tmap_4d(&h->m_slab[i], h->slab[i], dims, str, box);
  }
  const int conv_m_tiles = N * (R / rows_tile) * tpr, lin_m_tiles = gemm_m_tiles_plain(L);
  const GemmChoice g_conv = choose_gemm(C, conv_m_tiles, conv_k_stages(C)),
                   g_qkv = choose_gemm(3 * C, lin_m_tiles, gemm_k_stages(C)),
                   g_out = choose_gemm(C, lin_m_tiles, gemm_k_stages(C));
  ok &= encode_gemm_rows(&h->m_wconv, h->w_conv, C, 9ull * C, g_conv.b_box_rows());
  ok &= encode_gemm_rows(&h->m_t, h->t, L, C, 128);
  ok &= encode_gemm_rows(&h->m_wqkv, h->w_qkv, 3ull * C, C, g_qkv.b_box_rows());
  ok &= encode_gemm_rows(&h->m_o, h->o, L, C, 128);
  ok &= encode_gemm_rows(&h->m_wo, h->w_o, C, C, g_out.b_box_rows());
  const int heads = c.heads;
  ok &= encode_tmap_3d(&h->m_q, h->q, 64, L, heads, 128, (uint64_t)L * 128, 64, 128, 1);
  for (int i = 0; i < 2; ++i) {
    ok &= encode_attn_k(&h->m_k[i], h->kb[i], L, heads);
    ok &= encode_attn_v(&h->m_v[i], h->vb[i], L, heads);
  }
  if (!ok) return h->fail(DFP_E_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  TcGemmPlan& cp = h->conv_plan;
  cp = TcGemmPlan{};
  cp.M = L; cp.N = C; cp.K = 9 * C; cp.bn = g_conv.bn; cp.pair = g_conv.pair; cp.conv = 1;
  cp.P = N; cp.R = R; cp.W = W; cp.Cin = C;
  cp.cols_tile = cols_tile; cp.rows_tile = rows_tile; cp.tiles_per_row = tpr;
  TcGemmPlan& qp = h->qkv_plan;
  qp = TcGemmPlan{};
  qp.M = L; qp.N = 3 * C; qp.K = C; qp.bn = g_qkv.bn; qp.pair = g_qkv.pair;
  TcGemmPlan& op = h->out_plan;
  op = TcGemmPlan{};
  op.M = L; op.N = C; op.K = C; op.bn = g_out.bn; op.pair = g_out.pair;
  return DFP_OK;
}

// ------------------------------------------------------------------ weights

std::vector<WeightSpec> res_attn_weight_specs(const dfp_config& c);
std::vector<WeightSpec> weight_specs(dfp_ctx* h) {
  if (h->cfg.block == DFP_BLOCK_SDXL_STAGE) return stage_weight_specs(h->cfg, h->spec_names);
  if (h->cfg.block == DFP_BLOCK_UNET) return unet_weight_specs(h);
  return res_attn_weight_specs(h->cfg);
}
std::vector<WeightSpec> res_attn_weight_specs(const dfp_config& c) {
  const long long C = c.C;
  return {
      {"gn1.weight", {C}}, {"gn1.bias", {C}}, {"conv1.weight", {C, C, 3, 3}}, {"conv1.bias", {C}},
      {"gn2.weight", {C}}, {"gn2.bias", {C}}, {"attn.to_q.weight", {C, C}}, {"attn.to_k.weight", {C, C}},
      {"attn.to_v.weight", {C, C}}, {"attn.to_out.weight", {C, C}}, {"attn.to_out.bias", {C}},
  };
}

// Read n elements of the given dtype from host memory as float.
void read_as_float(const void* src, dfp_dtype dt, size_t n, std::vector<float>& out) {
  out.resize(n);
  if (dt == DFP_F32) {
    std::memcpy(out.data(), src, n * 4);
  } else {
    const uint16_t* s = static_cast<const uint16_t*>(src);
    for (size_t i = 0; i < n; ++i) out[i] = bf16_bits_to_f32(s[i]);
  }
}

// Convert float values to the storage dtype (host bytes).
std::vector<uint8_t> to_storage(const std::vector<float>& v, dfp_dtype dt) {
  std::vector<uint8_t> out(v.size() * dtype_size(dt));
  if (dt == DFP_F32) {
    std::memcpy(out.data(), v.data(), v.size() * 4);
  } else {
    uint16_t* d = reinterpret_cast<uint16_t*>(out.data());
    for (size_t i = 0; i < v.size(); ++i) d[i] = f32_to_bf16_bits(v[i]);
  }
  return out;
}

template <typename T>
dfp_status run_step(dfp_ctx* h, const void* x, int step, int is_sync, int p0 = 0, int p1 = -1);

}  // namespace

// ====================================================================== C ABI
extern "C" {

dfp_status dfp_create(const dfp_config* cfg, void* cuda_stream, dfp_handle* out) {
  if (!out) { g_create_error = "out is NULL"; return DFP_E_ARG; }
  *out = nullptr;
  if (!cfg) { g_create_error = "cfg is NULL"; return DFP_E_ARG; }
  std::string why;
  dfp_status st = check_config(cfg, why);
  if (st != DFP_OK) { g_create_error = why; return st; }
  dfp_ctx* h = new (std::nothrow) dfp_ctx();
  if (!h) { g_create_error = "host allocation failed"; return DFP_E_NOMEM; }
  h->cfg = *cfg;
  h->stream = static_cast<cudaStream_t>(cuda_stream);
  h->R = cfg->H / cfg->n_patches;
  h->L = cfg->H * cfg->W;
  h->Lp = h->R * cfg->W;
  h->esz = dtype_size(cfg->dtype);
  h->family = cfg->dtype == DFP_BF16 ? 0 : 1;
  h->B = cfg->batch > 1 ? cfg->batch : 1;
  // buffers hold all B images: N and L below count patches and tokens over the batch
  const size_t C = cfg->C, N = (size_t)h->B * cfg->n_patches, G = cfg->gn_groups, W = cfg->W, R = h->R,
               L = (size_t)h->B * h->L;
  const size_t map = L * C * h->esz;
  const bool is_stage = cfg->block == DFP_BLOCK_SDXL_STAGE, is_unet = cfg->block == DFP_BLOCK_UNET;
  bool ok = true;
  if (!is_stage && !is_unet) {
    ok &= h->alloc(&h->w_conv, 9 * C * C * h->esz);
    ok &= h->alloc((void**)&h->b_conv, C * 4);
    ok &= h->alloc(&h->w_qkv, 3 * C * C * h->esz);
    ok &= h->alloc(&h->w_o, C * C * h->esz);
    ok &= h->alloc((void**)&h->b_o, C * 4);
    ok &= h->alloc((void**)&h->gn1_g, C * 4);
    ok &= h->alloc((void**)&h->gn1_b, C * 4);
    ok &= h->alloc((void**)&h->gn2_g, C * 4);
    ok &= h->alloc((void**)&h->gn2_b, C * 4);
    for (int i = 0; i < 2; ++i) {
      ok &= h->alloc(&h->slab[i], N * (R + 2) * W * C * h->esz);
      ok &= h->alloc(&h->kb[i], map);
      ok &= h->alloc(&h->vb[i], map);
      ok &= h->alloc((void**)&h->mom1[i], N * G * 2 * 4);
      ok &= h->alloc((void**)&h->mom2[i], N * G * 2 * 4);
    }
    ok &= h->alloc(&h->h, map);
    ok &= h->alloc(&h->t, map);
    ok &= h->alloc(&h->y, map);
  }
  ok &= h->alloc(&h->q, map);
  ok &= h->alloc(&h->o, map);
  ok &= h->alloc(&h->xin, map);
  ok &= h->alloc((void**)&h->mr1, N * G * 2 * 4);
  ok &= h->alloc((void**)&h->mr2, N * G * 2 * 4);
  ok &= h->alloc((void**)&h->part, gn_part_floats((int)N, (int)(R * W), (int)G) * 4);
  ok &= h->alloc((void**)&h->counter, 64);
  ok &= h->alloc((void**)&h->dev_err, 64);
  if (cfg->dtype == DFP_BF16) {
    // persistent attention: one CTA per SM, two partial-result slots per CTA
    h->attn_ctas = sm_count();
    const size_t f = attention_scratch_floats(h->attn_ctas);
    ok &= h->alloc((void**)&h->attn_part_o, f * 4);
    ok &= h->alloc((void**)&h->attn_part_ml, f / 32 * 4);
    ok &= h->alloc((void**)&h->attn_flags, (size_t)h->attn_ctas * 2 * 4 + 64);
  }
  if (!ok) {
    g_create_error = "device allocation failed";
    dfp_destroy(h);
    return DFP_E_NOMEM;
  }
  // zero everything the kernels rely on: slab halo rows at the image edges, the
  // GroupNorm block counter, the device error word, and all caches
  cudaError_t e = cudaSuccess;
  if (!is_stage && !is_unet) {
    for (void* p : {h->slab[0], h->slab[1]})
      if (e == cudaSuccess) e = cudaMemset(p, 0, N * (R + 2) * W * C * h->esz);
    for (void* p : {h->kb[0], h->kb[1], h->vb[0], h->vb[1], h->h, h->t, h->y})
      if (e == cudaSuccess) e = cudaMemset(p, 0, map);
  }
  for (void* p : {h->q, h->o})
    if (e == cudaSuccess) e = cudaMemset(p, 0, map);
  if (e == cudaSuccess) e = cudaMemset(h->counter, 0, 64);
  if (e == cudaSuccess) e = cudaMemset(h->dev_err, 0, 64);
  if (e == cudaSuccess && h->attn_flags) e = cudaMemset(h->attn_flags, 0, (size_t)h->attn_ctas * 2 * 4 + 64);
  if (e != cudaSuccess) {
    g_create_error = std::string("cudaMemset: ") + cudaGetErrorString(e);
    dfp_destroy(h);
    return DFP_E_CUDA;
  }
  if (is_stage) {
    st = stage_create(h);
  } else if (is_unet) {
    st = unet_create(h);
  } else if (cfg->dtype == DFP_BF16) {
    st = build_tmaps(h);
  }
  if (st != DFP_OK) {
    g_create_error = h->err;
    dfp_destroy(h);
    return st;
  }
  *out = h;
  return DFP_OK;
}

dfp_status dfp_load_weights(dfp_handle h, const dfp_tensor* w, int n) {
  if (!h) return DFP_E_ARG;
  if (n < 0 || (n > 0 && !w)) return h->fail(DFP_E_ARG, "bad weight list");
  const dfp_config& c = h->cfg;
  const std::vector<WeightSpec> specs = weight_specs(h);
  for (int i = 0; i < n; ++i) {
    const dfp_tensor& t = w[i];
    if (!t.name || !t.ptr) return h->fail(DFP_E_ARG, "weight with NULL name or pointer");
    const WeightSpec* spec = nullptr;
    for (const auto& s : specs)
      if (std::strcmp(s.name, t.name) == 0) spec = &s;
    if (!spec) return h->fail(DFP_E_ARG, std::string("unknown weight name ") + t.name);
    if (t.dtype != DFP_F32 && t.dtype != DFP_BF16) return h->fail(DFP_E_ARG, std::string("bad dtype for ") + t.name);
    if (t.ndim != (int)spec->shape.size() || !t.shape)
      return h->fail(DFP_E_ARG, std::string("wrong rank for ") + t.name);
    size_t numel = 1;
    for (int d = 0; d < t.ndim; ++d) {
      if (t.shape[d] != spec->shape[d]) return h->fail(DFP_E_ARG, std::string("wrong shape for ") + t.name);
      numel *= (size_t)t.shape[d];
    }
    // bring the values to the host as float
    std::vector<uint8_t> staging;
    const void* src = t.ptr;
    if (t.on_device) {
      staging.resize(numel * dtype_size(t.dtype));
      cudaError_t e = cudaMemcpy(staging.data(), t.ptr, staging.size(), cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return h->cuda_fail(e, "weight copy to host");
      src = staging.data();
    }
    std::vector<float> v;
    read_as_float(src, t.dtype, numel, v);
    const std::string name = t.name;
    if (h->stage || h->unet) {
      dfp_status lst = DFP_OK;
      const bool known = h->stage ? stage_load_weight(h, name, v, lst) : unet_load_weight(h, name, v, lst);
      if (!known) return h->fail(DFP_E_ARG, "unknown weight name " + name);
      if (lst != DFP_OK) return lst;
      h->loaded.insert(name);
      continue;
    }
    const size_t C = c.C;
    void* dst = nullptr;
    std::vector<uint8_t> bytes;
    size_t offset = 0;
    if (name == "conv1.weight") {
      // [Cout][Cin][3][3] -> [Cout][tap][Cin], tap = 3 r + s
      std::vector<float> r(numel);
      for (size_t co = 0; co < C; ++co)
        for (size_t ci = 0; ci < C; ++ci)
          for (int tap = 0; tap < 9; ++tap) r[(co * 9 + tap) * C + ci] = v[(co * C + ci) * 9 + tap];
      bytes = to_storage(r, c.dtype);
      dst = h->w_conv;
    } else if (name == "attn.to_q.weight" || name == "attn.to_k.weight" || name == "attn.to_v.weight") {
      const int which = name == "attn.to_q.weight" ? 0 : (name == "attn.to_k.weight" ? 1 : 2);
      bytes = to_storage(v, c.dtype);
      dst = h->w_qkv;
      offset = (size_t)which * C * C * h->esz;
    } else if (name == "attn.to_out.weight") {
      bytes = to_storage(v, c.dtype);
      dst = h->w_o;
    } else {
      // fp32 vectors
      bytes.resize(numel * 4);
      std::memcpy(bytes.data(), v.data(), numel * 4);
      if (name == "conv1.bias") dst = h->b_conv;
      else if (name == "attn.to_out.bias") dst = h->b_o;
      else if (name == "gn1.weight") dst = h->gn1_g;
      else if (name == "gn1.bias") dst = h->gn1_b;
      else if (name == "gn2.weight") dst = h->gn2_g;
      else if (name == "gn2.bias") dst = h->gn2_b;
    }
    cudaError_t e = cudaMemcpy(static_cast<uint8_t*>(dst) + offset, bytes.data(), bytes.size(),
                               cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return h->cuda_fail(e, "weight copy to device");
    h->loaded.insert(name);
  }
  if (h->stage) return stage_finish_load(h);
  if (h->unet) return unet_finish_load(h);
  return DFP_OK;
}

dfp_status dfp_step(dfp_handle h, const void* x, int step, int is_sync) {
  if (!h) return DFP_E_ARG;
  if (!x) return h->fail(DFP_E_ARG, "x is NULL");
  if (is_sync != 0 && is_sync != 1) return h->fail(DFP_E_ARG, "is_sync must be 0 or 1");
  if (step < 0) return h->fail(DFP_E_ARG, "step must be >= 0");
  if (h->loaded.size() != weight_specs(h).size())
    return h->fail(DFP_E_STATE, "weights not loaded (every weight must be given before the first step)");
  if (step == 0 && !is_sync) return h->fail(DFP_E_STATE, "step 0 must be synchronous: the context cache is empty");
  if (step != 0 && step != h->last_step + 1)
    return h->fail(DFP_E_STATE, "steps must be consecutive (or restart at 0)");
  dfp_status st = h->stage ? stage_step(h, x, step, is_sync)
                 : h->unet ? unet_step(h, x, step, is_sync)
                 : h->cfg.dtype == DFP_BF16 ? run_step<__nv_bfloat16>(h, x, step, is_sync)
                                            : run_step<float>(h, x, step, is_sync);
  if (st == DFP_OK) h->last_step = step;
  return st;
}

dfp_status dfp_step_patches(dfp_handle h, const void* x, int step, int p_begin, int p_end) {
  if (!h) return DFP_E_ARG;
  if (!x) return h->fail(DFP_E_ARG, "x is NULL");
  const dfp_config& c = h->cfg;
  if (h->stage || h->unet || c.dtype != DFP_BF16 || h->family != 0 || h->B != 1)
    return h->fail(DFP_E_UNSUPPORTED, "a patch range runs the layer block of one bf16 image on the tensor-core kernels");
  if (c.gn_mode == DFP_GN_SYNC && c.context != DFP_CTX_NAIVE)
    return h->fail(DFP_E_UNSUPPORTED, "the GroupNorm sync mode needs every patch's statistics of this step");
  if (p_begin < 0 || p_end > c.n_patches || p_begin >= p_end) return h->fail(DFP_E_ARG, "bad patch range");
  if (h->loaded.size() != weight_specs(h).size())
    return h->fail(DFP_E_STATE, "weights not loaded (every weight must be given before the first step)");
  if (step <= 0 || step != h->last_step + 1)
    return h->fail(DFP_E_STATE, "a patch-range step is displaced: it must follow the previous step (step >= 1)");
  dfp_status st = run_step<__nv_bfloat16>(h, x, step, 0, p_begin, p_end);
  if (st == DFP_OK) h->last_step = step;
  return st;
}

dfp_status dfp_context_buffer(dfp_handle h, const char* name, int parity, void** ptr, long long* bytes) {
  if (!h) return DFP_E_ARG;
  if (!name || !ptr || !bytes) return h->fail(DFP_E_ARG, "NULL argument");
  if (parity != 0 && parity != 1) return h->fail(DFP_E_ARG, "parity must be 0 or 1");
  if (h->stage || h->unet) return h->fail(DFP_E_UNSUPPORTED, "context buffers of the layer block only");
  const dfp_config& c = h->cfg;
  const long long map = (long long)h->B * h->L * c.C * (long long)h->esz;
  const long long mom = (long long)h->B * c.n_patches * c.gn_groups * 2 * 4;
  const std::string n = name;
  if (n == "k") { *ptr = h->kb[parity]; *bytes = map; }
  else if (n == "v") { *ptr = h->vb[parity]; *bytes = map; }
  else if (n == "mom1") { *ptr = h->mom1[parity]; *bytes = mom; }
  else if (n == "mom2") { *ptr = h->mom2[parity]; *bytes = mom; }
  else if (n == "slab") {
    *ptr = h->slab[parity];
    *bytes = (long long)h->B * c.n_patches * (h->R + 2) * c.W * c.C * (long long)h->esz;
  } else if (n == "y") { *ptr = h->y; *bytes = map; }
  else return h->fail(DFP_E_ARG, std::string("unknown context buffer ") + name);
  return DFP_OK;
}

dfp_status dfp_set_timestep(dfp_handle h, float timestep) {
  if (!h) return DFP_E_ARG;
  if (!h->unet) return h->fail(DFP_E_UNSUPPORTED, "timesteps belong to the UNet block");
  if (!(timestep >= 0.f)) return h->fail(DFP_E_ARG, "timestep must be >= 0");
  unet_set_timestep(h, timestep);
  return DFP_OK;
}

dfp_status dfp_ddim_sample(dfp_handle h, const float* x_T, int n_steps, int n_sync, int n_train, float beta_start,
                           float beta_end, float* x_out) {
  if (!h) return DFP_E_ARG;
  if (!h->unet) return h->fail(DFP_E_UNSUPPORTED, "DDIM runs the UNet block");
  if (!x_T || !x_out) return h->fail(DFP_E_ARG, "x_T / x_out is NULL");
  if (n_steps < 1 || n_sync < 1 || n_train < n_steps || n_train > 100000)
    return h->fail(DFP_E_ARG, "need n_steps >= 1, n_sync >= 1 and n_steps <= n_train <= 100000");
  if (!(beta_start > 0.f && beta_start < beta_end && beta_end < 1.f)) return h->fail(DFP_E_ARG, "bad beta range");
  if (h->loaded.size() != weight_specs(h).size())
    return h->fail(DFP_E_STATE, "weights not loaded (every weight must be given before the first step)");
  return unet_ddim(h, x_T, n_steps, n_sync, n_train, beta_start, beta_end, x_out, dfp_step);
}

dfp_status dfp_step_host(dfp_handle h, const void* x_host, void* y_host, int step, int is_sync) {
  if (!h) return DFP_E_ARG;
  if (h->unet) return h->fail(DFP_E_UNSUPPORTED, "host-buffer steps of the layer blocks only");
  if (!x_host || !y_host) return h->fail(DFP_E_ARG, "x_host / y_host is NULL");
  const size_t bytes = (size_t)h->B * h->L * h->cfg.C * h->esz;
  cudaError_t e = cudaMemcpyAsync(h->xin, x_host, bytes, cudaMemcpyHostToDevice, h->stream);
  if (e != cudaSuccess) return h->cuda_fail(e, "input copy");
  dfp_status st = dfp_step(h, h->xin, step, is_sync);
  if (st != DFP_OK) return st;
  e = cudaMemcpyAsync(y_host, h->y, bytes, cudaMemcpyDeviceToHost, h->stream);
  if (e != cudaSuccess) return h->cuda_fail(e, "output copy");
  e = cudaStreamSynchronize(h->stream);
  if (e != cudaSuccess) return h->cuda_fail(e, "stream synchronize");
  return DFP_OK;
}

dfp_status dfp_step_host_async(dfp_handle h, const void* x_host, void* y_host, int step, int is_sync) {
  if (!h) return DFP_E_ARG;
  if (h->unet) return h->fail(DFP_E_UNSUPPORTED, "host-buffer steps of the layer blocks only");
  if (!x_host || !y_host) return h->fail(DFP_E_ARG, "x_host / y_host is NULL");
  const size_t bytes = (size_t)h->B * h->L * h->cfg.C * h->esz;
  cudaError_t e = cudaSuccess;
  if (!h->async_ready) {
    // set up on first use; a failed set-up leaves nothing behind, so a later call retries
    if (!h->s_in) e = cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking);
    if (e == cudaSuccess && !h->s_out) e = cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
      if (!h->ev_in[i]) e = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming);
      if (e == cudaSuccess && !h->ev_done[i]) e = cudaEventCreateWithFlags(&h->ev_done[i], cudaEventDisableTiming);
      if (e == cudaSuccess && !h->ev_out[i]) e = cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return h->cuda_fail(e, "async host step set-up");
    bool ok = true;
    for (int i = 0; i < 2; ++i) ok = ok && h->alloc(&h->xin2[i], bytes) && h->alloc(&h->ystage[i], bytes);
    if (!ok) {
      for (int i = 0; i < 2; ++i) { h->release(h->xin2[i]); h->release(h->ystage[i]); }
      return h->fail(DFP_E_NOMEM, "device allocation failed");
    }
    h->async_ready = true;
  }
  const int b = (int)(h->n_async & 1);
  const bool reuse = h->n_async >= 2;   // buffer b was used two calls ago
  // input: into xin2[b] once the step two calls ago has finished reading it
  if (reuse && (e = cudaStreamWaitEvent(h->s_in, h->ev_done[b], 0)) != cudaSuccess) return h->cuda_fail(e, "input order");
  if ((e = cudaMemcpyAsync(h->xin2[b], x_host, bytes, cudaMemcpyHostToDevice, h->s_in)) != cudaSuccess)
    return h->cuda_fail(e, "input copy");
  if ((e = cudaEventRecord(h->ev_in[b], h->s_in)) != cudaSuccess) return h->cuda_fail(e, "input event");
  if ((e = cudaStreamWaitEvent(h->stream, h->ev_in[b], 0)) != cudaSuccess) return h->cuda_fail(e, "input order");
  dfp_status st = dfp_step(h, h->xin2[b], step, is_sync);
  if (st != DFP_OK) return st;
  // output: staged to ystage[b] (once its previous copy-out is done), copied out on s_out
  if (reuse && (e = cudaStreamWaitEvent(h->stream, h->ev_out[b], 0)) != cudaSuccess) return h->cuda_fail(e, "output order");
  if ((e = cudaMemcpyAsync(h->ystage[b], h->y, bytes, cudaMemcpyDeviceToDevice, h->stream)) != cudaSuccess)
    return h->cuda_fail(e, "output staging");
  if ((e = cudaEventRecord(h->ev_done[b], h->stream)) != cudaSuccess) return h->cuda_fail(e, "step event");
  if ((e = cudaStreamWaitEvent(h->s_out, h->ev_done[b], 0)) != cudaSuccess) return h->cuda_fail(e, "output order");
  if ((e = cudaMemcpyAsync(y_host, h->ystage[b], bytes, cudaMemcpyDeviceToHost, h->s_out)) != cudaSuccess)
    return h->cuda_fail(e, "output copy");
  if ((e = cudaEventRecord(h->ev_out[b], h->s_out)) != cudaSuccess) return h->cuda_fail(e, "output event");
  ++h->n_async;
  return DFP_OK;
}

dfp_status dfp_synchronize(dfp_handle h) {
  if (!h) return DFP_E_ARG;
  cudaError_t e = cudaStreamSynchronize(h->stream);
  if (e == cudaSuccess && h->s_in) e = cudaStreamSynchronize(h->s_in);
  if (e == cudaSuccess && h->s_out) e = cudaStreamSynchronize(h->s_out);
  if (e != cudaSuccess) return h->cuda_fail(e, "stream synchronize");
  return DFP_OK;
}

dfp_status dfp_output(dfp_handle h, const void** y) {
  if (!h) return DFP_E_ARG;
  if (!y) return h->fail(DFP_E_ARG, "y is NULL");
  *y = h->y;
  return DFP_OK;
}

static bool buffer_of(dfp_handle h, const char* name, const void** ptr, long long* bytes) {
  const long long map = (long long)h->B * h->L * h->cfg.C * (long long)h->esz;
  const long long st = (long long)h->B * h->cfg.n_patches * h->cfg.gn_groups * 2 * 4;
  const int cur = h->last_step < 0 ? 0 : (h->last_step & 1);
  const std::string n = name;
  if (h->unet) return unet_buffer(h, n, ptr, bytes);
  if (h->stage) {
    if (stage_buffer(h, n, ptr, bytes)) return true;
    if (n == "gn1" || n == "gn2") { *ptr = n == "gn1" ? h->mr1 : h->mr2; *bytes = st; return true; }
    if (n == "q" || n == "o") { *ptr = n == "q" ? h->q : h->o; *bytes = map; return true; }
    return false;
  }
  if (n == "y") { *ptr = h->y; *bytes = map; }
  else if (n == "h") { *ptr = h->h; *bytes = map; }
  else if (n == "t") { *ptr = h->t; *bytes = map; }
  else if (n == "o") { *ptr = h->o; *bytes = map; }
  else if (n == "q") { *ptr = h->q; *bytes = map; }
  else if (n == "k") { *ptr = h->kb[cur]; *bytes = map; }
  else if (n == "v") { *ptr = h->vb[cur]; *bytes = map; }
  else if (n == "gn1") { *ptr = h->mr1; *bytes = st; }
  else if (n == "gn2") { *ptr = h->mr2; *bytes = st; }
  else if (n == "slab") {
    *ptr = h->slab[cur];
    *bytes = (long long)h->B * h->cfg.n_patches * (h->R + 2) * h->cfg.W * h->cfg.C * (long long)h->esz;
  } else return false;
  return true;
}

dfp_status dfp_buffer_bytes(dfp_handle h, const char* name, long long* bytes) {
  if (!h) return DFP_E_ARG;
  if (!name || !bytes) return h->fail(DFP_E_ARG, "NULL argument");
  const void* p;
  if (!buffer_of(h, name, &p, bytes)) return h->fail(DFP_E_ARG, std::string("unknown buffer ") + name);
  return DFP_OK;
}

dfp_status dfp_copy_out(dfp_handle h, const char* name, void* dst, long long dst_bytes) {
  if (!h) return DFP_E_ARG;
  if (!name || !dst) return h->fail(DFP_E_ARG, "NULL argument");
  const void* p;
  long long bytes;
  if (!buffer_of(h, name, &p, &bytes)) return h->fail(DFP_E_ARG, std::string("unknown buffer ") + name);
  if (dst_bytes != bytes) return h->fail(DFP_E_ARG, "dst_bytes does not match the buffer size");
  cudaError_t e = cudaMemcpyAsync(dst, p, (size_t)bytes, cudaMemcpyDefault, h->stream);
  if (e != cudaSuccess) return h->cuda_fail(e, "buffer copy");
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, dst) != cudaSuccess || attr.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) return h->cuda_fail(e, "stream synchronize");
  }
  return DFP_OK;
}

dfp_status dfp_check_device(dfp_handle h) {
  if (!h) return DFP_E_ARG;
  cudaError_t e = cudaStreamSynchronize(h->stream);
  if (e != cudaSuccess) return h->cuda_fail(e, "stream synchronize");
  int flag = 0;
  e = cudaMemcpy(&flag, h->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return h->cuda_fail(e, "error flag read");
  if (flag != 0) {
    // a kernel that gave up left its grid-barrier counters mid-count: re-arm them (no kernel
    // is in flight after the synchronize above) so the next step starts clean
    cudaMemset(h->dev_err, 0, sizeof(int));
    cudaMemset(h->counter, 0, 64);
    return h->fail(DFP_E_DEVICE, "a kernel wait ran past its limit (device error code " + std::to_string(flag) + ")");
  }
  return DFP_OK;
}

int dfp_launches_per_step(dfp_handle h) { return h ? h->launches : -1; }

int dfp_attention_schedule_check(int L, int Lp, int n_patches, int heads, int mode, int kv_len, int images,
                                 int ctas, int p_begin, int p_end, long long kv_budget_bytes) {
  if (mode < kAttnSync || mode > kAttnCross) return 1;
  return attention_schedule_check(L, Lp, n_patches, heads, mode, kv_len, images, ctas, p_begin, p_end,
                                  kv_budget_bytes);
}

dfp_status dfp_set_launch_overlap(dfp_handle h, int enable) {
  if (!h) return DFP_E_ARG;
  if (enable != 0 && enable != 1) return h->fail(DFP_E_ARG, "enable must be 0 or 1");
  h->overlap = enable != 0;
  return DFP_OK;
}

dfp_status dfp_set_attention_kv_budget(dfp_handle h, long long bytes) {
  if (!h) return DFP_E_ARG;
  if (bytes < 0) return h->fail(DFP_E_ARG, "the K/V budget must be >= 0");
  h->attn_kv_budget = bytes;
  return DFP_OK;
}

dfp_status dfp_set_kernel_family(dfp_handle h, int family) {
  if (!h) return DFP_E_ARG;
  if (family != 0 && family != 1) return h->fail(DFP_E_ARG, "family must be 0 or 1");
  if (family == 0 && h->cfg.dtype != DFP_BF16)
    return h->fail(DFP_E_UNSUPPORTED, "tensor-core kernels need bf16 storage");
  if (family == 1 && h->B * h->cfg.n_patches * h->cfg.gn_groups > 512)
    return h->fail(DFP_E_UNSUPPORTED, "the SIMT kernels need batch * n_patches * gn_groups <= 512");
  h->family = family;
  return DFP_OK;
}

dfp_status dfp_set_profiling(dfp_handle h, int enable) {
  if (!h) return DFP_E_ARG;
  if (enable && !h->ev[0]) {
    for (int i = 0; i < dfp_ctx::kMaxEv; ++i) {
      cudaError_t e = cudaEventCreate(&h->ev[i]);
      if (e != cudaSuccess) return h->cuda_fail(e, "event create");
    }
  }
  h->profiling = enable != 0;
  h->n_ev = 0;
  return DFP_OK;
}

int dfp_kernel_times(dfp_handle h, float* ms, const char** names, int max_n) {
  if (!h) return -1;
  if (!h->profiling || h->n_ev < 2) return 0;
  if (cudaEventSynchronize(h->ev[h->n_ev - 1]) != cudaSuccess) return -1;
  const int n = h->n_ev - 1 < max_n ? h->n_ev - 1 : max_n;
  for (int i = 0; i < n; ++i) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, h->ev[i], h->ev[i + 1]) != cudaSuccess) return -1;
    if (ms) ms[i] = t;
    if (names) names[i] = h->ev_name[i];
  }
  return n;
}

dfp_status dfp_destroy(dfp_handle h) {
  if (!h) return DFP_OK;
  cudaStreamSynchronize(h->stream);
  for (cudaStream_t cs : {h->s_in, h->s_out})
    if (cs) { cudaStreamSynchronize(cs); cudaStreamDestroy(cs); }
  for (int i = 0; i < 2; ++i)
    for (cudaEvent_t ev : {h->ev_in[i], h->ev_done[i], h->ev_out[i]})
      if (ev) cudaEventDestroy(ev);
  for (int i = 0; i < dfp_ctx::kMaxEv; ++i)
    if (h->ev[i]) cudaEventDestroy(h->ev[i]);
  for (void* p : h->allocs) cudaFree(p);
  delete_stage(h->stage);
  delete_unet(h->unet);
  delete h;
  return DFP_OK;
}

const char* dfp_last_error(dfp_handle h) {
  if (!h) return g_create_error.c_str();
  return h->err.c_str();
}

}  // extern "C"

// ====================================================================== step scheduler
namespace {

// p0, p1: the patches computed, [p0, p1) of the one image (a patch-parallel rank's range;
// the whole map when p1 < 0).  Range steps are displaced tensor-core steps of one image.
template <typename T>
dfp_status run_step(dfp_ctx* h, const void* xv, int step, int is_sync, int p0, int p1) {
  const dfp_config& c = h->cfg;
  // N, L per image; NB, LB over the batch (B images, patch b*N + p, token b*L + i)
  const int N = c.n_patches, C = c.C, G = c.gn_groups, W = c.W, R = h->R, L = h->L, Lp = h->Lp;
  const int B = h->B, NB = B * N, LB = B * L;
  const bool range = p1 >= 0;
  if (!range) { p0 = 0; p1 = NB; }
  const int n_run = p1 - p0;
  const int cur = step & 1, prv = cur ^ 1;
  const bool naive = c.context == DFP_CTX_NAIVE;
  const bool displaced = !is_sync && !naive;
  cudaStream_t s = h->stream;
  const T* x = static_cast<const T*>(xv);
  T* slab = static_cast<T*>(h->slab[cur]);
  int launches = 0;
  cudaError_t e;
  h->n_ev = 0;

  // ---- GN1 statistics (+ corrected merge) and apply + SiLU into the slab interior
  GnArgs g{};
  g.x = x; g.N = NB; g.per_image = N; g.pix_per_patch = Lp; g.C = C; g.G = G; g.eps = c.gn_eps;
  g.part = h->part; g.counter = h->counter;
  g.fresh_out = h->mom1[cur]; g.stale = h->mom1[prv];
  g.gamma = h->gn1_g; g.beta = h->gn1_b; g.mean_rstd = h->mr1;
  g.is_sync = is_sync; g.mode = (int)c.gn_mode; g.naive = naive ? 1 : 0;
  g.p0 = p0; g.n_run = n_run;
  // consecutive tensor-core-family kernels overlap launch and set-up with their
  // predecessor's tail (each waits for the predecessor before touching memory)
  const int pdl = h->overlap ? 1 : 0;
  g.pdl = pdl;
  h->conv_plan.pdl = h->qkv_plan.pdl = h->out_plan.pdl = pdl;
  // the apply also fills the halo rows: the neighbours' boundary rows of this step
  // (sync) or of the previous step (displaced, read from the other slab buffer)
  const int halo_mode = (naive || N == 1) ? 0 : (displaced ? 2 : 1);
  if (h->family == 0) {
    // statistics, merge and apply in one cooperative launch
    const GnOut go{slab, h->slab[prv], (long long)(R + 2) * W, W, W, halo_mode};
    DFP_LAUNCH(launch_gn_fused<T>(g, go, true, h->dev_err, s), "gn1 + SiLU + halo (fused)");
  } else {
    DFP_LAUNCH(launch_gn_stats_merge<T>(g, s), "gn1 statistics");
    DFP_LAUNCH(launch_gn_apply<T>(x, slab, static_cast<const T*>(h->slab[prv]), h->mr1, h->gn1_g, h->gn1_b, G, NB, N,
                                  Lp, C, W, (long long)(R + 2) * W, W, true, halo_mode, s), "gn1 apply + halo");
  }
  // ---- conv3x3 (+ bias) -> h
  Epilogue ec{};
  ec.kind = 0; ec.out = h->h; ec.bias = h->b_conv; ec.ldo = C;
  // a patch range computes the conv tiles of its patches and the projections of its rows
  TcGemmPlan conv_plan = h->conv_plan, qkv_plan = h->qkv_plan, out_plan = h->out_plan;
  conv_plan.p0 = p0; conv_plan.P = n_run;
  qkv_plan.m_base = out_plan.m_base = p0 * Lp;
  qkv_plan.M = out_plan.M = p1 * Lp;
  if (h->family == 0) {
    DFP_LAUNCH(launch_tc_gemm(conv_plan, h->m_slab[cur], h->m_wconv, ec, h->dev_err, s), "conv (tcgen05)");
  } else {
    ConvA cv{slab, NB, R, W, C};
    DFP_LAUNCH(launch_simt_gemm<T>(nullptr, &cv, static_cast<const T*>(h->w_conv), LB, C, 9 * C, ec, s), "conv (simt)");
  }
  // ---- GN2 (no SiLU) -> t
  g.x = h->h; g.fresh_out = h->mom2[cur]; g.stale = h->mom2[prv];
  g.gamma = h->gn2_g; g.beta = h->gn2_b; g.mean_rstd = h->mr2;
  if (h->family == 0) {
    const GnOut go{h->t, nullptr, (long long)Lp, 0, W, 0};
    DFP_LAUNCH(launch_gn_fused<T>(g, go, false, h->dev_err, s), "gn2 (fused)");
  } else {
    DFP_LAUNCH(launch_gn_stats_merge<T>(g, s), "gn2 statistics");
    DFP_LAUNCH(launch_gn_apply<T>(static_cast<const T*>(h->h), static_cast<T*>(h->t), nullptr, h->mr2, h->gn2_g,
                                  h->gn2_b, G, NB, N, Lp, C, W, (long long)Lp, 0, false, 0, s), "gn2 apply");
  }
  // ---- Q, K, V projections; K/V land in this step's cache buffers
  Epilogue eq{};
  eq.kind = 1; eq.q = h->q; eq.k = h->kb[cur]; eq.v = h->vb[cur]; eq.L = LB; eq.C = C;
  if (h->family == 0) {
    DFP_LAUNCH(launch_tc_gemm(qkv_plan, h->m_t, h->m_wqkv, eq, h->dev_err, s), "qkv (tcgen05)");
  } else {
    DFP_LAUNCH(launch_simt_gemm<T>(static_cast<const T*>(h->t), nullptr, static_cast<const T*>(h->w_qkv), LB, 3 * C, C, eq, s), "qkv (simt)");
  }
  // ---- displaced attention
  const int mode = naive ? kAttnNaive : (is_sync ? kAttnSync : kAttnDisplaced);
  if (h->family == 0) {
    TcAttnArgs a{};
    a.L = L; a.Lp = Lp; a.N = N; a.heads = c.heads; a.C = C; a.mode = mode; a.o = h->o; a.err = h->dev_err;
    a.images = B; a.kv_stride = L; a.pdl = pdl;
    a.p_lo = p0; a.p_hi = p1;
    a.ctas = h->attn_ctas; a.n_qtiles = (Lp + 127) / 128;
    a.part_o = h->attn_part_o; a.part_ml = h->attn_part_ml; a.flags = h->attn_flags;
    a.kv_budget = h->attn_kv_budget;
    DFP_LAUNCH(launch_tc_attention(a, h->m_q, h->m_k[cur], h->m_v[cur], h->m_k[prv], h->m_v[prv], s), "attention (tcgen05)");
  } else {
    DFP_LAUNCH(launch_simt_attention<T>(static_cast<const T*>(h->q), static_cast<const T*>(h->kb[cur]),
                                        static_cast<const T*>(h->vb[cur]), static_cast<const T*>(h->kb[prv]),
                                        static_cast<const T*>(h->vb[prv]), static_cast<T*>(h->o), L, Lp, N, B,
                                        c.heads, C, mode, s), "attention (simt)");
  }
  // ---- output projection (+ bias) -> y
  Epilogue eo{};
  eo.kind = 0; eo.out = h->y; eo.bias = h->b_o; eo.ldo = C;
  if (h->family == 0) {
    DFP_LAUNCH(launch_tc_gemm(out_plan, h->m_o, h->m_wo, eo, h->dev_err, s), "out projection (tcgen05)");
  } else {
    DFP_LAUNCH(launch_simt_gemm<T>(static_cast<const T*>(h->o), nullptr, static_cast<const T*>(h->w_o), LB, C, C, eo, s), "out projection (simt)");
  }
  DFP_LAUNCH_END();
  return DFP_OK;
}

}  // namespace
