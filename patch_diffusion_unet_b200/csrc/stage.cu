// The SDXL-style stage (DFP_BLOCK_SDXL_STAGE) on the displaced-patch path:
//   ResNet block   r0 = x + conv2(SiLU(GN2(conv1(SiLU(GN1(x))))))   -- both GroupNorms and
//                  both convs displaced (stale statistics / halo rows on displaced steps)
//   transformer block b (x n_xformer), pre-LayerNorm, residual everywhere:
//                  r += to_out(SA(LN1(r)))    self-attention, other patches' K/V stale
//                  r += to_out(CA(LN2(r)))    cross-attention to a fixed text context
//                  r += W2 (a * GELU(g)),  [a, g] = W1 LN3(r) + b1   (GEGLU feed-forward)
// The pages wrap exactly these three kinds of layers -- convolution, self/cross
// attention and GroupNorm ("DistriFusion源码探秘" source walkthrough, Patch
// Parallelism section items 1-3); LayerNorm, the projections and the feed-forward
// act per token and need no cross-patch context.
//
// Device memory (bf16 storage, fp32 statistics / accumulation; B images one after
// another, L tokens and N patches each, as in the res-attn block):
//   slab1[2], slab2[2]   [B*N][R+2][W][C]  conv inputs with halo rows, parity-alternating
//   h1                   [B*L][C]          conv1 output
//   r[1 + 3 n_xformer]   [B*L][C]          residual stream after the ResNet block and after
//                                          each attention / feed-forward sub-layer
//   u                    [B*L][C]          LayerNorm output (A operand of the projections)
//   g                    [B*L][F]          GEGLU output
//   per block: k[2], v[2] [heads][B*L][64] self-attention cache; ctx_k, ctx_v
//                        [heads][B*ctx_rows][64] projected context of each image (at load)
#include <cmath>
#include <cstring>

#include "handle.h"

namespace dfp {

struct XfBlock {
  float *ln_g[3] = {}, *ln_b[3] = {};
  void *w_qkv = nullptr, *w_o1 = nullptr, *w_q2 = nullptr, *w_o2 = nullptr, *w_k2 = nullptr, *w_v2 = nullptr;
  void *w_ff1 = nullptr, *w_ff2 = nullptr;
  float *b_o1 = nullptr, *b_o2 = nullptr, *b_ff1 = nullptr, *b_ff2 = nullptr;
  void* kb[2] = {};
  void* vb[2] = {};
  void *ctx_k = nullptr, *ctx_v = nullptr;
  bool ctx_ready = false;
  CUtensorMap m_wqkv, m_wo1, m_wq2, m_wo2, m_wff1, m_wff2, m_k[2], m_v[2], m_ck, m_cv;
  TcGemmPlan p_qkv{}, p_o1{}, p_q2{}, p_o2{}, p_ff1{}, p_ff2{};
};

struct Stage {
  float *n1_g = nullptr, *n1_b = nullptr, *n2_g = nullptr, *n2_b = nullptr;
  void *w_c1 = nullptr, *w_c2 = nullptr;
  float *b_c1 = nullptr, *b_c2 = nullptr;
  void* slab1[2] = {};
  void* slab2[2] = {};
  float* mom1[2] = {};
  float* mom2[2] = {};
  void* h1 = nullptr;
  std::vector<void*> r;
  void *u = nullptr, *g = nullptr, *ctx = nullptr;
  XfBlock xf[2];
  CUtensorMap m_slab1[2], m_slab2[2], m_wc1, m_wc2, m_u, m_o, m_g;
  TcGemmPlan p_c1{}, p_c2{};
  bool ctx_loaded = false;
};

namespace {

// rows per head of the context K/V buffers: ctx_len padded with zeros to whole 128-key tiles
size_t ctx_rows(size_t ctx_len) { return (ctx_len + 127) / 128 * 128; }

uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

dfp_status upload_bf16(dfp_ctx* h, void* dst, const std::vector<float>& v) {
  std::vector<uint16_t> b(v.size());
  for (size_t i = 0; i < v.size(); ++i) b[i] = f32_to_bf16(v[i]);
  cudaError_t e = cudaMemcpy(dst, b.data(), b.size() * 2, cudaMemcpyHostToDevice);
  return e == cudaSuccess ? DFP_OK : h->cuda_fail(e, "weight copy to device");
}
dfp_status upload_f32(dfp_ctx* h, void* dst, const std::vector<float>& v) {
  cudaError_t e = cudaMemcpy(dst, v.data(), v.size() * 4, cudaMemcpyHostToDevice);
  return e == cudaSuccess ? DFP_OK : h->cuda_fail(e, "weight copy to device");
}

}  // namespace

void delete_stage(Stage* s) { delete s; }

std::vector<WeightSpec> stage_weight_specs(const dfp_config& c, std::vector<std::string>& names) {
  const long long C = c.C, D = c.ctx_dim, F = c.ffn_inner, T = c.ctx_len;
  names.clear();
  std::vector<std::pair<std::string, std::vector<long long>>> v = {
      {"resnet.norm1.weight", {C}}, {"resnet.norm1.bias", {C}},
      {"resnet.conv1.weight", {C, C, 3, 3}}, {"resnet.conv1.bias", {C}},
      {"resnet.norm2.weight", {C}}, {"resnet.norm2.bias", {C}},
      {"resnet.conv2.weight", {C, C, 3, 3}}, {"resnet.conv2.bias", {C}},
      {"context", c.batch > 1 ? std::vector<long long>{c.batch, T, D} : std::vector<long long>{T, D}},
  };
  for (int b = 0; b < c.n_xformer; ++b) {
    const std::string p = "xf" + std::to_string(b) + ".";
    for (const char* n : {"norm1", "norm2", "norm3"}) {
      v.push_back({p + n + ".weight", {C}});
      v.push_back({p + n + ".bias", {C}});
    }
    v.push_back({p + "attn1.to_q.weight", {C, C}});
    v.push_back({p + "attn1.to_k.weight", {C, C}});
    v.push_back({p + "attn1.to_v.weight", {C, C}});
    v.push_back({p + "attn1.to_out.weight", {C, C}});
    v.push_back({p + "attn1.to_out.bias", {C}});
    v.push_back({p + "attn2.to_q.weight", {C, C}});
    v.push_back({p + "attn2.to_k.weight", {C, D}});
    v.push_back({p + "attn2.to_v.weight", {C, D}});
    v.push_back({p + "attn2.to_out.weight", {C, C}});
    v.push_back({p + "attn2.to_out.bias", {C}});
    v.push_back({p + "ff.proj.weight", {2 * F, C}});
    v.push_back({p + "ff.proj.bias", {2 * F}});
    v.push_back({p + "ff.out.weight", {C, F}});
    v.push_back({p + "ff.out.bias", {C}});
  }
  std::vector<WeightSpec> out;
  names.reserve(v.size());
  for (auto& kv : v) names.push_back(kv.first);
  for (size_t i = 0; i < v.size(); ++i) out.push_back(WeightSpec{names[i].c_str(), v[i].second});
  return out;
}

dfp_status stage_create(dfp_ctx* h) {
  const dfp_config& c = h->cfg;
  Stage* st = new (std::nothrow) Stage();
  if (!st) return h->fail(DFP_E_NOMEM, "host allocation failed");
  h->stage = st;
  // N and L count patches and tokens over the batch; T context tokens per image
  const size_t B = h->B, C = c.C, N = B * c.n_patches, G = c.gn_groups, W = c.W, R = h->R, L = B * h->L;
  const size_t F = c.ffn_inner, T = c.ctx_len, D = c.ctx_dim, heads = c.heads;
  const size_t map = L * C * 2, slab = N * (R + 2) * W * C * 2, ctx_all = B * ctx_rows(T);
  bool ok = true;
  ok &= h->alloc((void**)&st->n1_g, C * 4) && h->alloc((void**)&st->n1_b, C * 4);
  ok &= h->alloc((void**)&st->n2_g, C * 4) && h->alloc((void**)&st->n2_b, C * 4);
  ok &= h->alloc(&st->w_c1, 9 * C * C * 2) && h->alloc(&st->w_c2, 9 * C * C * 2);
  ok &= h->alloc((void**)&st->b_c1, C * 4) && h->alloc((void**)&st->b_c2, C * 4);
  for (int i = 0; i < 2; ++i) {
    ok &= h->alloc(&st->slab1[i], slab) && h->alloc(&st->slab2[i], slab);
    ok &= h->alloc((void**)&st->mom1[i], N * G * 8) && h->alloc((void**)&st->mom2[i], N * G * 8);
  }
  ok &= h->alloc(&st->h1, map) && h->alloc(&st->u, map) && h->alloc(&st->g, L * F * 2);
  ok &= h->alloc(&st->ctx, B * T * D * 2);
  st->r.assign(1 + 3 * c.n_xformer, nullptr);
  for (auto& p : st->r) ok &= h->alloc(&p, map);
  for (int b = 0; b < c.n_xformer; ++b) {
    XfBlock& x = st->xf[b];
    for (int k = 0; k < 3; ++k) ok &= h->alloc((void**)&x.ln_g[k], C * 4) && h->alloc((void**)&x.ln_b[k], C * 4);
    ok &= h->alloc(&x.w_qkv, 3 * C * C * 2) && h->alloc(&x.w_o1, C * C * 2) && h->alloc(&x.w_q2, C * C * 2);
    ok &= h->alloc(&x.w_o2, C * C * 2) && h->alloc(&x.w_k2, C * D * 2) && h->alloc(&x.w_v2, C * D * 2);
    ok &= h->alloc(&x.w_ff1, 2 * F * C * 2) && h->alloc(&x.w_ff2, C * F * 2);
    ok &= h->alloc((void**)&x.b_o1, C * 4) && h->alloc((void**)&x.b_o2, C * 4);
    ok &= h->alloc((void**)&x.b_ff1, 2 * F * 4) && h->alloc((void**)&x.b_ff2, C * 4);
    for (int i = 0; i < 2; ++i) ok &= h->alloc(&x.kb[i], map) && h->alloc(&x.vb[i], map);
    // context K/V: ctx_len rows per head padded with zeros to whole 128-key tiles
    ok &= h->alloc(&x.ctx_k, heads * ctx_all * 64 * 2) && h->alloc(&x.ctx_v, heads * ctx_all * 64 * 2);
  }
  if (!ok) return h->fail(DFP_E_NOMEM, "device allocation failed");
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
    e = cudaMemset(st->slab1[i], 0, slab);
    if (e == cudaSuccess) e = cudaMemset(st->slab2[i], 0, slab);
  }
  for (int b = 0; b < c.n_xformer && e == cudaSuccess; ++b)
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
      e = cudaMemset(st->xf[b].kb[i], 0, map);
      if (e == cudaSuccess) e = cudaMemset(st->xf[b].vb[i], 0, map);
    }
  for (int b = 0; b < c.n_xformer && e == cudaSuccess; ++b) {
    e = cudaMemset(st->xf[b].ctx_k, 0, heads * ctx_all * 64 * 2);
    if (e == cudaSuccess) e = cudaMemset(st->xf[b].ctx_v, 0, heads * ctx_all * 64 * 2);
  }
  if (e != cudaSuccess) return h->cuda_fail(e, "cudaMemset");
  h->y = st->r.back();

  // ---- TMA descriptors and GEMM plans
  int cols_tile = W < 128 ? (int)W : 128, tpr = ((int)W + cols_tile - 1) / cols_tile;
  int rows_tile = 128 / cols_tile;
  if (rows_tile < 1) rows_tile = 1;
  while ((int)R % rows_tile) --rows_tile;
  ok = true;
  for (int i = 0; i < 2; ++i) {
    const uint64_t dims[4] = {C, W, R + 2, N};
    const uint64_t strides[3] = {C * 2, W * C * 2, (R + 2) * W * C * 2};
    const uint32_t box[4] = {64, (uint32_t)cols_tile, (uint32_t)rows_tile, 1};
    ok &= encode_tmap_4d(&st->m_slab1[i], st->slab1[i], dims, strides, box);
    ok &= encode_tmap_4d(&st->m_slab2[i], st->slab2[i], dims, strides, box);
  }
  const int lin_m = gemm_m_tiles_plain((int)L);
  const GemmChoice g_c = choose_gemm((int)C, (int)N * ((int)R / rows_tile) * tpr, conv_k_stages((int)C));
  ok &= encode_gemm_rows(&st->m_wc1, st->w_c1, C, 9 * C, g_c.b_box_rows());
  ok &= encode_gemm_rows(&st->m_wc2, st->w_c2, C, 9 * C, g_c.b_box_rows());
  ok &= encode_gemm_rows(&st->m_u, st->u, L, C, 128);
  ok &= encode_gemm_rows(&st->m_o, h->o, L, C, 128);
  ok &= encode_gemm_rows(&st->m_g, st->g, L, F, 128);
  ok &= encode_tmap_3d(&h->m_q, h->q, 64, L, heads, 128, L * 128, 64, 128, 1);
  auto plan = [&](TcGemmPlan& p, int M, int Nn, int K, const GemmChoice& g) {
    p = TcGemmPlan{};
    p.M = M; p.N = Nn; p.K = K; p.bn = g.bn; p.pair = g.pair;
  };
  for (int b = 0; b < c.n_xformer; ++b) {
    XfBlock& x = st->xf[b];
    const int ks = gemm_k_stages((int)C);
    const GemmChoice bq = choose_gemm(3 * (int)C, lin_m, ks), bc = choose_gemm((int)C, lin_m, ks);
    // GEGLU: 128-wide tiles of 64 value + 64 gate columns (the weight rows are interleaved so)
    const GemmChoice bf = choose_gemm(2 * (int)F, lin_m, ks, 128);
    const GemmChoice b2 = choose_gemm((int)C, lin_m, gemm_k_stages((int)F));
    ok &= encode_gemm_rows(&x.m_wqkv, x.w_qkv, 3 * C, C, bq.b_box_rows());
    ok &= encode_gemm_rows(&x.m_wo1, x.w_o1, C, C, bc.b_box_rows());
    ok &= encode_gemm_rows(&x.m_wq2, x.w_q2, C, C, bc.b_box_rows());
    ok &= encode_gemm_rows(&x.m_wo2, x.w_o2, C, C, bc.b_box_rows());
    ok &= encode_gemm_rows(&x.m_wff1, x.w_ff1, 2 * F, C, bf.b_box_rows());
    ok &= encode_gemm_rows(&x.m_wff2, x.w_ff2, C, F, b2.b_box_rows());
    for (int i = 0; i < 2; ++i) {
      ok &= encode_attn_k(&x.m_k[i], x.kb[i], L, heads);
      ok &= encode_attn_v(&x.m_v[i], x.vb[i], L, heads);
    }
    ok &= encode_attn_k(&x.m_ck, x.ctx_k, ctx_all, heads);
    ok &= encode_attn_v(&x.m_cv, x.ctx_v, ctx_all, heads);
    plan(x.p_qkv, (int)L, 3 * (int)C, (int)C, bq);
    plan(x.p_o1, (int)L, (int)C, (int)C, bc);
    plan(x.p_q2, (int)L, (int)C, (int)C, bc);
    plan(x.p_o2, (int)L, (int)C, (int)C, bc);
    plan(x.p_ff1, (int)L, 2 * (int)F, (int)C, bf);
    plan(x.p_ff2, (int)L, (int)C, (int)F, b2);
  }
  if (!ok) return h->fail(DFP_E_CUDA, "cuTensorMapEncodeTiled failed");
  for (TcGemmPlan* p : {&st->p_c1, &st->p_c2}) {
    *p = TcGemmPlan{};
    p->M = (int)L; p->N = (int)C; p->K = 9 * (int)C; p->bn = g_c.bn; p->pair = g_c.pair; p->conv = 1;
    p->P = (int)N; p->R = (int)R; p->W = (int)W; p->Cin = (int)C;
    p->cols_tile = cols_tile; p->rows_tile = rows_tile; p->tiles_per_row = tpr;
  }
  return DFP_OK;
}

bool stage_load_weight(dfp_ctx* h, const std::string& name, const std::vector<float>& v, dfp_status& out) {
  Stage* st = h->stage;
  const dfp_config& c = h->cfg;
  const size_t C = c.C, F = c.ffn_inner;
  auto conv = [&](void* dst) {
    // [Cout][Cin][3][3] -> [Cout][tap][Cin]
    std::vector<float> r(v.size());
    for (size_t co = 0; co < C; ++co)
      for (size_t ci = 0; ci < C; ++ci)
        for (int tap = 0; tap < 9; ++tap) r[(co * 9 + tap) * C + ci] = v[(co * C + ci) * 9 + tap];
    return upload_bf16(h, dst, r);
  };
  out = DFP_OK;
  if (name == "resnet.norm1.weight") out = upload_f32(h, st->n1_g, v);
  else if (name == "resnet.norm1.bias") out = upload_f32(h, st->n1_b, v);
  else if (name == "resnet.norm2.weight") out = upload_f32(h, st->n2_g, v);
  else if (name == "resnet.norm2.bias") out = upload_f32(h, st->n2_b, v);
  else if (name == "resnet.conv1.weight") out = conv(st->w_c1);
  else if (name == "resnet.conv2.weight") out = conv(st->w_c2);
  else if (name == "resnet.conv1.bias") out = upload_f32(h, st->b_c1, v);
  else if (name == "resnet.conv2.bias") out = upload_f32(h, st->b_c2, v);
  else if (name == "context") { out = upload_bf16(h, st->ctx, v); st->ctx_loaded = true; for (auto& x : st->xf) x.ctx_ready = false; }
  else if (name.size() > 4 && name.compare(0, 2, "xf") == 0) {
    const int b = name[2] - '0';
    if (b < 0 || b >= c.n_xformer || name[3] != '.') return false;
    XfBlock& x = st->xf[b];
    const std::string n = name.substr(4);
    if (n == "norm1.weight") out = upload_f32(h, x.ln_g[0], v);
    else if (n == "norm1.bias") out = upload_f32(h, x.ln_b[0], v);
    else if (n == "norm2.weight") out = upload_f32(h, x.ln_g[1], v);
    else if (n == "norm2.bias") out = upload_f32(h, x.ln_b[1], v);
    else if (n == "norm3.weight") out = upload_f32(h, x.ln_g[2], v);
    else if (n == "norm3.bias") out = upload_f32(h, x.ln_b[2], v);
    else if (n == "attn1.to_q.weight" || n == "attn1.to_k.weight" || n == "attn1.to_v.weight") {
      const int which = n[9] == 'q' ? 0 : (n[9] == 'k' ? 1 : 2);
      out = upload_bf16(h, static_cast<uint8_t*>(x.w_qkv) + which * C * C * 2, v);
    } else if (n == "attn1.to_out.weight") out = upload_bf16(h, x.w_o1, v);
    else if (n == "attn1.to_out.bias") out = upload_f32(h, x.b_o1, v);
    else if (n == "attn2.to_q.weight") out = upload_bf16(h, x.w_q2, v);
    else if (n == "attn2.to_k.weight") { out = upload_bf16(h, x.w_k2, v); x.ctx_ready = false; }
    else if (n == "attn2.to_v.weight") { out = upload_bf16(h, x.w_v2, v); x.ctx_ready = false; }
    else if (n == "attn2.to_out.weight") out = upload_bf16(h, x.w_o2, v);
    else if (n == "attn2.to_out.bias") out = upload_f32(h, x.b_o2, v);
    else if (n == "ff.proj.weight" || n == "ff.proj.bias") {
      // interleave per 128-row tile: 64 value rows (f0..f0+63) then their 64 gate rows (F+f0..)
      const size_t cols = n == "ff.proj.weight" ? C : 1;
      std::vector<float> r(v.size());
      for (size_t t = 0; t < 2 * F / 128; ++t)
        for (size_t j = 0; j < 128; ++j) {
          const size_t src = j < 64 ? 64 * t + j : F + 64 * t + (j - 64);
          std::memcpy(&r[(t * 128 + j) * cols], &v[src * cols], cols * 4);
        }
      out = cols == 1 ? upload_f32(h, x.b_ff1, r) : upload_bf16(h, x.w_ff1, r);
    } else if (n == "ff.out.weight") out = upload_bf16(h, x.w_ff2, v);
    else if (n == "ff.out.bias") out = upload_f32(h, x.b_ff2, v);
    else return false;
  } else {
    return false;
  }
  return true;
}

dfp_status stage_finish_load(dfp_ctx* h) {
  // context K/V of every block whose inputs are all present: [ctx_len, ctx_dim] x W^T -> head-major
  Stage* st = h->stage;
  const dfp_config& c = h->cfg;
  if (!st->ctx_loaded) return DFP_OK;
  for (int b = 0; b < c.n_xformer; ++b) {
    XfBlock& x = st->xf[b];
    const std::string p = "xf" + std::to_string(b) + ".";
    if (x.ctx_ready || !h->loaded.count(p + "attn2.to_k.weight") || !h->loaded.count(p + "attn2.to_v.weight"))
      continue;
    // image i's context rows land at rows [i * ctx_rows, i * ctx_rows + ctx_len) of every head
    const size_t cr = ctx_rows(c.ctx_len);
    for (int img = 0; img < h->B; ++img)
      for (int kv = 0; kv < 2; ++kv) {
        Epilogue e{};
        e.kind = 1;
        e.q = static_cast<__nv_bfloat16*>(kv == 0 ? x.ctx_k : x.ctx_v) + img * cr * 64;
        e.L = (int)(h->B * cr); e.C = c.C;   // head stride: the padded rows of all images
        cudaError_t ce = launch_simt_gemm<__nv_bfloat16>(
            static_cast<const __nv_bfloat16*>(st->ctx) + (size_t)img * c.ctx_len * c.ctx_dim, nullptr,
            static_cast<const __nv_bfloat16*>(kv == 0 ? x.w_k2 : x.w_v2), c.ctx_len, c.C, c.ctx_dim, e, h->stream);
        if (ce != cudaSuccess) return h->cuda_fail(ce, "context projection");
      }
    cudaError_t ce = cudaStreamSynchronize(h->stream);
    if (ce != cudaSuccess) return h->cuda_fail(ce, "context projection");
    x.ctx_ready = true;
  }
  return DFP_OK;
}

dfp_status stage_step(dfp_ctx* h, const void* xv, int step, int is_sync) {
  Stage* st = h->stage;
  const dfp_config& c = h->cfg;
  // N, L per image; NB, LB over the batch (B images, patch b*N + p, token b*L + i)
  const int N = c.n_patches, C = c.C, G = c.gn_groups, W = c.W, R = h->R, L = h->L, Lp = h->Lp;
  const int B = h->B, NB = B * N, LB = B * L;
  const int cur = step & 1, prv = cur ^ 1;
  const bool naive = c.context == DFP_CTX_NAIVE;
  const bool displaced = !is_sync && !naive;
  for (int b = 0; b < c.n_xformer; ++b)
    if (!st->xf[b].ctx_ready) return h->fail(DFP_E_STATE, "cross-attention context not projected (load the context)");
  cudaStream_t s = h->stream;
  int launches = 0;
  cudaError_t e;
  h->n_ev = 0;
  using bf = __nv_bfloat16;
  const int halo_mode = (naive || N == 1) ? 0 : (displaced ? 2 : 1);

  // ---- ResNet block: GN1 + SiLU -> conv1 -> GN2 + SiLU -> conv2 + x
  GnArgs g{};
  const int pdl = h->overlap ? 1 : 0;   // see run_step: launch overlap between kernels
  st->p_c1.pdl = st->p_c2.pdl = pdl;
  for (int b = 0; b < c.n_xformer; ++b)
    for (TcGemmPlan* p : {&st->xf[b].p_qkv, &st->xf[b].p_o1, &st->xf[b].p_q2, &st->xf[b].p_o2, &st->xf[b].p_ff1,
                          &st->xf[b].p_ff2})
      p->pdl = pdl;
  g.pdl = pdl;
  g.x = xv; g.N = NB; g.per_image = N; g.pix_per_patch = Lp; g.C = C; g.G = G; g.eps = c.gn_eps;
  g.part = h->part; g.counter = h->counter;
  g.is_sync = is_sync; g.mode = (int)c.gn_mode; g.naive = naive ? 1 : 0;
  g.fresh_out = st->mom1[cur]; g.stale = st->mom1[prv]; g.gamma = st->n1_g; g.beta = st->n1_b; g.mean_rstd = h->mr1;
  {
    const GnOut go{st->slab1[cur], st->slab1[prv], (long long)(R + 2) * W, W, W, halo_mode};
    DFP_LAUNCH(launch_gn_fused<bf>(g, go, true, h->dev_err, s), "norm1 + SiLU + halo (fused)");
  }
  Epilogue ec{};
  ec.kind = 0; ec.out = st->h1; ec.bias = st->b_c1; ec.ldo = C;
  DFP_LAUNCH(launch_tc_gemm(st->p_c1, st->m_slab1[cur], st->m_wc1, ec, h->dev_err, s), "conv1 (tcgen05)");
  g.x = st->h1; g.fresh_out = st->mom2[cur]; g.stale = st->mom2[prv]; g.gamma = st->n2_g; g.beta = st->n2_b;
  g.mean_rstd = h->mr2;
  {
    const GnOut go{st->slab2[cur], st->slab2[prv], (long long)(R + 2) * W, W, W, halo_mode};
    DFP_LAUNCH(launch_gn_fused<bf>(g, go, true, h->dev_err, s), "norm2 + SiLU + halo (fused)");
  }
  ec.out = st->r[0]; ec.bias = st->b_c2; ec.residual = xv;
  DFP_LAUNCH(launch_tc_gemm(st->p_c2, st->m_slab2[cur], st->m_wc2, ec, h->dev_err, s), "conv2 + residual (tcgen05)");

  // ---- transformer blocks
  const int sa_mode = naive ? kAttnNaive : (is_sync ? kAttnSync : kAttnDisplaced);
  for (int b = 0; b < c.n_xformer; ++b) {
    XfBlock& x = st->xf[b];
    void* rin = st->r[3 * b];
    void* r_sa = st->r[3 * b + 1];
    void* r_ca = st->r[3 * b + 2];
    void* r_ff = st->r[3 * b + 3];
    // self-attention on displaced K/V
    DFP_LAUNCH(launch_layernorm(rin, st->u, x.ln_g[0], x.ln_b[0], LB, C, 1e-5f, pdl != 0, s), "layernorm 1");
    Epilogue eq{};
    eq.kind = 1; eq.q = h->q; eq.k = x.kb[cur]; eq.v = x.vb[cur]; eq.L = LB; eq.C = C;
    DFP_LAUNCH(launch_tc_gemm(x.p_qkv, st->m_u, x.m_wqkv, eq, h->dev_err, s), "self-attn qkv (tcgen05)");
    TcAttnArgs a{};
    a.L = L; a.Lp = Lp; a.N = N; a.heads = c.heads; a.C = C; a.mode = sa_mode; a.o = h->o; a.err = h->dev_err;
    a.images = B; a.kv_stride = L; a.pdl = pdl;
    a.n_qtiles = (Lp + 127) / 128; a.ctas = h->attn_ctas;
    a.part_o = h->attn_part_o; a.part_ml = h->attn_part_ml; a.flags = h->attn_flags;
    a.kv_budget = h->attn_kv_budget;
    DFP_LAUNCH(launch_tc_attention(a, h->m_q, x.m_k[cur], x.m_v[cur], x.m_k[prv], x.m_v[prv], s),
               "self-attention (tcgen05)");
    Epilogue eo{};
    eo.kind = 0; eo.out = r_sa; eo.bias = x.b_o1; eo.residual = rin; eo.ldo = C;
    DFP_LAUNCH(launch_tc_gemm(x.p_o1, st->m_o, x.m_wo1, eo, h->dev_err, s), "self-attn out + residual (tcgen05)");
    // cross-attention to the fixed context (same for every patch: no staleness)
    DFP_LAUNCH(launch_layernorm(r_sa, st->u, x.ln_g[1], x.ln_b[1], LB, C, 1e-5f, pdl != 0, s), "layernorm 2");
    Epilogue e2{};
    e2.kind = 1; e2.q = h->q; e2.L = LB; e2.C = C;
    DFP_LAUNCH(launch_tc_gemm(x.p_q2, st->m_u, x.m_wq2, e2, h->dev_err, s), "cross-attn q (tcgen05)");
    TcAttnArgs ca{};
    ca.L = L; ca.Lp = L; ca.N = 1; ca.heads = c.heads; ca.C = C; ca.mode = kAttnCross; ca.kv_len = c.ctx_len;
    ca.images = B; ca.kv_stride = (int)ctx_rows(c.ctx_len);   // image b reads its own context
    ca.pdl = pdl;
    ca.o = h->o; ca.err = h->dev_err; ca.n_qtiles = (L + 127) / 128; ca.ctas = h->attn_ctas;
    ca.part_o = h->attn_part_o; ca.part_ml = h->attn_part_ml; ca.flags = h->attn_flags;
    ca.kv_budget = h->attn_kv_budget;
    DFP_LAUNCH(launch_tc_attention(ca, h->m_q, x.m_ck, x.m_cv, x.m_ck, x.m_cv, s), "cross-attention (tcgen05)");
    eo.out = r_ca; eo.bias = x.b_o2; eo.residual = r_sa;
    DFP_LAUNCH(launch_tc_gemm(x.p_o2, st->m_o, x.m_wo2, eo, h->dev_err, s), "cross-attn out + residual (tcgen05)");
    // GEGLU feed-forward
    DFP_LAUNCH(launch_layernorm(r_ca, st->u, x.ln_g[2], x.ln_b[2], LB, C, 1e-5f, pdl != 0, s), "layernorm 3");
    Epilogue ef{};
    ef.kind = 2; ef.out = st->g; ef.bias = x.b_ff1; ef.ldo = c.ffn_inner;
    DFP_LAUNCH(launch_tc_gemm(x.p_ff1, st->m_u, x.m_wff1, ef, h->dev_err, s), "ff proj + GEGLU (tcgen05)");
    eo.out = r_ff; eo.bias = x.b_ff2; eo.residual = r_ca;
    DFP_LAUNCH(launch_tc_gemm(x.p_ff2, st->m_g, x.m_wff2, eo, h->dev_err, s), "ff out + residual (tcgen05)");
  }
  DFP_LAUNCH_END();
  return DFP_OK;
}

bool stage_buffer(dfp_ctx* h, const std::string& name, const void** ptr, long long* bytes) {
  Stage* st = h->stage;
  const dfp_config& c = h->cfg;
  const long long map = (long long)h->B * h->L * c.C * 2;
  const int cur = h->last_step < 0 ? 0 : (h->last_step & 1);
  if (name == "y") { *ptr = st->r.back(); *bytes = map; return true; }
  if (name == "resnet") { *ptr = st->r[0]; *bytes = map; return true; }
  if (name == "h") { *ptr = st->h1; *bytes = map; return true; }
  if (name == "slab" || name == "slab2") {
    *ptr = name == "slab" ? st->slab1[cur] : st->slab2[cur];
    *bytes = (long long)h->B * c.n_patches * (h->R + 2) * c.W * c.C * 2;
    return true;
  }
  for (int b = 0; b < c.n_xformer; ++b) {
    const std::string p = "xf" + std::to_string(b) + ".";
    if (name == p + "sa") { *ptr = st->r[3 * b + 1]; *bytes = map; return true; }
    if (name == p + "ca") { *ptr = st->r[3 * b + 2]; *bytes = map; return true; }
    if (name == p + "out") { *ptr = st->r[3 * b + 3]; *bytes = map; return true; }
  }
  return false;
}

}  // namespace dfp
