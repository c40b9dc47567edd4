// Host-side launchers of libdfp's kernels (internal; not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dfp {

// Attention context mode of one launch.
enum AttnMode : int { kAttnSync = 0, kAttnDisplaced = 1, kAttnNaive = 2, kAttnCross = 3 };

// ---------------------------------------------------------------- GroupNorm
struct GnArgs {
  const void* x;          // [N * pix_per_patch, C] input map, patch-major rows
  int N, pix_per_patch, C, G;
  int per_image;          // patches per image: N = images * per_image; the merge runs over
                          // the patches of one image and halos stop at image edges
  float eps;
  float* part;            // scratch [N][n_chunks][G][2] partial (sum x, sum x^2)
  unsigned* counter;      // scratch, one word, zero between launches
  float* fresh_out;       // [N][G][2] this step's (mean, variance) per (patch, group)
  const float* stale;     // [N][G][2] (mean, variance) of step t-1 (read on displaced steps)
  const float* gamma;     // [C] fp32
  const float* beta;      // [C] fp32
  float* mean_rstd;       // [N][G][2] (mean, rstd) applied -- also read by the separate apply kernel
  int is_sync, mode, naive;
  int pdl;                // fused kernel: launch with programmatic stream serialization
  int p0, n_run;          // fused kernel: patches [p0, p0 + n_run) are computed (0, 0: all N);
                          // part is indexed by the patch's place in that range
};
// Output side of the fused GroupNorm: out [N][out_patch_stride pixels][C] starting at
// pixel out_off of each patch (the haloed slab, or a plain map with stride pix_per_patch
// and offset 0), halo_mode as for launch_gn_apply.
struct GnOut {
  void* out;
  const void* prev_slab;
  long long out_patch_stride, out_off;
  int W, halo_mode;
};
int gn_stats_chunks(int N, int pix_per_patch);
// floats of GroupNorm partial sums any patch range of N patches needs (the part scratch)
size_t gn_part_floats(int N, int pix_per_patch, int G);
// statistics + merge + apply (+SiLU) in one cooperative launch; a.counter needs two
// zeroed words; a.mean_rstd receives (mean, rstd)
template <typename T> cudaError_t launch_gn_fused(const GnArgs& a, const GnOut& o, bool silu, int* err, cudaStream_t s);
template <typename T> cudaError_t launch_gn_stats_merge(const GnArgs& a, cudaStream_t s);
// halo_mode: 0 none (plain output), 1 sync (fresh neighbour rows), 2 displaced
// (the previous step's rows, read from prev_slab); N patches in all, per_image per image
template <typename T>
cudaError_t launch_gn_apply(const T* x, T* out, const T* prev_slab, const float* mean_rstd, const float* gamma,
                            const float* beta, int G, int N, int per_image, int pix_per_patch, int C, int W,
                            long long out_patch_stride_pix, long long out_pix_off, bool silu, int halo_mode,
                            cudaStream_t s);

// Per-token LayerNorm over C channels (biased variance), bf16 in / out, fp32 math.
// pdl: launch with programmatic stream serialization (the kernel waits for its predecessor).
cudaError_t launch_layernorm(const void* x, void* y, const float* gamma, const float* beta, int L, int C,
                             float eps, bool pdl, cudaStream_t s);

// ---------------------------------------------------------------- multi-level UNet helpers
// The haloed conv input slab [N][R+2][W][C] filled from a map [N*R][W][src_C] (upsample:
// from the map at half resolution, each pixel repeated 2 x 2); channels past src_C zero;
// halo_mode as for launch_gn_apply (2 reads the neighbours' rows from prev_slab).
cudaError_t launch_slab_fill(const void* src, int src_C, void* slab, const void* prev_slab, int C, int N, int R,
                             int W, int halo_mode, bool upsample, bool pdl, cudaStream_t s);
// out [L][Ca+Cb] = a [L][Ca] then b [L][Cb], bf16
cudaError_t launch_concat(const void* a, int Ca, const void* b, int Cb, void* out, long long L, bool pdl,
                          cudaStream_t s);
// y = act(W x + b (+ add)), fp32, W [rows][cols]; x_tau >= 0: x is the sinusoidal
// embedding of timestep x_tau (cols entries)
cudaError_t launch_gemv(const float* W, const float* b, const float* add, const float* x, float x_tau, float* y,
                        int rows, int cols, bool silu_out, bool pdl, cudaStream_t s);
// y_s = W_s x + b_s (+ add_s) for up to kGemvSegs segments over one x [cols] (cols % 4 == 0,
// 16-byte aligned W and x), one launch
constexpr int kGemvSegs = 8;
struct GemvSeg {
  const float* W;     // [rows][cols]
  const float* b;
  const float* add;   // may be null
  float* y;
  int rows;
};
struct GemvBatch {
  GemvSeg seg[kGemvSegs];
  int n;
};
cudaError_t launch_gemv_multi(const GemvBatch& batch, const float* x, int cols, bool pdl, cudaStream_t s);
// DDIM update lat = c1 lat + c2 eps (fp32 latent, bf16 eps), and its bf16 copy
cudaError_t launch_ddim_update(float* lat, const void* eps, void* x_bf, long long n, float c1, float c2, bool pdl,
                               cudaStream_t s);
cudaError_t launch_to_bf16(const float* a, void* b, long long n, cudaStream_t s);

// ---------------------------------------------------------------- GEMM epilogues
struct Epilogue {
  // 0: out[m, n] = acc + bias[n] (+ residual[m, n]); bias / residual may be null
  // 1: Q/K/V scatter: column n -> (n / C: 0 q, 1 k, 2 v; head; d) into [heads][L][64]
  // 2: GEGLU: the 128 columns of a tile are 64 values then the 64 matching gates;
  //    out[m, n0/2 + j] = (v_j + bias) * GELU(g_j + bias), GELU exact (erf)
  int kind;
  void* out;              // kinds 0, 2: [M, ldo]
  const float* bias;
  const void* residual;   // kind 0: [M, ldo] bf16, may alias out (same element read then written)
  int ldo;
  int subsample;          // kind 0, conv: store only even (row, column) pixels, into the
                          // half-resolution map (a stride-2 conv)
  int n_store;            // kind 0: columns stored (0: all); a layer padded to a wider tile
  void* q; void* k; void* v;
  int L, C;
};
// A operand of the conv: the haloed per-patch slab [N][R+2][W][Cin]; row m of the
// implicit GEMM is pixel m of the full map, column k = tap * Cin + ci.
struct ConvA {
  const void* slab;
  int N, R, W, Cin;
};

// SIMT (CUDA-core) contractions: the fp32 path, and a cross-check for bf16.
template <typename T>
cudaError_t launch_simt_gemm(const T* A, const ConvA* conv, const T* B, int M, int N, int K,
                             const Epilogue& epi, cudaStream_t s);
template <typename T>
cudaError_t launch_simt_attention(const T* q, const T* kf, const T* vf, const T* ks, const T* vs,
                                  T* o, int L, int Lp, int N, int images, int heads, int C, int mode,
                                  cudaStream_t s);

// ---------------------------------------------------------------- tensor-core path (bf16)
// TMA descriptors are built once per buffer on the host.
bool encode_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t outer_stride_bytes, uint32_t box_inner, uint32_t box_outer);
bool encode_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);
bool encode_tmap_4d(CUtensorMap* m, const void* base, const uint64_t dims[4],
                    const uint64_t strides_bytes[3], const uint32_t box[4]);
bool encode_tmap_5d(CUtensorMap* m, const void* base, const uint64_t dims[5],
                    const uint64_t strides_bytes[4], const uint32_t box[5]);
// GEMM operand: row-major [rows][K] bf16, K a multiple of 64; box = box_rows x two 64-wide K chunks
bool encode_gemm_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows);

struct TcGemmPlan {
  int M, N, K;            // GEMM sizes (conv: M = H*W, K = 9*Cin); plain: rows [m_base, M) are computed
  int bn;                 // N tile (64, 128, 160 or 256)
  int conv;               // 1: A is the haloed slab (4-D map), 0: plain [M, K] (2-D map)
  int m_base;             // plain: first row computed (a patch range of a patch-parallel rank; else 0)
  int p0;                 // conv: first patch computed; P patches from there
  // conv geometry
  int P, R, W, Cin;       // patches computed, rows per patch, width, input channels
  int cols_tile, rows_tile, tiles_per_row;
  int pair;               // 1: CTA-pair kernel (256 x bn tiles; B's map boxes bn/2 rows)
  int m_tiles;            // filled by launch_tc_gemm
  int sms;                // persistent grid size (SM count), filled by launch_tc_gemm
  int pdl;                // launch with programmatic stream serialization
};
cudaError_t launch_tc_gemm(const TcGemmPlan& plan, const CUtensorMap& mapA, const CUtensorMap& mapB,
                           const Epilogue& epi, int* err, cudaStream_t s);
// N-tile width and CTA-pairing (pair: 256-row tiles over two SMs, B's map boxes bn/2
// rows) minimising waves x operand rows per SM and k-stage; k_stages = two-chunk (128-wide)
// K stages per tile; force_bn fixes the width.
struct GemmChoice {
  int bn, pair;
  uint32_t b_box_rows() const { return pair ? bn / 2 : bn; }
};
GemmChoice choose_gemm(int N, int m_tiles, int k_stages, int force_bn = 0);
// two-chunk K stages of a plain GEMM (K) and of the conv (Cin): what choose_gemm takes
inline int gemm_k_stages(int K) { return (K / 64 + 1) / 2; }
inline int conv_k_stages(int Cin) { return 9 * ((Cin / 64 + 1) / 2); }
int gemm_m_tiles_plain(int M);

struct TcAttnArgs {
  int L, Lp, N, heads, C, mode;   // per image: L tokens in N patches of Lp
  int p_lo, p_hi;         // query patches [p_lo, p_hi) of the image-major patch list (0, 0: all)
  int images;             // images of the batch; q, o, k and v hold them one after another
  int kv_stride;          // K/V rows per image: L, or the padded context rows (kAttnCross)
  int kv_len;             // cross-attention: number of context tokens (mode kAttnCross)
  void* o;                // [images * L, C] bf16
  int* err;
  int n_qtiles;           // ceil(Lp / 128)
  int ctas;               // persistent CTAs (one per SM); the scratch below is sized for them
  float* part_o;          // scratch [ctas][256][64]: unnormalised O of the CTA's first piece when
                          // it continues a pair another CTA started
  float* part_ml;         // scratch [ctas][256][2]:  (running max, row sum) of the same
  unsigned* flags;        // scratch [ctas][2]: publish flags of the CTAs' first pieces (zeroed once)
  // set by the launcher: the work split (whole-unit rounds, then a stream-K tail)
  int whole_rounds;       // rounds of whole units dealt one per CTA
  int total_tiles;        // tiles of the tail (the units after whole_rounds * ctas)
  int tail_base;          // tiles of the units before the tail
  int head_tiles;         // tiles of one head's units
  unsigned epoch;         // set by the launcher: this launch's flag value (never 0, never reused)
  int pdl;                // launch with programmatic stream serialization
  long long kv_budget;    // K/V bytes above which whole-unit rounds are used (0: the kernel's own)
};
// floats of part_o for `ctas` CTAs (part_ml needs 1/32 of it)
size_t attention_scratch_floats(int ctas);
// Host walk of the attention work split over `ctas` CTAs (0: every property holds)
// kv_budget: K/V bytes above which whole-unit rounds are used (< 0: the launcher's own)
int attention_schedule_check(int L, int Lp, int N, int heads, int mode, int kv_len, int images, int ctas,
                             int p_lo = 0, int p_hi = 0, long long kv_budget = -1);
int sm_count();
// V operand of the attention: [heads][rows][64] bf16 (rows a multiple of 4, every KV tile
// starting at a multiple of 4) seen as a 5-D view whose 128-row box lands in shared memory
// with rows 1 and 2 of every group of 4 swapped -- the key order in which the softmax
// threads pack P (see the attention kernel).
bool encode_attn_v(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads);
// K operand of the attention: [heads][rows][64] bf16, one box per KV tile
bool encode_attn_k(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads);
// maps: q [heads][L][64]; k fresh and stale (box 128 rows x 64); v from encode_attn_v
cudaError_t launch_tc_attention(const TcAttnArgs& a, const CUtensorMap& mq, const CUtensorMap& mkf,
                                const CUtensorMap& mvf, const CUtensorMap& mks,
                                const CUtensorMap& mvs, cudaStream_t s);

}  // namespace dfp
