/*
 * dfp.h -- C ABI of the displaced-patch UNet layer step on one B200 (libdfp.so).
 *
 * The method (DistriFusion, CVPR 2024) splits the latent feature map into N row
 * patches.  Each patch computes fresh activations for its own rows; the context
 * it needs from the other patches is read from the previous denoising step:
 *   - conv3x3 halo rows      (DistriConv2dPP; "DistriFusion源码探秘" source
 *                             walkthrough, Patch Parallelism section, item 1)
 *   - self-attention K/V     (DistriSelfAttentionPP; same section, item 2)
 *   - GroupNorm statistics   (DistriGroupNorm; same section, item 3; the
 *                             "corrected asynchronous" default of the
 *                             --sync_mode flag, project README, Benchmarks)
 * The first steps run synchronously (project README, Overview (c); paper
 * reading blog, Implementation details).  Here all N patches run inside one
 * GPU and a double-buffered device-resident cache replaces the all_gather of
 * the multi-GPU original (walkthrough, forward-pass section; blog, Ablation).
 *
 * Conventions for every entry point
 *   - Returns a dfp_status; never aborts, never exits.  On failure the handle's
 *     dfp_last_error() text says why (a NULL handle gets a static message).
 *   - Argument checks run on the host before any launch.
 *   - Work is enqueued on the handle's CUDA stream; no call blocks on the device
 *     except dfp_step_host, dfp_synchronize, dfp_copy_out (host destination) and
 *     dfp_check_device.
 *   - Tensors are row-major.  The feature map is NHWC: [B, H, W, C] with B =
 *     dfp_config.batch images (B = 1: [H, W, C]).  Tokens of attention are the
 *     pixels of one image in row-major (h, w) order; L = H * W per image.
 *   - Patch p (0 <= p < N) of every image owns rows [p*H/N, (p+1)*H/N).  The images
 *     of a batch share the weights and the step schedule and nothing else: each has
 *     its own GroupNorm statistics, halo rows, K/V context and (transformer stage)
 *     cross-attention context.
 *   - One handle is not thread-safe; distinct handles are independent.
 */
#ifndef DFP_H
#define DFP_H

#if defined(__GNUC__)
#define DFP_API __attribute__((visibility("default")))
#else
#define DFP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dfp_ctx* dfp_handle;

typedef enum {
  DFP_OK = 0,
  DFP_E_ARG = 1,          /* a bad pointer, size, name, dtype or shape            */
  DFP_E_STATE = 2,        /* call out of order (e.g. displaced step, empty cache) */
  DFP_E_CUDA = 3,         /* a CUDA runtime/driver call or a kernel launch failed */
  DFP_E_NOMEM = 4,        /* device or host allocation failed                     */
  DFP_E_UNSUPPORTED = 5,  /* valid request the library does not implement         */
  DFP_E_DEVICE = 6        /* a kernel reported an error through the device flag   */
} dfp_status;

typedef enum { DFP_F32 = 0, DFP_BF16 = 1 } dfp_dtype;

typedef enum {
  DFP_BLOCK_RES_ATTN = 0,   /* GN+SiLU -> conv3x3 -> GN -> self-attention (Q,K,V,O) */
  DFP_BLOCK_SDXL_STAGE = 1, /* ResNet block + transformer blocks                     */
  /* A whole SDXL-shaped UNet (project README, Performance: SDXL, 50-step DDIM; source
   * walkthrough, Patch Parallelism: every conv, norm and attention layer of the UNet is
   * wrapped): latent [H, W, 4]; levels H, H/2, H/4 with widths C, 2C, 4C; one ResNet block
   * per level (timestep embedding added after its first conv), transformer blocks at the
   * two lower levels, stride-2 convs down, nearest x2 + conv up, skip concatenation;
   * every conv, GroupNorm and self-attention displaced, the same N row patches at every
   * level.  A step is one UNet evaluation at the timestep set by dfp_set_timestep; its
   * output (dfp_output) is the predicted noise [H*W, 4] bf16.  Weights: the names and
   * PyTorch shapes of the workload's generator (time_embedding.linear_{1,2}, conv_in,
   * down{0,1,2}.resnet.*, down{1,2}.xf.*, down{0,1}.downsample, up{1,0}.upsample,
   * up1.resnet.*, up1.xf.*, up0.resnet.*, norm_out, conv_out, and "context").  bf16,
   * batch 1, heads * 64 == C, H a multiple of 4 N, W of 4, 6 C <= 4096. */
  DFP_BLOCK_UNET = 2
} dfp_block;

typedef enum {
  /* est_p = mean_j m_j(t-1) + (m_p(t) - m_p(t-1)), m = (E[x], E[x^2]) per (patch, group) */
  DFP_GN_CORRECTED = 0,
  /* est_p = (m_p(t) + sum_{j != p} m_j(t-1)) / N */
  DFP_GN_STALE_OTHERS = 1,
  /* GroupNorm-only variants of the pages' --sync_mode flag (project README, Benchmarks),
   * conv halos and attention K/V still displaced:
   * est_p = mean_j m_j(t): this step's full-map statistics on displaced steps too */
  DFP_GN_SYNC = 2,
  /* est_p = m_p(t): patch-local statistics on displaced steps (sync steps stay exact) */
  DFP_GN_SEPARATE = 3
} dfp_gn_mode;

typedef enum {
  DFP_CTX_DISPLACED = 0,  /* the method: stale context on displaced steps          */
  DFP_CTX_NAIVE = 1       /* naive-patch baseline: no cross-patch context at all
                             (project README, Overview (b))                        */
} dfp_context;

typedef struct {
  int H, W, C;          /* feature map; C = heads * head_dim                          */
  int n_patches;        /* N: H % N == 0; (H/N)*W % 8 == 0                            */
  int gn_groups;        /* G: C % G == 0                                               */
  float gn_eps;         /* GroupNorm epsilon                                           */
  int heads, head_dim;  /* head_dim must be 64                                         */
  dfp_dtype dtype;      /* storage and MMA operand type; statistics/accumulation fp32 */
  dfp_block block;
  dfp_gn_mode gn_mode;
  dfp_context context;
  int n_xformer, ffn_inner, ctx_len, ctx_dim;  /* DFP_BLOCK_SDXL_STAGE only           */
  /* Images per step, 1..8 (0 counts as 1).  2 is the classifier-free-guidance batch
   * (conditional and unconditional branch; guidance scale 5 by default) that the
   * project README's latency benchmark splits across GPU groups unless
   * --no_split_batch is given (README, Benchmarks: COCO quality and Latency).  On one
   * GPU the images run through the same launches, every image-specific step indexed
   * by image.  The SIMT family (fp32) needs batch * n_patches * gn_groups <= 512. */
  int batch;
} dfp_config;

typedef struct {
  const char* name;          /* PyTorch module naming, e.g. "conv1.weight"            */
  const void* ptr;           /* host or device pointer to the values, contiguous       */
  int on_device;             /* 1 if ptr is a device pointer                           */
  dfp_dtype dtype;           /* element type at ptr                                    */
  int ndim;
  const long long* shape;    /* PyTorch layout: conv [Cout,Cin,3,3], linear [out,in]   */
} dfp_tensor;

/* Create a handle for one layer (or stage) configuration and allocate its device
 * buffers: the double-buffered context caches, intermediates and the output.  The
 * configuration plays the part of the pages' DistriConfig (project README, Usage:
 * height, width, warmup_steps; Benchmarks: --sync_mode, --parallelism naive_patch),
 * reduced to one layer: the map size, the patch count, the GroupNorm merge mode and
 * the context mode; the caller passes which steps are synchronous (dfp_step).
 * cuda_stream: a cudaStream_t (NULL = legacy default stream); all work of this
 * handle is enqueued on it.  *out receives the handle (NULL on failure).
 * Errors: DFP_E_ARG for invalid sizes (see dfp_config), DFP_E_UNSUPPORTED for a
 * block type not built, DFP_E_NOMEM / DFP_E_CUDA for allocation failures. */
DFP_API dfp_status dfp_create(const dfp_config* cfg, void* cuda_stream, dfp_handle* out);

/* Copy the weights in (host or device source; the library keeps its own re-laid
 * copy, the caller's memory may be freed after the call returns).  The counterpart of
 * the pages' from_pretrained (project README, Usage: the SDXL pipeline loads its fp16
 * weights) for one layer, with the PyTorch module names the wrapped layers keep
 * (source walkthrough, Patch Parallelism section: DistriConv2dPP, DistriGroupNorm and
 * DistriSelfAttentionPP replace the UNet's conv, norm and attention modules in place).  Every weight
 * of the block must be named exactly once across calls before the first step;
 * names for DFP_BLOCK_RES_ATTN: gn1.weight gn1.bias conv1.weight conv1.bias
 * gn2.weight gn2.bias attn.to_q.weight attn.to_k.weight attn.to_v.weight
 * attn.to_out.weight attn.to_out.bias.  DFP_BLOCK_SDXL_STAGE: resnet.{norm1,conv1,
 * norm2,conv2}.{weight,bias}, xf<b>.{norm1,norm2,norm3}.{weight,bias},
 * xf<b>.attn1.to_{q,k,v,out}.weight, xf<b>.attn1.to_out.bias, the same for attn2
 * (to_k / to_v are [C, ctx_dim]), xf<b>.ff.proj.{weight,bias} ([2F, C], GEGLU value
 * rows then gate rows), xf<b>.ff.out.{weight,bias}, and "context": the text context,
 * [ctx_len, ctx_dim] for one image or [B, ctx_len, ctx_dim], one per image, for a
 * batch (conditional and unconditional context of the guidance batch).  Blocks
 * until the copies are done.
 * Errors: DFP_E_ARG for an unknown name, wrong shape or dtype. */
DFP_API dfp_status dfp_load_weights(dfp_handle h, const dfp_tensor* w, int n);

/* One layer step (project README, Overview (c): every patch computes its own rows
 * fresh and reuses the previous step's activations of the other patches as context;
 * the first steps are synchronous -- paper reading blog, Implementation details: step 0
 * plus the warm-up steps; source walkthrough, forward-pass section: split the input
 * into patches, compute, gather the patch outputs into the full map).
 * x: caller-owned device pointer [B, H, W, C] of the config dtype,
 * contiguous; it must stay valid until the stream work completes.
 * step: 0 starts a new run and must be synchronous (is_sync = 1); otherwise
 * step must equal the previous step + 1.  is_sync = 1 uses fresh context
 * everywhere (exact full-image layer); is_sync = 0 uses the previous step's
 * cached context for every cross-patch read.  Every step refreshes the caches.
 * Asynchronous: returns once the kernels are enqueued.
 * Errors: DFP_E_STATE (order, weights missing), DFP_E_ARG, DFP_E_CUDA. */
DFP_API dfp_status dfp_step(dfp_handle h, const void* x, int step, int is_sync);

/* Patch parallelism across GPUs (project README, Overview (c): one patch per device, the
 * other patches' activations of the previous step as context, exchanged asynchronously;
 * paper reading blog, Ablation: patch parallelism gathers activations with AllGather).
 * A rank holds a handle for the whole map and computes only its patches [p_begin, p_end)
 * on displaced steps; between steps the ranks all-gather what each computed -- this
 * step's K/V rows, GroupNorm moments, the boundary rows of the conv input and the output
 * rows -- into every rank's buffers (dfp_context_buffer), so the next displaced step finds
 * the other patches' context of the previous step in place.  Synchronous steps run the
 * whole map on every rank (dfp_step).  Requirements: DFP_BLOCK_RES_ATTN, bf16, the
 * tensor-core kernels, batch 1, a gn_mode that needs no statistics of other patches of
 * the same step (not DFP_GN_SYNC), step >= 1 following the previous step; else
 * DFP_E_UNSUPPORTED / DFP_E_STATE / DFP_E_ARG (bad range).  Only the range's rows of the
 * outputs are written: y, this step's K/V, moments and slab rows of the range; the
 * conv input's halo rows at the range's ends must hold the neighbours' boundary rows of
 * the previous step (the exchange puts them there).  Asynchronous like dfp_step. */
DFP_API dfp_status dfp_step_patches(dfp_handle h, const void* x, int step, int p_begin, int p_end);

/* Device pointer and size of a library-owned buffer that the patch-parallel exchange
 * reads and fills (no counterpart in the pages beyond the all_gather buffers).  parity =
 * step & 1 selects the step's buffer of the alternating pairs.  Names and layouts:
 * "k", "v"      [heads][B*L][64] the step's keys / values
 * "mom1","mom2" [B*N][G][2] fp32 (mean, variance) of GN1 / GN2 per (patch, group)
 * "slab"        [B*N][R+2][W][C] the conv input with one halo row above / below each patch
 * "y"           [B*L][C] the block output (parity ignored)
 * Valid until dfp_destroy.  DFP_E_ARG for an unknown name or a parity other than 0 / 1. */
DFP_API dfp_status dfp_context_buffer(dfp_handle h, const char* name, int parity, void** ptr, long long* bytes);

/* The timestep the next DFP_BLOCK_UNET step embeds (DFP_E_UNSUPPORTED for other blocks). */
DFP_API dfp_status dfp_set_timestep(dfp_handle h, float timestep);

/* The DDIM loop around a DFP_BLOCK_UNET handle (paper reading blog, Implementation details:
 * 50-step DDIM, the first steps synchronous; project README, Performance): deterministic
 * DDIM (eta = 0) on a scaled-linear beta schedule of n_train training steps (beta_i =
 * (sqrt(beta_start) + i (sqrt(beta_end) - sqrt(beta_start)) / (n_train - 1))^2), visiting
 * timesteps (n_steps - 1 - k) floor(n_train / n_steps) + 1 for k = 0 .. n_steps - 1; step k runs the
 * UNet at step index k, synchronous for k < n_sync, then x <- sqrt(ab') (x - sqrt(1 - ab) eps)
 * / sqrt(ab) + sqrt(1 - ab') eps in fp32.  x_T, x_out: device fp32 [H, W, 4] (may be the
 * same buffer).  Asynchronous on the handle's stream.  DFP_E_ARG unless n_steps >= 1,
 * 1 <= n_sync, n_steps <= n_train <= 100000 and 0 < beta_start < beta_end < 1. */
DFP_API dfp_status dfp_ddim_sample(dfp_handle h, const float* x_T, int n_steps, int n_sync, int n_train,
                                   float beta_start, float beta_end, float* x_out);

/* Same step with HOST buffers: copies x_host ([B,H,W,C], config dtype; pinned
 * memory gives asynchronous copies) to the device, runs the step, copies the
 * output to y_host and waits for the stream. */
DFP_API dfp_status dfp_step_host(dfp_handle h, const void* x_host, void* y_host, int step, int is_sync);

/* Pipelined form of dfp_step_host (no counterpart in the pages: a serving loop).  Enqueues
 * the copy of x_host to the device on a copy stream, the step on the handle's stream and
 * the copy of its output to y_host on a second copy stream, then returns without waiting:
 * consecutive calls overlap one step's copies with the neighbouring steps' kernels.
 * x_host and y_host must be pinned (page-locked) for the copies to overlap.  The caller
 * must not modify x_host or read y_host of a call until dfp_synchronize returns (or, when
 * alternating two host buffers, until two calls later plus dfp_synchronize); device-side
 * buffers are double-buffered and ordered by events.  Errors are as for dfp_step. */
DFP_API dfp_status dfp_step_host_async(dfp_handle h, const void* x_host, void* y_host, int step, int is_sync);

/* Wait until every step and copy enqueued on the handle (its stream and the copy streams
 * of dfp_step_host_async) has completed. */
DFP_API dfp_status dfp_synchronize(dfp_handle h);

/* Self-test of failure detection (no counterpart in the pages).  Every spin-wait in the
 * library's kernels is bounded: after ~4e9 SM clocks (about 2 s) it records an error code in
 * a device word and the kernel winds down, so a lost arrival surfaces as DFP_E_DEVICE from
 * dfp_check_device instead of a hung GPU.  This call runs one thread that waits, through the
 * same code, on an mbarrier nothing arrives on (on the current device and the legacy default
 * stream), and returns the code it recorded in *code_out (1: a TMA stage never filled) and
 * the wait's length in SM clocks in *cycles_out (may be NULL).  The context stays usable.
 * Blocks for the length of the wait.  DFP_E_CUDA if a CUDA call fails. */
DFP_API dfp_status dfp_selftest_wait_timeout(int* code_out, long long* cycles_out);

/* Self-test of the softmax's polynomial exponential (no counterpart in the pages).  Part of
 * the attention's exponentials run on the FMA pipe as 2^x = 2^j * p(f), j = rint(x),
 * |f| <= 1/2, p the degree-3 minimax fit of 2^f in relative error (max 7.48e-5), x clamped
 * to >= -125.  This call evaluates that same device code: y[i] = 2^x[i] as fp32 and, if
 * y_bf16 is not NULL, as the truncated bf16 the softmax stores.  x, y: device fp32 [n];
 * y_bf16: device bf16 [n], 4-byte aligned, or NULL.  Enqueued on cuda_stream (a
 * cudaStream_t; NULL = legacy default stream).  DFP_E_ARG for n < 0, n > 2^30, NULL x / y
 * (n > 0) or a misaligned y_bf16; DFP_E_CUDA if the launch fails. */
DFP_API dfp_status dfp_selftest_exp2_poly(const float* x, float* y, void* y_bf16, int n, void* cuda_stream);

/* Library-owned device pointer to the last step's output [B*H*W, C] (config dtype):
 * the N patch outputs assembled into the full map, as the wrapped UNet's forward pass
 * gathers them (source walkthrough, forward-pass section); valid until the next
 * dfp_step or dfp_destroy. */
DFP_API dfp_status dfp_output(dfp_handle h, const void** y);

/* Copy an internal buffer of the last step to dst (device or host pointer,
 * dst_bytes must equal the buffer size, see dfp_buffer_bytes).  Names:
 * "y" output [B*L,C]; "slab" GN1+SiLU output with its halo rows [B*N,H/N+2,W,C];
 * "h" conv output [B,H,W,C];
 * "t" GN2 output [B,H,W,C]; "q","k","v" this step's projections [heads,B*L,64];
 * "o" attention output [B*L,C]; "gn1","gn2" per-(image,patch,group) (mean, rstd)
 * fp32 [B*N,G,2].  Stream-ordered; a host dst makes the call wait for the stream. */
DFP_API dfp_status dfp_copy_out(dfp_handle h, const char* name, void* dst, long long dst_bytes);
DFP_API dfp_status dfp_buffer_bytes(dfp_handle h, const char* name, long long* bytes);

/* Wait for the stream and read the device error flag that bounded waits inside
 * the kernels set instead of hanging.  DFP_OK if clean, DFP_E_DEVICE otherwise (the
 * flag is cleared and the GroupNorm grid-barrier counters are re-armed, so further
 * steps run normally), DFP_E_CUDA if a launch failed asynchronously. */
DFP_API dfp_status dfp_check_device(dfp_handle h);

/* Number of kernel launches one dfp_step of this handle enqueues. */
DFP_API int dfp_launches_per_step(dfp_handle h);

/* Host-side check of the tensor-core attention's work split (no counterpart in the
 * pages; no GPU needed).  The units of work are (head, image patch, query-tile pair), each
 * a list of KV tiles, in head-major order.  When the K/V the list reads (every head, fresh
 * and stale rows) exceed kv_budget_bytes (< 0: the kernel's own budget, 48 MB), the first
 * whole_rounds * ctas units are dealt whole, unit k * ctas + c to CTA c, so the CTAs' units
 * in flight share one or two heads' K/V in L2; the remaining units (the tail) are cut into
 * `ctas` contiguous ranges of KV tiles (stream-K).  Walks every CTA's pieces as the kernel
 * does and checks: every CTA has work and every piece stays inside its unit; every unit is
 * covered once; a pair cut between CTAs has its first KV tiles at the end of one CTA's
 * tail range (that CTA merges) and its other pieces each at the start of a range; the
 * kernel's publisher and flag warps predict exactly those pieces; the softmax's per-piece
 * table of partial tiles gives every KV tile the valid key count of the TMA warp's per-tile
 * walk.  L tokens per image in
 * n_patches patches of Lp tokens; mode 0 sync, 1 displaced, 2 naive, 3 cross-attention
 * (Lp = L, n_patches = 1, kv_len context tokens).  Only the query patches [p_begin, p_end)
 * of the image-major patch list are listed (p_begin = p_end = 0: all), as for a
 * patch-parallel rank's range.  Returns 0 if every property holds, else the number of the
 * first that fails (1: bad arguments). */
DFP_API int dfp_attention_schedule_check(int L, int Lp, int n_patches, int heads, int mode, int kv_len, int images,
                                         int ctas, int p_begin, int p_end, long long kv_budget_bytes);

/* Launch overlap between the kernels of a step (no counterpart in the pages; on by
 * default): every tensor-core-family kernel is launched with programmatic stream
 * serialization, so its blocks are scheduled, and set up their barriers and tensor
 * memory, while the previous kernel on the stream finishes; each waits for that kernel
 * to complete before it touches device memory, so results do not change.  enable = 0
 * launches every kernel only after its predecessor has completed.  DFP_E_ARG unless
 * enable is 0 or 1. */
DFP_API dfp_status dfp_set_launch_overlap(dfp_handle h, int enable);

/* Choose the kernel family for the contractions: 0 = tcgen05/TMA tensor-core
 * kernels (default for bf16), 1 = SIMT CUDA-core kernels (the only family for
 * fp32).  Returns DFP_E_UNSUPPORTED for tensor cores with fp32. */
DFP_API dfp_status dfp_set_kernel_family(dfp_handle h, int family);

/* Work split of the tensor-core attention (no counterpart in the pages; a tuning knob): when
 * the K/V bytes one launch reads (every head, fresh and stale rows) exceed `bytes`, the launch
 * deals rounds of whole (head, patch, query-tile pair) units to its CTAs, so the CTAs in
 * flight share one or two heads' K/V in L2; below it, every KV tile is split stream-K.
 * 0 (the default) takes the kernel's own budget, 48 MB; 1 forces the whole-unit rounds
 * wherever there are at least as many units as CTAs.  Results do not depend on it beyond
 * rounding order.  DFP_E_ARG for bytes < 0. */
DFP_API dfp_status dfp_set_attention_kv_budget(dfp_handle h, long long bytes);

/* Per-kernel timing.  With profiling on, dfp_step brackets every kernel launch
 * with CUDA events recorded on the handle's stream.  dfp_kernel_times waits for
 * the last step's events and writes up to max_n durations (milliseconds) and the
 * matching static kernel names; it returns the number of durations written (at
 * most max_n; 0 when profiling is off, no step ran or the step made more than 127
 * launches), or -1 on a CUDA error. */
DFP_API dfp_status dfp_set_profiling(dfp_handle h, int enable);
DFP_API int dfp_kernel_times(dfp_handle h, float* ms, const char** names, int max_n);

/* GroupNorm over N row patches with the displaced (stale/fresh) statistics merge,
 * normalise and optional SiLU, as ONE call that allocates no memory.  The paper
 * has no counterpart to this entry point: it exists for callers that cannot
 * allocate device memory when they need the op (a fixed memory pool that bans the
 * CUDA allocator, a pre-planned or capped memory region, a latency-critical host
 * path that must not take allocator locks).
 *   x, y            device [H, W, C] of dtype (input, output; the two ranges must not
 *                   overlap: the op does not run in place)
 *   gamma, beta     device fp32 [C]
 *   stale_moments   device fp32 [N, G, 2] (mean, variance) per (patch, group) of the
 *                   previous step -- the previous call's fresh_moments -- or NULL for a
 *                   synchronous step (exact full-map statistics).  It is read after
 *                   this call's fresh_moments are written, so the two must be distinct
 *                   buffers: alternate two buffers between consecutive calls
 *   fresh_moments   device fp32 [N, G, 2], out: this call's moments (mean, variance):
 *                   the merge rules of dfp_gn_mode are evaluated on these central
 *                   moments (the same value as on (E[x], E[x^2]) in exact arithmetic,
 *                   without the fp32 cancellation of E[x^2] - mean^2 at large means)
 *   mean_rstd       device fp32 [N, G, 2], out: the (mean, 1/std) applied, or NULL;
 *                   must not overlap the two moment buffers
 * Overlapping buffers among these return DFP_E_ARG before anything is enqueued.
 *   cuda_stream     cudaStream_t the work is enqueued on (asynchronous)
 * Scratch comes from a fixed 256 KiB array in the library's device memory (held by
 * every GPU that loads the library until exit).  The first call on a device, with
 * that device current, looks up the array's device address; make that first call
 * before any stream capture begins.  All calls share the array and it keeps the
 * last call's contents (the counter that must start at zero is cleared by every
 * call), so calls that overlap on the GPU race.  Limits: n_patches * groups <= 256
 * and the (patch, group, block) partial sums <= 64960 floats (about
 * n_patches * groups * 2 * min(148 / n_patches + 1, pixels per patch / 16)); larger
 * requests return DFP_E_ARG with the reason in
 * dfp_group_norm_noalloc_error().  Never calls cudaMalloc or cudaFree. */
DFP_API dfp_status dfp_group_norm_noalloc(const void* x, void* y, dfp_dtype dtype, int H, int W, int C,
                                          int n_patches, int groups, float eps, const float* gamma,
                                          const float* beta, const float* stale_moments, dfp_gn_mode mode,
                                          int apply_silu, float* fresh_moments, float* mean_rstd,
                                          void* cuda_stream);
DFP_API const char* dfp_group_norm_noalloc_error(void);

/* Free everything the handle owns (waits for its stream first).  NULL is a no-op. */
DFP_API dfp_status dfp_destroy(dfp_handle h);

/* Text of the last error of h (or of the last failed dfp_create when h is NULL). */
DFP_API const char* dfp_last_error(dfp_handle h);

#ifdef __cplusplus
}
#endif
#endif /* DFP_H */
