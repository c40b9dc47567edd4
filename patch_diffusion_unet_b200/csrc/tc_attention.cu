// Displaced self-attention on tcgen05 / TMEM / TMA (sm_100a), bf16 operands, fp32
// softmax statistics and accumulation, head width 64.
//
// DistriSelfAttentionPP ("DistriFusion源码探秘" source walkthrough, Patch
// Parallelism section item 2): the queries of patch p attend to all L tokens; the
// K/V of its own rows are this step's, those of every other patch come from the
// previous step's cache (project README, Overview (c): activations of the
// previous step are reused).  The KV loop walks a list of segments:
//   sync       [0, L) fresh
//   displaced  own patch fresh, then [0, p*Lp) stale, then [(p+1)*Lp, L) stale
//   naive      own patch fresh only (the naive-patch baseline, README Overview (b))
// Segment ends need not be multiples of the 128-key tile: columns past a
// segment's end are masked.  A batch of images (the guidance batch) is images x N
// patches: Q, O, K and V hold the images one after another (rows img * L + token;
// cross-attention contexts at img * kv_stride), and a patch reads only the keys of
// its own image.
//
// CTA layout (640 threads, five warpgroups): two softmax groups of 8 warps, each
// owning one 128-query tile.  Warps w and w+4 of a group read the same 32 TMEM
// lanes (query rows); the first takes key columns 0-63, the second 64-127, and
// they exchange their partial row maxima through shared memory -- at head width
// 64 the softmax work per tile is large next to the MMAs, and two threads per
// row double the latency hiding.  In the fifth warpgroup warp 16 issues TMA
// (the Q-tile pair of each piece into a double buffer, K/V through 3-stage rings
// shared by the groups) and warp 17 issues the MMAs from one elected lane; warps 18
// and 19 publish and acquire the flags of cut query-tile pairs (below); this
// warpgroup hands most of its registers to the softmax warpgroups (setmaxnreg).
// Per KV tile j and group g:
//   S_g = Q_g K_j^T            tcgen05.mma, A and B from shared memory, D in TMEM
//   P_g = exp2(S_g * c - m_g)  softmax threads, written back over S_g in TMEM as
//                              bf16 pairs (byte-permute truncation)
//   O_g += P_g [V_j | 1]       tcgen05.mma with A = P from TMEM; the ones block
//                              appended to V makes the tensor core produce the row
//                              sums of the same truncated P, so the truncation
//                              cancels in O / l
// The groups ping-pong: the MMAs of one group run while the other computes its
// softmax.  The running maximum is lazy: O and l are rescaled (in TMEM) only
// when a row's maximum grows by more than 2^8.  Part of the exponentials run as
// a polynomial on the FMA pipe (range reduction to 2^j * 2^f, |f| <= 1/2, with a
// degree-3 minimax polynomial for 2^f, max relative error 7.48e-5; exp2_poly.cuh)
// to offload the MUFU unit.
//
// Work split: a unit of work is the KV list of one Q-tile pair of one (head, patch), the
// patches of all images of the batch in one head-major list.  When the K and V the list
// reads do not fit in L2 (the 240 x 240 map reads 295 MB of them), rounds of whole units
// are dealt one per CTA, unit k * G + c to CTA c: the units in flight are then neighbours
// in the list and share one or two heads' K and V in L2.  The rest (the tail; all of the
// list for smaller maps) is stream-K: its KV tiles are cut into one contiguous range per
// SM, so every CTA gets the same number of KV tiles whatever the number of pairs.  A CTA
// walks its work as a sequence of pieces (a whole unit, or the part of one pair's KV list
// that falls in its tail range): the first piece of its tail range, then its whole units,
// then the rest of its tail range.
// Q is double-buffered so the next piece's queries load while the current piece
// runs, and the K/V ring does not drain between pieces.  A pair whose KV list is
// cut between CTAs is finished by the CTA holding its first KV tiles (the end of that
// CTA's tail range, so processed last there, after the other pieces, which open their
// CTAs' sequences):
// the other pieces leave their unnormalised O, running max and row sum in a per-CTA
// slot and publish a flag; the first piece merges them with its own O in KV order,
// so the result does not depend on timing.  Only a merging piece ever waits, and only
// for pieces that wait for nothing: with one resident CTA per SM this cannot cycle.
#include <algorithm>
#include <atomic>
#include <vector>

#include "dfp_common.cuh"
#include "exp2_poly.cuh"
#include "kernels.h"

namespace dfp {

namespace {

constexpr int kThreads = 640;
constexpr int kWarpTma = 16, kWarpMma = 17;
constexpr int kTile = 128;
constexpr uint32_t kTileBytes = 128 * 64 * 2;   // one 128 x 64 bf16 tile
constexpr int kStages = 3;
constexpr int kOCols = 80;                      // 64 outputs + 16 row-sum columns
constexpr uint32_t kTmemCols = 512;             // S/P: [128g, 128g+128), O: [256+128g, +80)
constexpr float kRescale = 8.f;                 // lazy rescale threshold (log2 units)
constexpr int kPolyPer8 = 2;
// registers per thread after the split: 128 x 64 + 512 x 104 = 640 x 96 (the launch's)
constexpr int kRegsTmaMma = 64, kRegsSoftmax = 104;                    // of every 8 columns, this many use the polynomial

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// KV tiles of one query-tile pair of patch p.  The KV list walks the segments
//   sync       [0, L) fresh
//   cross      [0, kv_len) (the fixed context)
//   naive      own patch fresh only
//   displaced  own patch fresh, then [0, p*Lp) stale, then [(p+1)*Lp, L) stale
// each rounded up to whole 128-key tiles (the columns past a segment's end are masked).
__host__ __device__ __forceinline__ int unit_tiles(int mode, int p, int Lp, int L, int kv_len) {
  if (mode == kAttnSync) return cdiv(L, kTile);
  if (mode == kAttnCross) return cdiv(kv_len, kTile);
  int t = cdiv(Lp, kTile);
  if (mode == kAttnDisplaced) t += cdiv(p * Lp, kTile) + cdiv(L - (p + 1) * Lp, kTile);
  return t;
}

// tile j of patch p's KV list -> (stale?, first key row, valid keys)
__host__ __device__ __forceinline__ void tile_src(int mode, int p, int Lp, int L, int kv_len, int j, int& stale,
                                         int& row, int& valid) {
  stale = 0;
  if (mode == kAttnSync || mode == kAttnCross) {
    row = j * kTile;
    valid = min(kTile, (mode == kAttnSync ? L : kv_len) - row);
    return;
  }
  const int own = cdiv(Lp, kTile);
  if (j < own) {
    row = p * Lp + j * kTile;
    valid = min(kTile, Lp - j * kTile);
    return;
  }
  stale = 1;
  j -= own;
  const int t1 = cdiv(p * Lp, kTile);
  if (j < t1) {
    row = j * kTile;
    valid = min(kTile, p * Lp - row);
    return;
  }
  row = (p + 1) * Lp + (j - t1) * kTile;
  valid = min(kTile, L - row);
}

// Only the last tile of each of the (at most three) segments of patch p's KV list can be
// partial: their indices in the list (-1: no such segment) and valid key counts, the same
// counts tile_src gives, taken once per piece instead of per tile.
struct TileEnds {
  int e0, v0, e1, v1, e2, v2;
};
__host__ __device__ __forceinline__ TileEnds tile_ends(int mode, int p, int Lp, int L, int kv_len) {
  TileEnds t{-1, kTile, -1, kTile, -1, kTile};
  if (mode == kAttnSync || mode == kAttnCross) {
    const int len = mode == kAttnSync ? L : kv_len;
    const int T = cdiv(len, kTile);
    t.e0 = T - 1;
    t.v0 = len - (T - 1) * kTile;
    return t;
  }
  const int own = cdiv(Lp, kTile);
  t.e0 = own - 1;
  t.v0 = Lp - (own - 1) * kTile;
  if (mode == kAttnDisplaced) {
    const int t1 = cdiv(p * Lp, kTile), t2 = cdiv(L - (p + 1) * Lp, kTile);
    if (t1 > 0) {
      t.e1 = own + t1 - 1;
      t.v1 = p * Lp - (t1 - 1) * kTile;
    }
    if (t2 > 0) {
      t.e2 = own + t1 + t2 - 1;
      t.v2 = L - (p + 1) * Lp - (t2 - 1) * kTile;
    }
  }
  return t;
}

// The unit list: head-major over (head, query patch, Q-tile pair) -- patch pg = img * N + p
// over the images' patches, so Q and O rows start at pg * Lp -- unit (head, pg, pair) has
// unit_tiles(pg % N) KV tiles.  Only the query patches [p_lo, p_hi) are listed (all of them
// unless a patch-parallel rank computes a range).
// All schedule arithmetic is 32-bit: the launcher checks total tiles * ctas < 2^31.
struct Unit {
  int p, head, pair, T;   // p: patch over the batch (img * N + patch within the image)
  int U0;                 // tail units: tail index of the unit's first tile; whole units: -1
};
__host__ __device__ __forceinline__ int patch_tiles(const TcAttnArgs& a, int p) {
  return unit_tiles(a.mode, p % a.N, a.Lp, a.L, a.kv_len);
}
// unit `idx` of the list
__host__ __device__ __forceinline__ Unit unit_at(const TcAttnArgs& a, int n_pairs, int idx) {
  const int per_head = (a.p_hi - a.p_lo) * n_pairs;
  Unit u{};
  u.head = idx / per_head;
  const int r = idx - u.head * per_head;
  u.p = a.p_lo + r / n_pairs;
  u.pair = r - (r / n_pairs) * n_pairs;
  u.T = patch_tiles(a, u.p);
  u.U0 = -1;
  return u;
}
// the unit holding tail tile x, its U0 the tail index of its first tile
__host__ __device__ __forceinline__ Unit locate(const TcAttnArgs& a, int n_pairs, int x) {
  const int X = x + a.tail_base;          // index among all tiles of the list
  Unit u{};
  u.head = X / a.head_tiles;
  int base = u.head * a.head_tiles;
  for (int p = a.p_lo; p < a.p_hi; ++p) {
    const int T = patch_tiles(a, p);
    if (X < base + T * n_pairs) {
      u.p = p; u.pair = (X - base) / T; u.T = T;
      u.U0 = base + u.pair * T - a.tail_base;
      return u;
    }
    base += T * n_pairs;
  }
  return u;   // not reached for x < total
}
// the tail unit after u (no division: pairs, then patches, then heads)
__host__ __device__ __forceinline__ void advance(const TcAttnArgs& a, int n_pairs, Unit& u) {
  u.U0 += u.T;
  if (++u.pair == n_pairs) {
    u.pair = 0;
    if (++u.p == a.p_hi) {
      u.p = a.p_lo;
      ++u.head;
    }
    u.T = patch_tiles(a, u.p);
  }
}
// the CTA whose tail range [c*TT/G, (c+1)*TT/G) holds tail tile x
__host__ __device__ __forceinline__ int cta_of(int x, int TT, int G) { return ((x + 1) * G + TT - 1) / TT - 1; }
__host__ __device__ __forceinline__ int range_start(int c, int TT, int G) { return c * TT / G; }

// The pieces of CTA c, in order (phase 0, 1, 2): the first piece of its tail range [X0, X1)
// (the tail: the units from whole_rounds * G on, their tiles numbered from 0), its
// whole_rounds whole units (units k * G + c, one piece each, merged by nobody), then the
// rest of its tail range, one piece per unit the range touches.  With every CTA on whole
// units at once the units in flight are consecutive in the list and share one or two
// heads' K and V in L2 whatever the map size; a piece that continues a pair another CTA
// started opens the sequence, so its partial is published early, and a pair this CTA
// merges ends it.
struct Walk {
  Unit tu;       // the tail unit last walked (the tail resumes after it)
  int j0, n;     // the piece: its unit's KV tiles [j0, j0 + n)
  int k;         // the piece's index in the CTA's sequence
  int x;         // the tail tile after the last tail piece walked
  int kw;        // whole units walked (phase 1: the current one)
  int phase;
};
struct Sched {
  int n_pairs, G, c, X0, X1;
};
// the unit of the current piece
__host__ __device__ __forceinline__ Unit walk_unit(const TcAttnArgs& a, const Sched& s, const Walk& w) {
  return w.phase == 1 ? unit_at(a, s.n_pairs, w.kw * s.G + s.c) : w.tu;
}
__host__ __device__ __forceinline__ void walk_whole(const TcAttnArgs& a, const Sched& s, Walk& w) {
  w.j0 = 0;
  w.n = unit_at(a, s.n_pairs, w.kw * s.G + s.c).T;
}
__host__ __device__ __forceinline__ bool walk_tail_next(const TcAttnArgs& a, const Sched& s, Walk& w) {
  if (w.x >= s.X1) return false;
  advance(a, s.n_pairs, w.tu);
  w.j0 = 0;
  w.n = min(w.tu.U0 + w.tu.T, s.X1) - w.x;
  w.x += w.n;
  return true;
}
__host__ __device__ __forceinline__ bool walk_first(const TcAttnArgs& a, const Sched& s, Walk& w) {
  w.k = 0;
  w.kw = 0;
  w.x = s.X0;
  if (s.X0 < s.X1) {
    w.tu = locate(a, s.n_pairs, s.X0);
    w.j0 = s.X0 - w.tu.U0;
    w.n = min(w.tu.U0 + w.tu.T, s.X1) - s.X0;
    w.x = s.X0 + w.n;
    w.phase = 0;
    return true;
  }
  if (a.whole_rounds > 0) {
    w.phase = 1;
    walk_whole(a, s, w);
    return true;
  }
  return false;
}
__host__ __device__ __forceinline__ bool walk_next(const TcAttnArgs& a, const Sched& s, Walk& w) {
  ++w.k;
  if (w.phase == 0 && a.whole_rounds > 0) {
    w.phase = 1;
    walk_whole(a, s, w);
    return true;
  }
  if (w.phase == 1 && ++w.kw < a.whole_rounds) {
    walk_whole(a, s, w);
    return true;
  }
  w.phase = 2;
  return walk_tail_next(a, s, w);
}
// KV tiles of CTA c in all
__host__ __device__ __forceinline__ int cta_tiles(const TcAttnArgs& a, const Sched& s) {
  int t = s.X1 - s.X0;
  for (int k = 0; k < a.whole_rounds; ++k) t += unit_at(a, s.n_pairs, k * s.G + s.c).T;
  return t;
}

__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// upper halves of two fp32 words -> one bf16 pair (lo = a, hi = b): truncation
__device__ __forceinline__ uint32_t pack_trunc(float a, float b) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(__float_as_uint(a)), "r"(__float_as_uint(b)));
  return r;
}

__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16x64b shapes: a warp reads / writes 16 TMEM lanes; lane t of the warp holds row
// 8*(t%2) + t/4 of those 16 and, per 2-column repeat r, column 2r + (t/2)%2.
__device__ __forceinline__ void tmem_ld_16x64b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x64b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_16x64b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.16x64b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_16x64b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.16x64b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Named barrier that also ORs a predicate over the participating threads: every
// thread leaves with the same answer, so a group can give up collectively.
__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(n) : "memory");
  return r != 0;
}
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// End of a piece for one softmax group: this thread's half row of O (32 columns)
// and the row sum, normalised into the output, or -- for a pair cut between CTAs --
// merged.  The pieces of a cut pair lie in consecutive CTAs' ranges; the first CTA's
// piece (the pair's first KV tiles) is the end of that CTA's range, so it is processed
// last there, after the later pieces, which open their CTAs' ranges.  That CTA merges:
// the later pieces leave their unnormalised O, running max and row sum in their CTA's
// slot and publish a flag (a release store of the launch's epoch, no round trip); the
// first piece waits for the flags (already set, as a rule) and merges in KV order, its
// own O straight from TMEM.  O streams through 8-column chunks so the epilogue needs
// few registers; it is out of line so that none of them count against the KV loop.
// Returns false if the final P V never completed or a merge waited in vain.
__device__ __noinline__ bool piece_epilogue(const TcAttnArgs& a, const Unit& u, uint32_t tO, uint32_t o_bar,
                                               uint32_t o_parity, float m_used, int g, int half, int row,
                                               int c, uint32_t pub_bar, uint32_t mrg_bar,
                                               const volatile int* merge_fail) {
  const int TT = a.total_tiles, G = gridDim.x;
  const bool have = mbar_wait(o_bar, o_parity, a.err, kErrWaitAttnO);
  float l = 1.f;
  if (have) {
    tc_fence_after();
    uint32_t r8[8];
    tmem_ld8(tO + 64, r8);
    tmem_wait_ld();
    l = __uint_as_float(r8[0]);
  }
  const int q_local = (2 * u.pair + g) * kTile + row;
  const bool row_ok = have && q_local < a.Lp;
  uint4* out_row = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) +
                                            (size_t)(u.p * a.Lp + q_local) * a.C + u.head * 64 + half * 32);
  // whole units are one piece; a tail unit spans the CTAs holding its first and last tiles
  const int c_first = u.U0 < 0 ? c : cta_of(u.U0, TT, G);
  const int npieces = u.U0 < 0 ? 1 : cta_of(u.U0 + u.T - 1, TT, G) - c_first + 1;
  if (npieces == 1) {
    if (have) {
      const float inv = 1.f / l;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t r8[8];
        tmem_ld8(tO + half * 32 + k * 8, r8);
        tmem_wait_ld();
        float w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = __uint_as_float(r8[e]) * inv;
        if (row_ok) out_row[k] = pack16(w8);
      }
    }
    return have;
  }
  if (c != c_first) {
    // a later piece: this CTA's first piece, into the CTA's slot
    const size_t prow = (size_t)c * 256 + g * 128 + row;
    if (have) {
      float4* po = reinterpret_cast<float4*>(a.part_o + prow * 64 + half * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t r8[8];
        tmem_ld8(tO + half * 32 + k * 8, r8);
        tmem_wait_ld();
        po[2 * k] = make_float4(__uint_as_float(r8[0]), __uint_as_float(r8[1]), __uint_as_float(r8[2]),
                                __uint_as_float(r8[3]));
        po[2 * k + 1] = make_float4(__uint_as_float(r8[4]), __uint_as_float(r8[5]), __uint_as_float(r8[6]),
                                    __uint_as_float(r8[7]));
      }
      if (half == 0) reinterpret_cast<float2*>(a.part_ml)[prow] = make_float2(m_used, l);
    }
    // publish: every thread's arrival (release, CTA scope) hands its partial stores to the
    // publisher warp, which releases the flag at GPU scope -- the group does not wait
    mbar_arrive(pub_bar);
    return have;
  }
  // the first piece: the flag warp has acquired the later pieces' flags (normally set long
  // before) and lets the groups in; then merge
  const bool flags_ok = mbar_wait(mrg_bar, 0, a.err, kErrWaitAttnMerge) && *merge_fail == 0;
  if (!flags_ok || !have) return false;
  // running maxima and row sums of every piece in KV order (this piece first); the second
  // piece's statistics and partial O are loaded together (one round trip for two pieces)
  const size_t sr1 = (size_t)(c_first + 1) * 256 + g * 128 + row;
  const float2 ml1 = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + sr1);
  float4 v1[8];
  {
    const float4* po = reinterpret_cast<const float4*>(a.part_o + sr1 * 64 + half * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) v1[i] = __ldcg(po + i);
  }
  float mm = fmaxf(m_used, ml1.x);
#pragma unroll 1
  for (int k = 2; k < npieces; ++k) {
    const size_t sr = (size_t)(c_first + k) * 256 + g * 128 + row;
    mm = fmaxf(mm, __ldcg(reinterpret_cast<const float2*>(a.part_ml) + sr).x);
  }
  float lsum = fmaf(l, ex2_mufu(m_used - mm), 0.f);
  lsum = fmaf(ml1.y, ex2_mufu(ml1.x - mm), lsum);
#pragma unroll 1
  for (int k = 2; k < npieces; ++k) {
    const size_t sr = (size_t)(c_first + k) * 256 + g * 128 + row;
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + sr);
    lsum = fmaf(ml.y, ex2_mufu(ml.x - mm), lsum);
  }
  const float inv = 1.f / lsum;
  // this piece's O from TMEM, then each later piece's 32 columns (eight 16-byte loads in
  // flight), every output element accumulated over the pieces in KV order
  float acc[4][8];
  {
    const float w = ex2_mufu(m_used - mm) * inv;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t r8[8];
      tmem_ld8(tO + half * 32 + q * 8, r8);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[q][e] = fmaf(__uint_as_float(r8[e]), w, 0.f);
    }
  }
  {
    const float w = ex2_mufu(ml1.x - mm) * inv;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[q][0] = fmaf(v1[2 * q].x, w, acc[q][0]); acc[q][1] = fmaf(v1[2 * q].y, w, acc[q][1]);
      acc[q][2] = fmaf(v1[2 * q].z, w, acc[q][2]); acc[q][3] = fmaf(v1[2 * q].w, w, acc[q][3]);
      acc[q][4] = fmaf(v1[2 * q + 1].x, w, acc[q][4]); acc[q][5] = fmaf(v1[2 * q + 1].y, w, acc[q][5]);
      acc[q][6] = fmaf(v1[2 * q + 1].z, w, acc[q][6]); acc[q][7] = fmaf(v1[2 * q + 1].w, w, acc[q][7]);
    }
  }
#pragma unroll 1
  for (int k = 2; k < npieces; ++k) {
    const size_t sr = (size_t)(c_first + k) * 256 + g * 128 + row;
    const float w = ex2_mufu(__ldcg(reinterpret_cast<const float2*>(a.part_ml) + sr).x - mm) * inv;
    const float4* po = reinterpret_cast<const float4*>(a.part_o + sr * 64 + half * 32);
    float4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __ldcg(po + i);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[q][0] = fmaf(v[2 * q].x, w, acc[q][0]); acc[q][1] = fmaf(v[2 * q].y, w, acc[q][1]);
      acc[q][2] = fmaf(v[2 * q].z, w, acc[q][2]); acc[q][3] = fmaf(v[2 * q].w, w, acc[q][3]);
      acc[q][4] = fmaf(v[2 * q + 1].x, w, acc[q][4]); acc[q][5] = fmaf(v[2 * q + 1].y, w, acc[q][5]);
      acc[q][6] = fmaf(v[2 * q + 1].z, w, acc[q][6]); acc[q][7] = fmaf(v[2 * q + 1].w, w, acc[q][7]);
    }
  }
  if (row_ok) {
#pragma unroll
    for (int q = 0; q < 4; ++q) out_row[q] = pack16(acc[q]);
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_attention_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mkf,
                    const __grid_constant__ CUtensorMap mvf, const __grid_constant__ CUtensorMap mks,
                    const __grid_constant__ CUtensorMap mvs, const TcAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                          // 2 buffers x 2 tiles x 16 KB
  uint8_t* sK = sQ + 4 * kTileBytes;           // kStages x 16 KB
  uint8_t* sV = sK + kStages * kTileBytes;     // kStages x 16 KB
  uint8_t* sOnes = sV + kStages * kTileBytes;  // 16 KB of bf16 1.0 (the row-sum columns of B)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOnes + kTileBytes);
  uint64_t* q_full = bars;                     // [2]
  uint64_t* q_empty = q_full + 2;              // [2]
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* v_full = k_empty + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_full = v_empty + kStages;        // [2]
  uint64_t* p_full = s_full + 2;               // [2]
  uint64_t* o_done = p_full + 2;               // [2]
  uint64_t* mma_drain = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  __shared__ volatile int s_abort;
  __shared__ float s_mrow[2][128];           // [group][row]: running max handed to the piece epilogue
  __shared__ int s_ring[4][8];                // pieces pi (slot pi % 4): p, head, pair, T, U0, first tile, tiles
  __shared__ __align__(8) uint64_t s_ready[4]; // slot filled (the TMA warp arrives once per piece)
  __shared__ __align__(8) uint64_t s_pub[2];   // [group]: the partial of the CTA's first piece is written
  __shared__ __align__(8) uint64_t s_mrg;      // the later pieces of the pair this CTA merges are published
  __shared__ volatile int s_merge_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int TT = a.total_tiles;                // tiles of the stream-K tail
  const int n_pairs = (a.n_qtiles + 1) / 2;
  const Sched sc{n_pairs, G, c, range_start(c, TT, G), range_start(c + 1, TT, G)};
  const int X0 = sc.X0, X1 = sc.X1;
  const int NT = cta_tiles(a, sc);             // every KV tile of this CTA, whole units included
  int* err = a.err;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&q_full[i]), 1); mbar_init(smem_u32(&q_empty[i]), 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&k_full[i]), 1); mbar_init(smem_u32(&k_empty[i]), 1);
      mbar_init(smem_u32(&v_full[i]), 1); mbar_init(smem_u32(&v_empty[i]), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(smem_u32(&s_full[g]), 1);
      mbar_init(smem_u32(&p_full[g]), 256);
      mbar_init(smem_u32(&o_done[g]), 1);
    }
    mbar_init(smem_u32(mma_drain), 1);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&s_ready[i]), 1);
    mbar_init(smem_u32(&s_pub[0]), 256);
    mbar_init(smem_u32(&s_pub[1]), 256);
    mbar_init(smem_u32(&s_mrg), 1);
    s_merge_fail = 0;
    fence_mbar_init();
  }
  {
    uint4* ones = reinterpret_cast<uint4*>(sOnes);
    for (int i = threadIdx.x; i < (int)(kTileBytes / 16); i += kThreads)
      ones[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the set-up above touches no global memory: overlap it with the prior kernel's tail
  wait_prior_grid();
  allow_next_grid();

  if (warp >= kWarpTma) {
   // Register split: this warpgroup (TMA, MMA, publisher and flag warps) gives registers to
   // the four softmax warpgroups (the launcher checks the launch's total covers it).
   asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsTmaMma) : "memory");
   // Both warps walk their loops with all lanes (addresses and descriptors stay
   // warp-uniform); the elected lane issues the copies, MMAs and commits.
   const bool leader = elect_one();
   if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (leader) tma_prefetch_desc(&mq);
    int gt = 0, pi = 0;   // tiles and pieces issued so far
    bool ok = true;
    Walk w;
    for (bool have = walk_first(a, sc, w); ok && have; ++pi, have = walk_next(a, sc, w)) {
      const Unit u = walk_unit(a, sc, w);
      const int jl0 = w.j0;
      const int n = w.n;
      // the piece's two query tiles into Q buffer pi & 1
      const int qb = pi & 1;
      if (pi >= 2 && !mbar_wait_warp(smem_u32(&q_empty[qb]), ((pi >> 1) - 1) & 1, err, kErrWaitStageFree)) {
        ok = false;
        break;
      }
      if (leader) {
        // the piece for the softmax groups (slot pi % 4 is free: the groups have started
        // piece pi - 3, which needs this warp's piece pi - 2 queries loaded and consumed)
        volatile int* r = s_ring[pi & 3];
        r[0] = u.p; r[1] = u.head; r[2] = u.pair; r[3] = u.T; r[4] = u.U0; r[5] = jl0; r[6] = n;
        mbar_arrive(smem_u32(&s_ready[pi & 3]));
        const int qrow = u.p * a.Lp + 2 * u.pair * kTile;
        const uint32_t qbar = smem_u32(&q_full[qb]);
        mbar_arrive_expect_tx(qbar, 2 * kTileBytes);
        tma_load_3d(smem_u32(sQ + 2 * qb * kTileBytes), &mq, qbar, 0, qrow, u.head);
        tma_load_3d(smem_u32(sQ + (2 * qb + 1) * kTileBytes), &mq, qbar, 0, qrow + kTile, u.head);
      }
      __syncwarp();
      // the piece's patch within its image, and the image's first K/V row
      const int img = u.p / a.N, p_img = u.p - img * a.N, kv0 = img * a.kv_stride;
      for (int jj = 0; jj < n; ++jj, ++gt) {
        const int s = gt % kStages, round = gt / kStages;
        int stale, row, valid;
        tile_src(a.mode, p_img, a.Lp, a.L, a.kv_len, jl0 + jj, stale, row, valid);
        row += kv0;
        if (round > 0 && !mbar_wait_warp(smem_u32(&k_empty[s]), (round - 1) & 1, err, kErrWaitStageFree)) { ok = false; break; }
        if (leader) {
          mbar_arrive_expect_tx(smem_u32(&k_full[s]), kTileBytes);
          tma_load_3d(smem_u32(sK + s * kTileBytes), stale ? &mks : &mkf, smem_u32(&k_full[s]), 0, row, u.head);
        }
        if (round > 0 && !mbar_wait_warp(smem_u32(&v_empty[s]), (round - 1) & 1, err, kErrWaitStageFree)) {
          if (leader) mbar_arrive_expect_tx(smem_u32(&v_full[s]), 0);
          ++gt;
          ok = false;
          break;
        }
        if (leader) {
          mbar_arrive_expect_tx(smem_u32(&v_full[s]), kTileBytes);
          tma_load_5d(smem_u32(sV + s * kTileBytes), stale ? &mvs : &mvf, smem_u32(&v_full[s]), 0, 0, 0, row >> 2,
                      u.head);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (leader) s_abort = 1;
      // let the copies already in flight land before the CTA can exit
      for (int j = (gt > kStages ? gt - kStages : 0); j < gt; ++j) {
        mbar_wait(smem_u32(&k_full[j % kStages]), (j / kStages) & 1, err, kErrWaitTmaFull);
        mbar_wait(smem_u32(&v_full[j % kStages]), (j / kStages) & 1, err, kErrWaitTmaFull);
      }
      for (int q = (pi > 2 ? pi - 2 : 0); q < pi; ++q)
        mbar_wait(smem_u32(&q_full[q & 1]), (q >> 1) & 1, err, kErrWaitTmaFull);
    }
   } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Per MMA, every operand is a per-tile base plus a compile-time offset (the two
    // groups and the K slices are unrolled): runtime arithmetic between
    // tcgen05.mma instructions stalls their issue.
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTile, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, kOCols, false, true);
    constexpr uint64_t kTileDesc = kTileBytes >> 4;            // one tile in descriptor address units
    const uint64_t qd0 = sw128_kmajor_desc(smem_u32(sQ));
    const uint64_t kd0 = sw128_kmajor_desc(smem_u32(sK));
    // V stage 0 with the ones block as its second 64-column atom (leading byte offset);
    // stage st: start address + st tiles, leading byte offset - st tiles
    uint64_t vd0 = sw128_mnmajor_desc(smem_u32(sV));
    vd0 = (vd0 & ~(uint64_t(0x3FFF) << 16)) |
          (uint64_t(((smem_u32(sOnes) - smem_u32(sV)) >> 4) & 0x3FFF) << 16);
    // S_g = Q_g K^T, Q tile descriptor QD, K tile descriptor KD
#define DFP_ISSUE_S(G, QD, KD)                                               \
    do {                                                                     \
      if (leader) {                                                          \
        umma_f16_ss(tmem + 128 * (G), (QD), (KD), idesc_s, 0);               \
        umma_f16_ss(tmem + 128 * (G), (QD) + 2, (KD) + 2, idesc_s, 1);       \
        umma_f16_ss(tmem + 128 * (G), (QD) + 4, (KD) + 4, idesc_s, 1);       \
        umma_f16_ss(tmem + 128 * (G), (QD) + 6, (KD) + 6, idesc_s, 1);       \
        umma_commit(smem_u32(&s_full[G]));                                   \
      }                                                                      \
      __syncwarp();                                                          \
    } while (0)
    // O_g += P_g [V | 1], V tile at descriptor vd (P read from TMEM over S_g)
#define DFP_ISSUE_PV(G, VD, ACC0)                                                                \
    do {                                                                                         \
      if (leader) {                                                                              \
        umma_f16_ts(tmem + 256 + 128 * (G), tmem + 128 * (G), (VD), idesc_o, (ACC0));            \
        _Pragma("unroll") for (int kk = 1; kk < 8; ++kk)                                         \
          umma_f16_ts(tmem + 256 + 128 * (G), tmem + 128 * (G) + kk * 8, (VD) + (uint64_t)kk * 128, idesc_o, 1); \
        umma_commit(smem_u32(&o_done[G]));                                                       \
      }                                                                                          \
      __syncwarp();                                                                              \
    } while (0)
    // piece walk: for each tile, is it the first / last of its piece, and which piece
    // (called once per tile of the CTA, so a piece always follows).  The pieces' lengths come
    // from the TMA warp's descriptor ring (this warp is at most one piece ahead of the
    // softmax groups, the TMA warp at most two ahead of this one, so the slot is current).
    int left = 0, pc = -1;
    bool walk_ok = true;
    auto next_tile = [&](bool& first, bool& last, int& piece) {
      first = left == 0;
      if (first) {
        ++pc;
        walk_ok = walk_ok && mbar_wait_warp(smem_u32(&s_ready[pc & 3]), (uint32_t)(pc >> 2) & 1u, err, kErrWaitTmaFull);
        left = walk_ok ? s_ring[pc & 3][6] : 1;
      }
      --left;
      last = left == 0;
      piece = pc;
    };
    bool ok = true;
    bool cur_first, cur_last;
    int cur_piece;
    next_tile(cur_first, cur_last, cur_piece);
    ok = walk_ok;
    if (ok) {
      const int qb = cur_piece & 1;
      ok = mbar_wait_warp(smem_u32(&q_full[qb]), (cur_piece >> 1) & 1, err, kErrWaitTmaFull) &&
           mbar_wait_warp(smem_u32(&k_full[0]), 0, err, kErrWaitTmaFull);
      if (ok) {
        tc_fence_after();
        const uint64_t qd = qd0 + (uint64_t)(2 * qb) * kTileDesc;
        DFP_ISSUE_S(0, qd, kd0);
        DFP_ISSUE_S(1, qd + kTileDesc, kd0);
        if (leader) {
          if (cur_last) umma_commit(smem_u32(&q_empty[qb]));
          umma_commit(smem_u32(&k_empty[0]));
        }
        __syncwarp();
      }
    }
    for (int gt = 0; ok && gt < NT; ++gt) {
      const int st = gt % kStages, st1 = (gt + 1) % kStages;
      const uint32_t par = (uint32_t)(gt / kStages) & 1u, par1 = (uint32_t)((gt + 1) / kStages) & 1u;
      const bool more = gt + 1 < NT;
      const uint32_t acc0 = cur_first ? 0u : 1u;
      const uint64_t vd = vd0 + (uint64_t)st * (kTileDesc - (kTileDesc << 16));
      const uint64_t kd1 = kd0 + (uint64_t)st1 * kTileDesc;
      bool nx_first = false, nx_last = false;
      int nx_piece = cur_piece;
      if (more) next_tile(nx_first, nx_last, nx_piece);
      if (!walk_ok) { ok = false; break; }
      const int nqb = nx_piece & 1;
      const uint64_t nqd = qd0 + (uint64_t)(2 * nqb) * kTileDesc;
      if (!mbar_wait_warp(smem_u32(&v_full[st]), par, err, kErrWaitTmaFull)) { ok = false; break; }
      if (!mbar_wait_warp(smem_u32(&p_full[0]), (uint32_t)gt & 1u, err, kErrWaitAttnP)) { ok = false; break; }
      tc_fence_after();
      DFP_ISSUE_PV(0, vd, acc0);
      if (more) {
        if (!mbar_wait_warp(smem_u32(&k_full[st1]), par1, err, kErrWaitTmaFull)) { ok = false; break; }
        if (nx_first && !mbar_wait_warp(smem_u32(&q_full[nqb]), (nx_piece >> 1) & 1, err, kErrWaitTmaFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        DFP_ISSUE_S(0, nqd, kd1);
      }
      if (!mbar_wait_warp(smem_u32(&p_full[1]), (uint32_t)gt & 1u, err, kErrWaitAttnP)) { ok = false; break; }
      tc_fence_after();
      DFP_ISSUE_PV(1, vd, acc0);
      if (more) DFP_ISSUE_S(1, nqd + kTileDesc, kd1);
      if (leader) {
        umma_commit(smem_u32(&v_empty[st]));
        if (more) {
          umma_commit(smem_u32(&k_empty[st1]));
          if (nx_last) umma_commit(smem_u32(&q_empty[nqb]));
        }
      }
      __syncwarp();
      cur_first = nx_first;
      cur_last = nx_last;
      cur_piece = nx_piece;
    }
#undef DFP_ISSUE_S
#undef DFP_ISSUE_PV
    if (!ok && leader) s_abort = 1;
    // every MMA issued by this CTA completes before its TMEM can be released
    if (leader) umma_commit(smem_u32(mma_drain));
    __syncwarp();
    mbar_wait(smem_u32(mma_drain), 0, err, kErrWaitAccum);
   } else if (warp == kWarpMma + 1) {
    // ------------------------------------------------------------ publisher
    // The CTA's first tail piece continues a pair an earlier CTA started: once a group has
    // written its partial (its 256 threads arrived on s_pub[g], release at CTA scope),
    // release the group's flag at GPU scope for the merging CTA.
    const Unit u0 = locate(a, n_pairs, X0);
    const int cf = X1 > X0 ? cta_of(u0.U0, TT, G) : c;
    const int np = X1 > X0 ? cta_of(u0.U0 + u0.T - 1, TT, G) - cf + 1 : 1;
    if (np > 1 && c != cf && leader) {
      for (int g = 0; g < 2; ++g)
        if (mbar_wait(smem_u32(&s_pub[g]), 0, err, kErrWaitAttnMerge)) st_release_gpu(a.flags + 2 * c + g, a.epoch);
    }
    __syncwarp();
   } else if (warp == kWarpMma + 2) {
    // ------------------------------------------------------------ merge flags
    // The CTA's last tail piece holds the first KV tiles of a cut pair: acquire the later
    // pieces' flags of both groups while the CTA works, then let the groups merge.
    const Unit ul = locate(a, n_pairs, X1 - 1);
    const int cf = X1 > X0 ? cta_of(ul.U0, TT, G) : c;
    const int np = X1 > X0 ? cta_of(ul.U0 + ul.T - 1, TT, G) - cf + 1 : 1;
    if (np > 1 && c == cf && leader) {
      int failed = 0;
      for (int k = 1; k < np && !failed; ++k)
        for (int g = 0; g < 2 && !failed; ++g) {
          const unsigned* flag = a.flags + 2 * (cf + k) + g;
          const long long t0 = clock64();
          while (ld_acquire_gpu(flag) != a.epoch) {
            if (clock64() - t0 > kWaitLimitCycles) {
              atomicCAS(err, 0, kErrWaitAttnMerge);
              failed = 1;
              break;
            }
            __nanosleep(256);
          }
        }
      s_merge_fail = failed;
      mbar_arrive(smem_u32(&s_mrg));
    }
    __syncwarp();
   }
  } else {
    // ------------------------------------------------------------ softmax groups (warps 0..15)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax) : "memory");
    const int g = warp >> 3;                    // query tile of this warp
    const int q4 = warp & 3;                    // TMEM lane quadrant (fixed by the warp's SM sub-partition)
    const int h16 = (warp >> 2) & 1;            // which 16 lanes of the quadrant
    // KV loop (16x64b shapes): two lanes of a warp share a query row, each holding 64 of
    // its 128 score columns (2r + cq); they exchange row maxima with one shuffle.
    const int cq = (lane >> 1) & 1;
    const uint32_t lane16 = (uint32_t)(32 * q4 + 16 * h16) << 16;
    const uint32_t tS = tmem + 128 * g + lane16;
    const uint32_t tO = tmem + 256 + 128 * g + lane16;
    const int srow = 32 * q4 + 16 * h16 + 8 * (lane & 1) + (lane >> 2);
    // piece epilogue (32x32b shape): lane = row of the quadrant, h16 picks 32 output columns
    const int erow = 32 * q4 + lane;
    const uint32_t tOe = tmem + 256 + 128 * g + ((uint32_t)(32 * q4) << 16);
    const float sl2 = 0.125f * 1.4426950408889634f;   // (1/sqrt(64)) * log2(e)
    bool ok = true;
    // A failed wait makes the whole warp give up the piece (waits are agreed warp-wide,
    // so the TMEM instructions stay warp-uniform); the group then leaves together at the
    // piece barrier (bar.red.or), which every thread reaches once per piece.
    bool carry = false;
    // The pieces come from the TMA warp (a ring of four descriptors in shared memory, each
    // published with a release arrival): the groups do no walking of their own.
    int gt = 0, pi = 0;
    while (ok && gt < NT) {
      if (!mbar_wait_warp(smem_u32(&s_ready[pi & 3]), (uint32_t)(pi >> 2) & 1u, err, kErrWaitTmaFull)) {
        carry = true;
      }
      volatile int* sp = s_ring[pi & 3];
      const int n = carry ? 0 : sp[6];
      const int j0 = sp[5];
      const TileEnds te = tile_ends(a.mode, sp[0] % a.N, a.Lp, a.L, a.kv_len);
      float m_used = -INFINITY;
      for (int jj = 0; jj < n && !carry; ++jj, ++gt) {
        // the tile's valid key count (a segment's last tile may be partial)
        const int jt = j0 + jj;
        const int valid = jt == te.e0 ? te.v0 : jt == te.e1 ? te.v1 : jt == te.e2 ? te.v2 : kTile;
        if (!mbar_wait_warp(smem_u32(&s_full[g]), gt & 1, err, kErrWaitAttnS)) { carry = true; break; }
        tc_fence_after();
        float sc[64];   // sc[i] = S[row][2i + cq]
        {
          uint32_t r[32];
          tmem_ld_16x64b_x32(tS, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) sc[i] = __uint_as_float(r[i]);
          tmem_ld_16x64b_x32(tS + 64, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) sc[32 + i] = __uint_as_float(r[i]);
        }
        tmem_wait_ld();
        const bool full_tile = valid == kTile;
        if (!full_tile) {
#pragma unroll
          for (int i = 0; i < 64; ++i) sc[i] = 2 * i + cq < valid ? sc[i] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = max3(sc[i], sc[8 + i], sc[16 + i]);
#pragma unroll
        for (int i = 24; i < 64; i += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], sc[i + k], i + 8 + k < 64 ? sc[i + 8 + k] : mx[k]);
        }
        float mrow = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        mrow = fmaxf(mrow, __shfl_xor_sync(0xffffffffu, mrow, 2)) * sl2;   // the row's other half
        if (jj == 0) {
          m_used = mrow;
        } else {
          const bool need = mrow > m_used + kRescale;
          if (__any_sync(0xffffffffu, need)) {
            // both lanes of a row see the same mrow, so they agree on every decision
            const float m_new = need ? mrow : m_used;
            const float alpha = ex2_mufu(m_used - m_new);
            if (!mbar_wait_warp(smem_u32(&o_done[g]), (gt - 1) & 1, err, kErrWaitAttnO)) { carry = true; break; }
            tc_fence_after();
            // this lane's 40 of the row's 80 O columns (64 outputs + 16 row-sum columns)
#pragma unroll
            for (int cc = 0; cc < 5; ++cc) {
              uint32_t r8[8];
              tmem_ld_16x64b_x8(tO + cc * 16, r8);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 8; ++i) r8[i] = __float_as_uint(__uint_as_float(r8[i]) * alpha);
              tmem_st_16x64b_x8(tO + cc * 16, r8);
            }
            tmem_wait_st();
            m_used = m_new;
          }
        }
        const float nm = -m_used;
        // P over S in TMEM: this lane packs its own neighbours sc[2r'], sc[2r'+1] (score
        // columns 4r'+cq and 4r'+cq+2) into P column 2r'+cq, i.e. the key order within
        // each group of 4 is 0, 2, 1, 3 -- the order in which V's rows are loaded.
        if (full_tile) {
          // x = s * c - m on pairs (fp32x2); a fixed share of the pairs through the
          // polynomial on the FMA pipe, the rest through the MUFU
          const uint64_t sl2x2 = f2(sl2, sl2), nmx2 = f2(nm, nm);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint64_t x2 = fma2(f2(sc[cc * 16 + 2 * e], sc[cc * 16 + 2 * e + 1]), sl2x2, nmx2);
              if (e < kPolyPer8) {
                pk[e] = ex2_poly_pair_bf16(x2);
              } else {
                float x0, x1;
                f2_split(x2, x0, x1);
                pk[e] = pack_trunc(ex2_mufu(x0), ex2_mufu(x1));
              }
            }
            tmem_st_16x64b_x8(tS + cc * 16, pk);
          }
        } else {
          // partial tile: masked columns are -inf, which only the MUFU maps to exactly 0
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t pk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pk[e] = pack_trunc(ex2_mufu(fmaf(sc[cc * 16 + 2 * e], sl2, nm)),
                                 ex2_mufu(fmaf(sc[cc * 16 + 2 * e + 1], sl2, nm)));
            tmem_st_16x64b_x8(tS + cc * 16, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&p_full[g]));
      }
      // the row's lazily updated maximum, for the epilogue's (32x32b) row owner
      if (cq == 0) s_mrow[g][srow] = m_used;
      // every thread of the group reaches this barrier once per piece
      if (named_bar_or(2 + g, 256, carry)) { ok = false; break; }
      // ---- piece epilogue (out of line: its registers do not add to the KV loop's)
      Unit u;
      u.p = sp[0]; u.head = sp[1]; u.pair = sp[2]; u.T = sp[3]; u.U0 = sp[4];
      if (!piece_epilogue(a, u, tOe, smem_u32(&o_done[g]), (uint32_t)(gt - 1) & 1u, s_mrow[g][erow], g, h16,
                          erow, c, smem_u32(&s_pub[g]), smem_u32(&s_mrg), &s_merge_fail))
        carry = true;
      // next piece: every thread of the group is done with s_mrow before it changes
      named_bar(2 + g, 256);
      ++pi;
    }
    if (!ok || carry) s_abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool encode_attn_k(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads) {
  return encode_tmap_3d(m, base, 64, rows, heads, 128, rows * 128, 64, kTile, 1);
}

bool encode_attn_v(CUtensorMap* m, const void* base, uint64_t rows, uint64_t heads) {
  // key = 4 s + q + 2 e lands in shared-memory row 4 s + 2 q + e: dims (d, e, q, s, head)
  const uint64_t dims[5] = {64, 2, 2, (rows + 3) / 4, heads};
  const uint64_t strides[4] = {256, 128, 512, rows * 128};
  const uint32_t box[5] = {64, 2, 2, 32, 1};
  if (rows % 4) return false;
  return encode_tmap_5d(m, base, dims, strides, box);
}

// K/V bytes above which the whole-unit rounds are used: the list's K and V (every head,
// fresh and stale rows) no longer fit next to the Q and O streams in the 126 MB L2.
constexpr long long kL2KvBudget = 48ll << 20;

// The work split of `a` over at most `ctas` CTAs: fills whole_rounds, total_tiles (the tail),
// tail_base and head_tiles and returns the CTA count (0: no work; -1: too large for the
// kernel's 32-bit schedule arithmetic).
int plan_schedule(TcAttnArgs& a, int ctas, long long kv_budget = kL2KvBudget) {
  const int n_pairs = (a.n_qtiles + 1) / 2;
  const int np = a.p_hi - a.p_lo;
  long long per_head = 0;
  for (int p = a.p_lo; p < a.p_hi; ++p) per_head += (long long)patch_tiles(a, p) * n_pairs;
  const long long all = per_head * a.heads;
  if (all <= 0 || np <= 0 || n_pairs <= 0) return 0;
  const int G = (int)std::min<long long>(ctas, all);
  if (G <= 0 || all * G >= (1ll << 31)) return -1;
  const long long units = (long long)a.heads * np * n_pairs;
  const long long kv_rows =
      (long long)(a.mode == kAttnCross ? a.kv_len : a.mode == kAttnDisplaced ? 2 * a.L : a.L) * a.images;
  const long long kv_bytes = kv_rows * a.heads * 64 * 2 * 2;
  const int F = kv_bytes > kv_budget ? (int)(units / G) : 0;
  // tiles of the units before the tail (the first F * G of the head-major list)
  const long long fg = (long long)F * G, per_head_units = (long long)np * n_pairs;
  const long long h = fg / per_head_units, r = fg - h * per_head_units;
  long long base = h * per_head;
  const int lp = (int)(r / n_pairs), pair = (int)(r - (long long)lp * n_pairs);
  for (int q = 0; q < lp; ++q) base += (long long)patch_tiles(a, a.p_lo + q) * n_pairs;
  if (lp < np) base += (long long)pair * patch_tiles(a, a.p_lo + lp);
  a.whole_rounds = F;
  a.head_tiles = (int)per_head;
  a.tail_base = (int)base;
  a.total_tiles = (int)(all - base);
  return G;
}

size_t attention_scratch_floats(int ctas) { return (size_t)ctas * 256 * 64; }

cudaError_t launch_tc_attention(const TcAttnArgs& args, const CUtensorMap& mq, const CUtensorMap& mkf,
                                const CUtensorMap& mvf, const CUtensorMap& mks,
                                const CUtensorMap& mvs, cudaStream_t s) {
  const size_t smem = 1024 + (4 + 2 * kStages + 1) * (size_t)kTileBytes + (4 * kStages + 12) * 8 + 64;
  cudaError_t e = cudaFuncSetAttribute(tc_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // The register split inside the kernel (setmaxnreg) hands the launch's registers from
  // one warpgroup to the others; it needs the full 96 per thread at launch.
  static int regs = 0;
  if (!regs) {
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, tc_attention_kernel);
    if (e != cudaSuccess) return e;
    regs = fa.numRegs;
  }
  if (regs * kThreads < 128 * kRegsTmaMma + 512 * kRegsSoftmax) return cudaErrorInvalidConfiguration;
  TcAttnArgs a = args;
  if (a.images < 1 || a.kv_stride < 0) return cudaErrorInvalidValue;
  if (a.p_lo == 0 && a.p_hi == 0) a.p_hi = a.N * a.images;   // every query patch
  if (a.p_lo < 0 || a.p_hi > a.N * a.images || a.p_lo >= a.p_hi) return cudaErrorInvalidValue;
  // a fresh flag value per launch (flags hold the epoch of the launch that last set them)
  static std::atomic<unsigned> epoch{0};
  do a.epoch = ++epoch; while (a.epoch == 0);
  const int G = plan_schedule(a, a.ctas, a.kv_budget > 0 ? a.kv_budget : kL2KvBudget);
  if (G == 0) return cudaSuccess;
  if (G < 0) return cudaErrorInvalidValue;   // 32-bit schedule arithmetic
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, tc_attention_kernel, mq, mkf, mvf, mks, mvs, a);
}

// Host walk of the work split exactly as the kernel's walkers do it (the same plan,
// walk_first / walk_next, locate, cta_of, range_start), checking what the cut-pair merge
// relies on.
int attention_schedule_check(int L, int Lp, int N, int heads, int mode, int kv_len, int images, int ctas,
                             int p_lo, int p_hi, long long kv_budget) {
  TcAttnArgs a{};
  a.L = L; a.Lp = Lp; a.N = N; a.heads = heads; a.mode = mode; a.kv_len = kv_len; a.images = images;
  a.p_lo = p_lo; a.p_hi = p_hi > 0 ? p_hi : N * images;
  a.n_qtiles = cdiv(Lp, kTile);
  if (L <= 0 || Lp <= 0 || N <= 0 || heads <= 0 || images < 1 || ctas < 1) return 1;
  if (a.p_lo < 0 || a.p_hi > N * images || a.p_lo >= a.p_hi) return 1;
  const int G = plan_schedule(a, ctas, kv_budget < 0 ? kL2KvBudget : kv_budget);
  if (G == 0) return 1;
  if (G < 0) return 2;
  const int n_pairs = (a.n_qtiles + 1) / 2, np = a.p_hi - a.p_lo;
  const int TT = a.total_tiles;
  auto index_of = [&](const Unit& u) { return ((size_t)u.head * np + (u.p - a.p_lo)) * n_pairs + u.pair; };
  std::vector<long long> cover((size_t)heads * np * n_pairs, 0);   // tiles of each unit, summed over pieces
  for (int c = 0; c < G; ++c) {
    const Sched sc{n_pairs, G, c, range_start(c, TT, G), range_start(c + 1, TT, G)};
    const int X0 = sc.X0, X1 = sc.X1;
    if (cta_tiles(a, sc) <= 0) return 3;            // every CTA has work
    // what the publisher and flag warps conclude from the tail range's ends
    int expect_publish = 0, expect_merge = 0;
    if (X1 > X0) {
      const Unit u0 = locate(a, n_pairs, X0), ul = locate(a, n_pairs, X1 - 1);
      const int cf0 = cta_of(u0.U0, TT, G), np0 = cta_of(u0.U0 + u0.T - 1, TT, G) - cf0 + 1;
      const int cfl = cta_of(ul.U0, TT, G), npl = cta_of(ul.U0 + ul.T - 1, TT, G) - cfl + 1;
      expect_publish = np0 > 1 && c != cf0;
      expect_merge = npl > 1 && c == cfl;
    }
    int publishes = 0, merges = 0, whole = 0, pieces = 0, merge_k = -1;
    Walk w;
    for (bool have = walk_first(a, sc, w); have; have = walk_next(a, sc, w), ++pieces) {
      if (w.k != pieces) return 4;
      const Unit wu = walk_unit(a, sc, w);
      if (w.n <= 0 || w.j0 < 0 || w.j0 + w.n > wu.T) return 4;   // the piece stays inside its unit
      cover[index_of(wu)] += w.n;
      if (wu.U0 < 0) {                              // a whole unit
        if (w.j0 != 0 || w.n != wu.T) return 4;
        ++whole;
        continue;
      }
      const int x = wu.U0 + w.j0, x_end = x + w.n;
      if (x < X0 || x_end > X1) return 4;
      const int cf = cta_of(wu.U0, TT, G), npc = cta_of(wu.U0 + wu.T - 1, TT, G) - cf + 1;
      if (c < cf || c >= cf + npc) return 5;        // this CTA holds part of the unit
      if (npc > 1) {
        if (c == cf) {                               // the first KV tiles end the range
          if (x_end != X1) return 6;
          merge_k = w.k;
          ++merges;
        } else {                                     // a later piece opens the range, and the sequence
          if (x != X0 || w.k != 0) return 7;
          ++publishes;
        }
      }
    }
    if (whole != a.whole_rounds) return 11;
    if (publishes != expect_publish || merges != expect_merge) return 8;
    // the merging piece is the CTA's last, or its only tail piece (then it opens the sequence)
    if (merges && merge_k != pieces - 1 && !(merge_k == 0 && pieces - whole == 1)) return 12;
  }
  // the softmax's per-piece partial-tile table gives every tile the valid key count the
  // TMA warp's per-tile walk gives
  for (int p = 0; p < N; ++p) {
    const TileEnds te = tile_ends(mode, p, Lp, L, kv_len);
    for (int j = 0; j < unit_tiles(mode, p, Lp, L, kv_len); ++j) {
      int stale, row, valid;
      tile_src(mode, p, Lp, L, kv_len, j, stale, row, valid);
      const int v = j == te.e0 ? te.v0 : j == te.e1 ? te.v1 : j == te.e2 ? te.v2 : kTile;
      if (v != valid || valid < 1 || valid > kTile) return 13;
    }
  }
  // every unit covered exactly once, whole
  for (int h = 0; h < heads; ++h)
    for (int p = a.p_lo; p < a.p_hi; ++p)
      for (int q = 0; q < n_pairs; ++q) {
        Unit u{};
        u.head = h; u.p = p; u.pair = q;
        if (cover[index_of(u)] != patch_tiles(a, p)) return 10;
      }
  return 0;
}

}  // namespace dfp
