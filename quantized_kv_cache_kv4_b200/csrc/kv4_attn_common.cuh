// Pieces shared by the attention kernels (kv4_attention.cu: KV4-RL; kv4_baseline.cu:
// the BF16 and KV8 comparison kernels): shared-memory budget of a warp, region
// bookkeeping, the per-warp copy ring and the partial-record helpers.
#pragma once

#include <math_constants.h>

#include "kv4_device.cuh"
#include "kv4_internal.h"

#ifndef KV4_MIN_BLOCKS
#define KV4_MIN_BLOCKS 3  // CTAs per SM the register budget is sized for
#endif

namespace kv4 {

constexpr int kWarps = 4;                 // warps per CTA (independent work streams)
constexpr int kStages = 3;                // shared-memory stages per warp
constexpr int kStageBytes = 5120;         // two kv heads' INT4 page blocks; >= one INT8 tile
constexpr int kPWordsPerCol = 12;         // P' tile column stride in words (bank-conflict free)
constexpr int kPtileBytes = 2 * 4 * 8 * kPWordsPerCol * 4;  // [2 slots][4 groups][8 cols][12 w]
constexpr int kPtile8Bytes = 8 * 16 * 2;  // INT8 P': [8 heads][16 tokens] fp16
constexpr int kWarpSmem = kStages * kStageBytes + kPtileBytes + kPtile8Bytes + 64;
constexpr int kCtaSmem = kWarps * kWarpSmem;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegBig = -1.0e30f;  // running-max start: finite, so e^(m_old-m_new) is 0 not NaN
constexpr float kScaleLog2 = kLog2e * 0.08838834764831845f;  // log2(e) / sqrt(128)

// V codes enter the PV product as fp16 subnormals (see nib_pairs_v_sub): code c of an
// even output row is c * 2^-24, of an odd one 16c * 2^-24; the scales are undone on the
// output.
constexpr float kUnscaleV = kSubUnscale;     // C rows gid (dims 32g+4gid+2t)
constexpr float kUnscaleV1 = kSubUnscale16;  // C rows gid+8 (dims 32g+4gid+2t+1)

// INT8 stage: K codes | V codes | K scales | V scales
constexpr int kOffVc8 = 2048, kOffKs8 = 4096, kOffVs8 = 4128, kInt8Bytes = 4160;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------------------
// region bookkeeping shared by plan and attention
// ---------------------------------------------------------------------------
struct Regions {
  int has_prot;          // 1 if the INT8 protected set is non-empty
  int n_prompt;          // regions over pages shared with the sequence's prefix group
  int first_page;        // first page of the sequence's own INT4 chunks
  int int4_lo, int4_hi;  // INT4 token range [lo, hi)
  int n_chunks;          // the sequence's own INT4 chunks
};

// Regions of a sequence of length L, in merge order: the protected set (if any), then
// n_prompt regions over the INT4 pages [S/16, pe) that the sequence's prefix group reads
// once for all its members (pe = 0: no group), then its own chunks of C pages from
// max(S/16, pe) on. A group member's prompt regions exist even where its own INT4 range
// does not reach them (their partial states are then empty), so every member of a group
// has the same region layout up to its own chunks.
__device__ __forceinline__ Regions regions_of(int L, int S, int R, int C, int pe = 0) {
  Regions g;
  const int n_sink = min(S, L);
  const int rec_lo = max(S, L - R);
  g.has_prot = (n_sink > 0 || rec_lo < L) ? 1 : 0;
  g.int4_lo = S;
  g.int4_hi = L - R;
  const int p0 = S / kPage;
  g.n_prompt = pe > p0 ? (pe - p0 + C - 1) / C : 0;
  g.first_page = max(p0, pe);
  g.n_chunks = 0;
  if (g.int4_hi > g.int4_lo) {
    const int last = (g.int4_hi - 1) / kPage;
    if (last >= g.first_page) g.n_chunks = (last - g.first_page + C) / C;
  }
  return g;
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------
struct WarpCtx {
  uint8_t *stage0;     // first stage (generic pointer)
  uint32_t *ptile;     // INT4 P' tile [2 slots][4 groups][8 cols][12 words], zero padded
  uint16_t *ptile8;    // INT8 P' tile [8 heads][16 tokens]
  uint64_t *bars;      // kStages mbarriers
  uint32_t parity;     // bit s = parity of the next completion of stage s
  uint32_t wait_limit; // attempts of one bounded wait
  int lane, gid, tig;
  bool fault;          // testing hook: the current entry's first copy is withheld
  bool dead;           // a bounded wait gave up: stop taking work
};

// Whether an entry's copy k is issued by its prologue: the testing hook withholds copy 0
// of the chosen work item (nothing is issued, nothing is in flight, and the bounded wait
// on its stage gives up). Copies issued inside the page loops have k >= kStages.
__device__ __forceinline__ bool prologue_copy(const WarpCtx &x, int k) {
  return !(x.fault && k == 0);
}

// Power-of-two lift of the probability weights P' = p * vscale of one work entry, in
// log2 units. P' is rounded to fp16 for the PV product, and below 2^-14 an fp16 keeps
// only 2^-24 of absolute precision; with small values (vscale well below 1) most weights
// would land there. So the weights are computed as p * 2^E * vscale, with E chosen from
// the largest V scale s_max on the entry's first page so that s_max * 2^E < 1 (E = 0
// when s_max >= 1/2, at most 24). The lift needs no correction afterwards: the online
// softmax keeps its running maximum as m - E, so p arrives as exp2(s - (m - E)) and the
// partial state (m - E, l 2^E, acc 2^E) is the same state as (m, l, acc) for the exact
// merge. A later page whose scale would overflow fp16 under the lift makes the kernel
// redo the entry without it. bits: the fp16 bits of s_max (non-negative).
__device__ __forceinline__ float lift_for_scale(uint32_t bits) {
  if (bits == 0u) return 0.f;
  const float sm = __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
  const int e = static_cast<int>((__float_as_uint(sm) >> 23) & 0xFFu) - 127;  // [2^e, 2^(e+1))
  return static_cast<float>(min(24, max(0, -1 - e)));
}

// The largest of the fp16 values v0 .. v7 (non-negative fp16 bits in the low halves of
// the words, anything in the high halves) over the lanes that share this lane's tig:
// the V scales of one page's tokens.
__device__ __forceinline__ uint32_t page_max_scale(uint32_t m) {
  m &= 0xFFFFu;
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 8));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 16));
  return m;
}

// Whether any of n accumulators of the warp is not finite (an fp16 weight overflowed).
template <int N>
__device__ __forceinline__ bool any_not_finite(const float (&v)[N]) {
  bool bad = false;
#pragma unroll
  for (int i = 0; i < N; ++i) bad |= !(fabsf(v[i]) <= 3.0e38f);
  return __any_sync(0xffffffffu, bad);
}

// Online softmax update for this thread's two heads (2tig, 2tig+1) with logits of
// tokens (gid, gid+8) in log2 units. Returns p in s[][] and the rescale factors.
__device__ __forceinline__ void softmax_step(float (&s)[2][2], float (&m)[2], float (&l)[2],
                                             float (&alpha)[2], float lift = 0.f) {
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float t = fmaxf(s[0][e], s[1][e]);
    t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 4));
    t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 8));
    t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 16));
    const float mn = fmaxf(m[e], t - lift);  // running maximum kept as max - lift
    alpha[e] = fast_exp2(m[e] - mn);
    m[e] = mn;
    s[0][e] = fast_exp2(s[0][e] - mn);
    s[1][e] = fast_exp2(s[1][e] - mn);
    l[e] = l[e] * alpha[e] + s[0][e] + s[1][e];
  }
}

// Bounded wait for the next completion of `stage`; the stage's parity bit flips either
// way (a wait that gave up leaves the warp dead, and drain_copies knows its parity).
__device__ __forceinline__ bool wait_stage(WarpCtx &x, int stage, int32_t *err) {
  const bool ok = mbar_wait_bounded(&x.bars[stage], (x.parity >> stage) & 1u, x.wait_limit);
  x.parity ^= 1u << stage;
  if (!ok) {
    x.dead = true;
    if (x.lane == 0) set_err(err, KV4_DEVERR_TIMEOUT);
  }
  return ok;
}

// Waits for the next completion of `stage` like wait_stage, but on success leaves the
// stage's parity as it was, so that the page loop's own wait on it returns at once.
__device__ __forceinline__ bool peek_stage(WarpCtx &x, int stage, int32_t *err) {
  if (mbar_wait_bounded(&x.bars[stage], (x.parity >> stage) & 1u, x.wait_limit)) return true;
  x.parity ^= 1u << stage;
  x.dead = true;
  if (x.lane == 0) set_err(err, KV4_DEVERR_TIMEOUT);
  return false;
}

// After the wait for copy `failed` gave up: wait for copies from .. to-1 (every copy of
// the entry issued and not yet waited for, the one that timed out included, with the
// parity its wait had before it flipped), each up to 16 times the normal limit, so that
// none lands in shared memory after the warp (and possibly its CTA) has finished. A copy
// that does not complete even then is left behind; the TIMEOUT bit already marks the
// call's results as void. The warp takes no further work, so the parities are not kept.
__device__ inline void drain_copies(const WarpCtx &x, int from, int to, int failed) {
  const uint32_t longer = x.wait_limit > 0x0FFFFFFFu ? 0xFFFFFFFFu : x.wait_limit * 16u;
  for (int k = from; k < to; ++k) {
    if (!prologue_copy(x, k)) continue;  // withheld by the testing hook: never issued
    const int st = k % kStages;
    const uint32_t par = ((x.parity >> st) & 1u) ^ (k == failed ? 1u : 0u);
    mbar_wait_bounded(&x.bars[st], par, longer);
  }
}

// Per-warp state at the start of a persistent attention kernel. Kernels are instantiated
// twice: HOOK = false for normal calls (the constant wait limit and the absent hook fold
// into the code: nothing of the testing hook is left in it), HOOK = true only for a call
// with the testing hook armed (the wait limit and the withheld work item from the
// workspace descriptor).
template <bool HOOK>
__device__ __forceinline__ void init_warp(WarpCtx &x, const Workspace &w) {
  x.parity = 0;
  x.wait_limit = HOOK ? w.wait_limit : kWaitLimit;
  x.fault = false;
  x.dead = false;
}

template <bool HOOK>
__device__ __forceinline__ bool withheld_item(const Workspace &w, int item) {
  return HOOK && item == w.fault_item;
}

// Write the empty partial state (-inf, 0, 0) for the G heads of a record group.
__device__ inline void write_empty(float *rec, int G, int lane) {
  for (int j = 0; j < G; ++j) {
    float *r = rec + j * kRecordFloats;
    st_rec(reinterpret_cast<float4 *>(r) + lane, make_float4(0.f, 0.f, 0.f, 0.f));
    if (lane == 0) {
      st_rec(r + kHeadDim, -CUDART_INF_F);
      st_rec(r + kHeadDim + 1, 0.0f);
    }
  }
}

// Signature of a work list, written by the plan kernel into the workspace's header (ints
// 8..15) and checked by every kernel that reads the list: a call that reuses the list
// (kv4_batch.plan_reuse) with another batch shape or workspace layout is refused on the
// device (KV4_DEVERR_WORKSPACE) before any entry, offset or partial record is read.
constexpr int32_t kPlanMagic = 0x4b563450;
__device__ __forceinline__ void plan_signature(const CacheView &c, const Workspace &w,
                                               int32_t (&sig)[8]) {
  sig[0] = kPlanMagic;
  sig[1] = c.num_seqs;
  sig[2] = c.num_kv_heads;
  sig[3] = c.gqa | (w.heads_per_warp << 8) | (w.prefix_end != nullptr ? 1 << 16 : 0);
  sig[4] = w.chunk_pages;
  sig[5] = c.num_sinks | (c.num_recent << 16);
  sig[6] = w.cap_entries;
  sig[7] = w.cap_pairs;
}
__device__ __forceinline__ bool plan_matches(const CacheView &c, const Workspace &w) {
  int32_t want[8];
  plan_signature(c, w, want);
  const int32_t *have = w.counter + 8;
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) ok &= have[i] == want[i];
  return ok;
}

__device__ __forceinline__ float *record_of(const Workspace &w, int H, int G, int b, int h, int r) {
  return w.partials + static_cast<size_t>(w.unit_offsets[b * H + h] + r) * G * kRecordFloats;
}

__device__ __forceinline__ uint4 load_q8(const uint16_t *qrow, int dim0, bool live) {
  if (!live) return make_uint4(0, 0, 0, 0);
  return *reinterpret_cast<const uint4 *>(qrow + dim0);
}

// Fixed-point step of a query: 2^e with max|q| < 2^(e+14), so every |q / 2^e| <= 2^14
// (15 bits with the sign). amax is the lane's max|q|; the 4 lanes of a column combine.
__device__ __forceinline__ float query_step(float amax) {
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  int ex = 0;
  if (amax > 0.f) {
    frexpf(amax, &ex);  // amax < 2^ex
    ex -= 14;
  }
  return ldexpf(1.0f, ex);
}

}  // namespace kv4
