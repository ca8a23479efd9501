// Decode-step attention over the paged INT4 cache with INT8-protected sinks and recent
// window, split into regions whose partial softmax states are combined by an exact
// log-sum-exp merge (KV4-RL: "integer attention path and an exact regional softmax
// merge", ai4snews summary, "Interpretation" para. 3).
//
// Kernels:
//   plan_kernel  one CTA: turns seq_lens into a work list of (sequence, region) pairs
//                -- region 0 is the INT8 protected set, regions 1.. are chunks of
//                `chunk_pages` INT4 pages -- and the partial-record offsets per (b, h).
//   attn_kernel  persistent; every warp repeatedly takes one (pair, kv head) item from
//                an atomic counter and computes that region's partial state for the G
//                query heads of the kv head. Page tiles stream through a per-warp ring
//                of shared-memory stages filled by bulk async copies (TMA engine,
//                mbarrier completion). QK^T and PV run on the tensor cores
//                (mma m16n8k16, fp16 in, fp32 accumulate) directly on the integer codes:
//                codes are exact in fp16, and the per-group scale/min are applied
//                outside the dot products, so no dequantised K/V is ever materialised.
//   merge_kernel one warp per (b, h, query head): fixed-order exact merge -> bf16 out.
#include <math_constants.h>

#include "kv4_device.cuh"
#include "kv4_internal.h"

namespace kv4 {

constexpr int kWarps = 4;                 // warps per CTA (independent work streams)
constexpr int kStages = 3;                // shared-memory stages per warp
constexpr int kStageBytes = 4224;         // >= one INT8 tile (4160 B), multiple of 128
constexpr int kPtileBytes = 4 * 8 * 16 * 2;  // P' tile: [4 groups][8 heads][16 tokens] fp16
constexpr int kWarpSmem = kStages * kStageBytes + kPtileBytes + 64;
constexpr int kCtaSmem = kWarps * kWarpSmem;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegBig = -1.0e30f;  // running-max start: finite, so e^(m_old-m_new) is 0 not NaN

// INT4 stage: K codes | V codes | K params | V params
constexpr int kOffVc4 = 1024, kOffKp4 = 2048, kOffVp4 = 2304, kInt4Bytes = 2560;
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
  int has_prot;     // 1 if the INT8 protected set is non-empty
  int first_page;   // first page of the INT4 range
  int int4_lo, int4_hi;  // INT4 token range [lo, hi)
  int n_chunks;
};

__device__ __forceinline__ Regions regions_of(int L, int S, int R, int C) {
  Regions g;
  const int n_sink = min(S, L);
  const int rec_lo = max(S, L - R);
  g.has_prot = (n_sink > 0 || rec_lo < L) ? 1 : 0;
  g.int4_lo = S;
  g.int4_hi = L - R;
  if (g.int4_hi > g.int4_lo) {
    g.first_page = g.int4_lo / kPage;
    const int last = (g.int4_hi - 1) / kPage;
    g.n_chunks = (last - g.first_page + 1 + C - 1) / C;
  } else {
    g.first_page = 0;
    g.n_chunks = 0;
  }
  return g;
}

// ---------------------------------------------------------------------------
// plan: one CTA, 1024 threads
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__device__ int block_exclusive_scan(int v, int *sh, int *total) {
  const int tid = threadIdx.x;
  sh[tid] = v;
  __syncthreads();
  for (int off = 1; off < kPlanThreads; off <<= 1) {
    int t = tid >= off ? sh[tid - off] : 0;
    __syncthreads();
    sh[tid] += t;
    __syncthreads();
  }
  int incl = sh[tid];
  *total = sh[kPlanThreads - 1];
  __syncthreads();
  return incl - v;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(CacheView c, Workspace w,
                                                            int32_t *err) {
  __shared__ int sh[kPlanThreads];
  const int B = c.num_seqs, H = c.num_kv_heads, C = w.chunk_pages;
  const int S = c.num_sinks, R = c.num_recent;
  // pass 1: total number of pairs
  int carry = 0;
  for (int base = 0; base < B; base += kPlanThreads) {
    const int b = base + threadIdx.x;
    int items = 0;
    if (b < B) {
      int L = c.seq_lens[b];
      if (L < 0 || L > c.max_pages * kPage) L = 0;
      Regions g = regions_of(L, S, R, C);
      items = g.has_prot + g.n_chunks;
    }
    int tot;
    block_exclusive_scan(items, sh, &tot);
    carry += tot;
  }
  const bool fits = carry <= w.cap_pairs;
  // pass 2: write pairs and offsets (all-empty units if the workspace is too small)
  int run = 0;
  for (int base = 0; base < B; base += kPlanThreads) {
    const int b = base + threadIdx.x;
    int items = 0;
    if (b < B) {
      int L = c.seq_lens[b];
      if (L < 0 || L > c.max_pages * kPage) {
        set_err(err, KV4_DEVERR_SEQ_LEN);
        L = 0;
      }
      Regions g = regions_of(L, S, R, C);
      items = fits ? g.has_prot + g.n_chunks : 0;
    }
    int tot;
    const int off = run + block_exclusive_scan(items, sh, &tot);
    if (b < B) {
      for (int r = 0; r < items; ++r) w.pairs[off + r] = make_int2(b, r);
      for (int h = 0; h < H; ++h) w.unit_offsets[b * H + h] = H * off + h * items;
    }
    run += tot;
  }
  if (threadIdx.x == 0) {
    w.unit_offsets[B * H] = H * run;
    *w.n_items = run * H;
    *w.counter = 0;
    if (!fits) set_err(err, KV4_DEVERR_WORKSPACE);
  }
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------
struct WarpCtx {
  uint8_t *stage0;     // first stage (generic pointer)
  uint16_t *ptile;     // P' tile
  uint64_t *bars;      // kStages mbarriers
  uint32_t parity;     // bit s = parity of the next completion of stage s
  int lane, gid, tig;
  bool dead;           // a bounded wait gave up: stop taking work
};

// Online softmax update for this thread's two heads (2tig, 2tig+1) with logits of
// tokens (gid, gid+8) in log2 units. Returns p in s[][] and the rescale factors.
__device__ __forceinline__ void softmax_step(float (&s)[2][2], float (&m)[2], float (&l)[2],
                                             float (&alpha)[2]) {
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float t = fmaxf(s[0][e], s[1][e]);
    t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 4));
    t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 8));
    t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 16));
    const float mn = fmaxf(m[e], t);
    alpha[e] = fast_exp2(m[e] - mn);
    m[e] = mn;
    s[0][e] = fast_exp2(s[0][e] - mn);
    s[1][e] = fast_exp2(s[1][e] - mn);
    l[e] = l[e] * alpha[e] + s[0][e] + s[1][e];
  }
}

__device__ __forceinline__ bool wait_stage(WarpCtx &x, int stage, int32_t *err) {
  const bool ok = mbar_wait_bounded(&x.bars[stage], (x.parity >> stage) & 1u);
  x.parity ^= 1u << stage;
  if (!ok) {
    x.dead = true;
    if (x.lane == 0) set_err(err, KV4_DEVERR_TIMEOUT);
  }
  return ok;
}

// Write the empty partial state (-inf, 0, 0) for the G heads of an item.
__device__ void write_empty(float *rec, int G, int lane) {
  for (int j = 0; j < G; ++j) {
    float *r = rec + j * kRecordFloats;
    reinterpret_cast<float4 *>(r)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0) {
      r[kHeadDim] = -CUDART_INF_F;
      r[kHeadDim + 1] = 0.0f;
    }
  }
}

// Load this lane's query values: head gid (zero if gid >= G), dims off..off+7 for the
// given offsets, converted to fp16 (exact for |q| in fp16's normal range).
__device__ __forceinline__ uint4 load_q8(const uint16_t *qrow, int dim0, bool live) {
  if (!live) return make_uint4(0, 0, 0, 0);
  return *reinterpret_cast<const uint4 *>(qrow + dim0);
}

__device__ __forceinline__ float q_to_f16_pair(uint32_t bf2, uint32_t &out, bool &bad) {
  const float lo = __uint_as_float(bf2 << 16);
  const float hi = __uint_as_float(bf2 & 0xFFFF0000u);
  bad |= fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f;
  out = pack_h2(lo, hi);
  const float2 back = h2_to_f2(out);
  return back.x + back.y;
}

// ---------------------------- INT4 chunk --------------------------------
// Token order of the QK^T M-tile rows: rows 0-7 are tokens 0-7, rows 8-11 tokens 12-15,
// rows 12-15 tokens 8-11. With it a thread's two rows (gid, gid+8) are the tokens whose
// P' values it packs into one 32-bit word, the transposed V loads read those pairs, and
// neither the K nor the V ldmatrix phases hit a shared-memory bank twice.
__device__ __forceinline__ int row_token_hi(int r) { return 8 + ((r + 4) & 7); }

__device__ void process_int4(WarpCtx &x, const CacheView &c, const Workspace &w,
                             const uint16_t *__restrict__ q, int b, int h, int chunk,
                             const Regions &rg, float *rec, int32_t *err) {
  const int G = c.gqa, H = c.num_kv_heads;
  const int lane = x.lane, gid = x.gid, tig = x.tig;
  const int p0 = rg.first_page + chunk * w.chunk_pages;
  const int last = (rg.int4_hi - 1) / kPage;
  const int np = min(w.chunk_pages, last - p0 + 1);

  int pid = 0;
  if (lane < np) pid = c.page_table[static_cast<size_t>(b) * c.max_pages + p0 + lane];
  const bool bad = lane < np && (pid < 0 || pid >= c.num_pages);
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) set_err(err, KV4_DEVERR_PAGE_ID);
    write_empty(rec, G, lane);
    return;
  }

  auto issue = [&](int k) {
    const int pk = __shfl_sync(0xffffffffu, pid, k);
    if (lane == 0) {
      const int st = k % kStages;
      uint8_t *dst = x.stage0 + st * kStageBytes;
      const size_t blk = static_cast<size_t>(pk) * H + h;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&x.bars[st], kInt4Bytes);
      bulk_g2s(dst, c.k_codes + blk * kInt4CodeBytes, kInt4CodeBytes, &x.bars[st]);
      bulk_g2s(dst + kOffVc4, c.v_codes + blk * kInt4CodeBytes, kInt4CodeBytes, &x.bars[st]);
      bulk_g2s(dst + kOffKp4, reinterpret_cast<const uint8_t *>(c.k_params) + blk * kInt4ParamBytes,
               kInt4ParamBytes, &x.bars[st]);
      bulk_g2s(dst + kOffVp4, reinterpret_cast<const uint8_t *>(c.v_params) + blk * kInt4ParamBytes,
               kInt4ParamBytes, &x.bars[st]);
    }
  };
  const int npre = min(np, kStages);
  for (int k = 0; k < npre; ++k) issue(k);

  // ---- query fragments (B operand of QK^T), head gid, k-slot order matching nib_pairs4 ----
  // group g, k-tile kt: b01 = (q[32g+8tig+2kt], q[..+4]), b23 = (q[..+2kt+1], q[..+2kt+5])
  uint32_t qb[4][2][2];
  float qsum_own[4];
  bool qbad = false;
  {
    const bool live = gid < G;
    const uint16_t *qrow = q + (static_cast<size_t>(b) * c.num_kv_heads * G + h * G + gid) * kHeadDim;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint4 v = load_q8(qrow, 32 * g + 8 * tig, live);  // bf16 dims +0..+7
      const uint32_t p04 = (v.x & 0xFFFFu) | (v.z << 16);
      const uint32_t p15 = (v.x >> 16) | (v.z & 0xFFFF0000u);
      const uint32_t p26 = (v.y & 0xFFFFu) | (v.w << 16);
      const uint32_t p37 = (v.y >> 16) | (v.w & 0xFFFF0000u);
      float sum = 0.f;
      sum += q_to_f16_pair(p04, qb[g][0][0], qbad);
      sum += q_to_f16_pair(p15, qb[g][0][1], qbad);
      sum += q_to_f16_pair(p26, qb[g][1][0], qbad);
      sum += q_to_f16_pair(p37, qb[g][1][1], qbad);
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      qsum_own[g] = sum;  // sum over the group's 32 dims for head gid
    }
  }
  if (qbad) set_err(err, KV4_DEVERR_Q_RANGE);
  float2 qs[4];  // (head 2tig, head 2tig+1) sums, matching the C-fragment columns
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    qs[g].x = __shfl_sync(0xffffffffu, qsum_own[g], 4 * (2 * tig));
    qs[g].y = __shfl_sync(0xffffffffu, qsum_own[g], 4 * (2 * tig + 1));
  }

  float m[2] = {kNegBig, kNegBig}, l[2] = {0.f, 0.f};
  // o[g][mt][e] = (dim 32g+4gid+2mt, dim +1) of head 2tig+e
  float2 o[4][2][2];
  float2 mtp[4][2];  // sum p * vmin per group and head, split over the thread's two tokens
#pragma unroll
  for (int g = 0; g < 4; ++g)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      mtp[g][e] = make_float2(0.f, 0.f);
      o[g][0][e] = make_float2(0.f, 0.f);
      o[g][1][e] = make_float2(0.f, 0.f);
    }

  // ldmatrix lane addresses: matrix m = lane/8 covers strip m/2 (256 B each), row r = lane%8
  const int r8 = lane & 7;
  const int mhalf = (lane >> 3) & 1;
  const int strip_off = (lane >> 4) * 256;
  const int ld_k = strip_off + (mhalf ? row_token_hi(r8) : r8) * 16;
  // transposed V: matrix "lo" rows (2i, 2i+1) = tokens (i, 12+i), "hi" = (4+i, 8+i)
  const int ld_v = strip_off + (mhalf ? ((r8 & 1) ? 8 + (r8 >> 1) : 4 + (r8 >> 1))
                                      : ((r8 & 1) ? 12 + (r8 >> 1) : (r8 >> 1))) * 16;
  const int t0 = gid, t1 = row_token_hi(gid);  // tokens of this thread's C rows gid, gid+8
  const int tok_lo = rg.int4_lo, tok_hi = rg.int4_hi;
  uint32_t *ptw = reinterpret_cast<uint32_t *>(x.ptile);  // [4 g][8 heads][8 token pairs]
  const float2 kappa = make_float2(kLog2e * 0.08838834764831845f, kLog2e * 0.08838834764831845f);

  for (int k = 0; k < np; ++k) {
    const int st = k % kStages;
    if (!wait_stage(x, st, err)) {
      for (int kk = k + 1; kk < min(np, k + kStages); ++kk) wait_stage(x, kk % kStages, err);
      write_empty(rec, G, lane);
      return;
    }
    uint8_t *sp = x.stage0 + st * kStageBytes;
    const uint32_t sa = smem_u32(sp);

    // ---- S^T = K Q^T, one fp32 accumulator per 32-dim group ----
    uint32_t kw[2][4];
    ldsm_x4(kw[0], sa + ld_k);
    ldsm_x4(kw[1], sa + 512 + ld_k);
    float acc[4][4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t pl[4], ph[4];
      nib_pairs4(kw[g >> 1][(g & 1) * 2], pl);
      nib_pairs4(kw[g >> 1][(g & 1) * 2 + 1], ph);
      acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
      mma_f16(acc[g], pl[0], ph[0], pl[1], ph[1], qb[g][0][0], qb[g][0][1]);
      mma_f16(acc[g], pl[2], ph[2], pl[3], ph[3], qb[g][1][0], qb[g][1][1]);
    }
    // ---- logits: s = sum_g scale_g * (q . c)_g + min_g * sum_g(q), log2 units ----
    const uint4 kp[2] = {*reinterpret_cast<const uint4 *>(sp + kOffKp4 + t0 * 16),
                         *reinterpret_cast<const uint4 *>(sp + kOffKp4 + t1 * 16)};
    float2 sl[2];  // sl[hf] = logits of token (t0 | t1) for heads (2tig, 2tig+1)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t pw[4] = {kp[hf].x, kp[hf].y, kp[hf].z, kp[hf].w};
      float2 v = make_float2(0.f, 0.f);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float2 sm = h2_to_f2(pw[g]);
        v = ffma2(make_float2(sm.x, sm.x), make_float2(acc[g][2 * hf], acc[g][2 * hf + 1]), v);
        v = ffma2(make_float2(sm.y, sm.y), qs[g], v);
      }
      sl[hf] = fmul2(v, kappa);
    }
    const int tok0 = (p0 + k) * kPage;
    if (tok0 < tok_lo || tok0 + kPage > tok_hi) {  // ragged first/last page of the range
      const bool v0 = tok0 + t0 >= tok_lo && tok0 + t0 < tok_hi;
      const bool v1 = tok0 + t1 >= tok_lo && tok0 + t1 < tok_hi;
      if (!v0) sl[0] = make_float2(-CUDART_INF_F, -CUDART_INF_F);
      if (!v1) sl[1] = make_float2(-CUDART_INF_F, -CUDART_INF_F);
    }
    // ---- online softmax; the rescale is skipped while no running max moves ----
    float p[2][2];
    float2 alpha2[2];
    bool moved = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float s0 = e ? sl[0].y : sl[0].x, s1 = e ? sl[1].y : sl[1].x;
      float t = fmaxf(s0, s1);
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 4));
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 8));
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 16));
      const float mn = fmaxf(m[e], t);
      const float a = mn != m[e] ? fast_exp2(m[e] - mn) : 1.0f;
      moved |= mn != m[e];
      m[e] = mn;
      p[0][e] = fast_exp2(s0 - mn);
      p[1][e] = fast_exp2(s1 - mn);
      l[e] = fmaf(l[e], a, p[0][e] + p[1][e]);
      alpha2[e] = make_float2(a, a);
    }
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          mtp[g][e] = fmul2(mtp[g][e], alpha2[e]);
          o[g][0][e] = fmul2(o[g][0][e], alpha2[e]);
          o[g][1][e] = fmul2(o[g][1][e], alpha2[e]);
        }
    }
    // ---- P'_g = p * vscale_g as fp16 token pairs; sum p * vmin_g on the side ----
    const uint4 vp[2] = {*reinterpret_cast<const uint4 *>(sp + kOffVp4 + t0 * 16),
                         *reinterpret_cast<const uint4 *>(sp + kOffVp4 + t1 * 16)};
    const float2 pe[2] = {make_float2(p[0][0], p[1][0]), make_float2(p[0][1], p[1][1])};
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t w0 = g == 0 ? vp[0].x : g == 1 ? vp[0].y : g == 2 ? vp[0].z : vp[0].w;
      const uint32_t w1 = g == 0 ? vp[1].x : g == 1 ? vp[1].y : g == 2 ? vp[1].z : vp[1].w;
      const float2 f0 = h2_to_f2(w0), f1 = h2_to_f2(w1);
      const float2 sv = make_float2(f0.x, f1.x), mv = make_float2(f0.y, f1.y);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = 2 * tig + e;
        const float2 pv = fmul2(pe[e], sv);
        if (j < G) ptw[(g * 8 + j) * 8 + gid] = pack_h2(pv.x, pv.y);
        mtp[g][e] = ffma2(pe[e], mv, mtp[g][e]);
      }
    }
    __syncwarp();
    // ---- O^T += V^T P' per group: A = V codes (transposed ldmatrix), B = P'_g ----
    uint32_t vw[2][4];
    ldsm_x4_t(vw[0], sa + kOffVc4 + ld_v);
    ldsm_x4_t(vw[1], sa + kOffVc4 + 512 + ld_v);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t vl[4], vh[4];
      nib_pairs4(vw[g >> 1][(g & 1) * 2], vl);
      nib_pairs4(vw[g >> 1][(g & 1) * 2 + 1], vh);
      uint32_t b01 = 0, b23 = 0;
      if (gid < G) {
        b01 = ptw[(g * 8 + gid) * 8 + tig];
        b23 = ptw[(g * 8 + gid) * 8 + tig + 4];
      }
      float c0[4] = {o[g][0][0].x, o[g][0][1].x, o[g][0][0].y, o[g][0][1].y};
      mma_f16(c0, vl[0], vl[1], vh[0], vh[1], b01, b23);
      o[g][0][0] = make_float2(c0[0], c0[2]);
      o[g][0][1] = make_float2(c0[1], c0[3]);
      float c1[4] = {o[g][1][0].x, o[g][1][1].x, o[g][1][0].y, o[g][1][1].y};
      mma_f16(c1, vl[2], vl[3], vh[2], vh[3], b01, b23);
      o[g][1][0] = make_float2(c1[0], c1[2]);
      o[g][1][1] = make_float2(c1[1], c1[3]);
    }
    __syncwarp();
    if (k + kStages < np) issue(k + kStages);
  }

  // ---- finish: reduce per-thread sums over the 8 token lanes, write the partial ----
  float mt[4][2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], off);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      mt[g][e] = mtp[g][e].x + mtp[g][e].y;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
        mt[g][e] += __shfl_xor_sync(0xffffffffu, mt[g][e], off);
    }
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int j = 2 * tig + e;
    if (j < G) {
      float *r = rec + j * kRecordFloats;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 v = make_float4(o[g][0][e].x + mt[g][e], o[g][0][e].y + mt[g][e],
                                     o[g][1][e].x + mt[g][e], o[g][1][e].y + mt[g][e]);
        *reinterpret_cast<float4 *>(r + 32 * g + 4 * gid) = v;
      }
      if (gid == 0) {
        r[kHeadDim] = m[e] * kLn2;
        r[kHeadDim + 1] = l[e];
      }
    }
  }
}

// ------------------------- INT8 protected set ----------------------------
__device__ void process_protected(WarpCtx &x, const CacheView &c, const uint16_t *__restrict__ q,
                                  int b, int h, int L, float *rec, int32_t *err) {
  const int G = c.gqa, H = c.num_kv_heads;
  const int lane = x.lane, gid = x.gid, tig = x.tig;
  const int S = c.num_sinks, R = c.num_recent;
  const int n_sink = min(S, L);
  const int rec_lo = max(S, L - R);
  const int sink_tiles = (n_sink + kPage - 1) / kPage;
  const int ring_tiles = rec_lo < L ? (R + kPage - 1) / kPage : 0;
  const int nt = sink_tiles + ring_tiles;

  const int set = sink_tiles ? (c.sink_idx ? c.sink_idx[b] : b) : 0;
  const int ring = ring_tiles ? (c.ring_idx ? c.ring_idx[b] : b) : 0;
  if ((sink_tiles && (set < 0 || set >= c.num_sink_sets)) ||
      (ring_tiles && (ring < 0 || ring >= c.num_rings))) {
    if (lane == 0) set_err(err, KV4_DEVERR_SIDE_IDX);
    write_empty(rec, G, lane);
    return;
  }

  auto issue = [&](int k) {
    if (lane == 0) {
      const int st = k % kStages;
      uint8_t *dst = x.stage0 + st * kStageBytes;
      const int8_t *kc, *vc;
      const uint16_t *ks, *vs;
      if (k < sink_tiles) {
        const size_t t = (static_cast<size_t>(set) * H + h) * c.sink_tiles + k;
        kc = c.sink_k + t * kInt8CodeBytes; vc = c.sink_v + t * kInt8CodeBytes;
        ks = c.sink_ks + t * kPage; vs = c.sink_vs + t * kPage;
      } else {
        const size_t t = (static_cast<size_t>(ring) * H + h) * c.ring_tiles + (k - sink_tiles);
        kc = c.ring_k + t * kInt8CodeBytes; vc = c.ring_v + t * kInt8CodeBytes;
        ks = c.ring_ks + t * kPage; vs = c.ring_vs + t * kPage;
      }
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&x.bars[st], kInt8Bytes);
      bulk_g2s(dst, kc, kInt8CodeBytes, &x.bars[st]);
      bulk_g2s(dst + kOffVc8, vc, kInt8CodeBytes, &x.bars[st]);
      bulk_g2s(dst + kOffKs8, ks, kInt8ScaleBytes, &x.bars[st]);
      bulk_g2s(dst + kOffVs8, vs, kInt8ScaleBytes, &x.bars[st]);
    }
  };
  const int npre = min(nt, kStages);
  for (int k = 0; k < npre; ++k) issue(k);

  // query fragments for int8 strips: k-tile c: b01 = (q[16c+4tig], q[..+1]),
  // b23 = (q[16c+4tig+2], q[..+3])
  uint32_t qb[8][2];
  bool qbad = false;
  {
    const bool live = gid < G;
    const uint16_t *qrow = q + (static_cast<size_t>(b) * H * G + h * G + gid) * kHeadDim;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      uint2 v = live ? *reinterpret_cast<const uint2 *>(qrow + 16 * cc + 4 * tig) : make_uint2(0, 0);
      q_to_f16_pair(v.x, qb[cc][0], qbad);
      q_to_f16_pair(v.y, qb[cc][1], qbad);
    }
  }
  if (qbad) set_err(err, KV4_DEVERR_Q_RANGE);

  float m[2] = {kNegBig, kNegBig}, l[2] = {0.f, 0.f};
  float o[8][4];
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) o[cc][0] = o[cc][1] = o[cc][2] = o[cc][3] = 0.f;
  const int ld_off = ((lane >> 4) * 256) + ((lane >> 3) & 1) * 128 + (lane & 7) * 16;
  const int ring_base = L - R;  // ring slot s holds position ring_base + ((s - ring_base) mod R)

  for (int k = 0; k < nt; ++k) {
    const int st = k % kStages;
    if (!wait_stage(x, st, err)) {
      for (int kk = k + 1; kk < min(nt, k + kStages); ++kk) wait_stage(x, kk % kStages, err);
      write_empty(rec, G, lane);
      return;
    }
    uint8_t *sp = x.stage0 + st * kStageBytes;
    const uint32_t sa = smem_u32(sp);

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      uint32_t kw[4];
      ldsm_x4(kw, sa + pr * 512 + ld_off);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int cc = 2 * pr + hs;
        const uint32_t ulo = kw[2 * hs] ^ 0x80808080u, uhi = kw[2 * hs + 1] ^ 0x80808080u;
        mma_f16(acc, s8_pair<0x4140>(ulo), s8_pair<0x4140>(uhi), s8_pair<0x4342>(ulo),
                s8_pair<0x4342>(uhi), qb[cc][0], qb[cc][1]);
      }
    }
    const uint16_t *ks = reinterpret_cast<const uint16_t *>(sp + kOffKs8);
    const uint16_t *vs = reinterpret_cast<const uint16_t *>(sp + kOffVs8);
    float s[2][2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int slot = gid + 8 * hf;
      bool valid;
      if (k < sink_tiles) {
        valid = k * kPage + slot < n_sink;
      } else {
        const int rs = (k - sink_tiles) * kPage + slot;
        int d = (rs - ring_base) % R;
        if (d < 0) d += R;
        valid = rs < R && ring_base + d >= S;
      }
      const float sk = __half2float(__ushort_as_half(ks[slot]));
#pragma unroll
      for (int e = 0; e < 2; ++e)
        s[hf][e] = valid ? sk * acc[2 * hf + e] * (kLog2e * 0.08838834764831845f) : -CUDART_INF_F;
    }
    float alpha[2];
    softmax_step(s, m, l, alpha);
#pragma unroll
    for (int cc = 0; cc < 8; ++cc)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        o[cc][e] *= alpha[e];
        o[cc][2 + e] *= alpha[e];
      }
    const float sv0 = __half2float(__ushort_as_half(vs[gid]));
    const float sv1 = __half2float(__ushort_as_half(vs[gid + 8]));
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = 2 * tig + e;
      if (j < G) {
        x.ptile[j * 16 + gid] = __half_as_ushort(__float2half_rn(s[0][e] * sv0));
        x.ptile[j * 16 + gid + 8] = __half_as_ushort(__float2half_rn(s[1][e] * sv1));
      }
    }
    __syncwarp();
    uint32_t b01 = 0, b23 = 0;
    if (gid < G) {
      b01 = *reinterpret_cast<const uint32_t *>(&x.ptile[gid * 16 + 2 * tig]);
      b23 = *reinterpret_cast<const uint32_t *>(&x.ptile[gid * 16 + 2 * tig + 8]);
    }
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      uint32_t vw[4];
      ldsm_x4_t(vw, sa + kOffVc8 + pr * 512 + ld_off);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int cc = 2 * pr + hs;
        const uint32_t ulo = vw[2 * hs] ^ 0x80808080u, uhi = vw[2 * hs + 1] ^ 0x80808080u;
        mma_f16(o[cc], s8_pair<0x4240>(ulo), s8_pair<0x4341>(ulo), s8_pair<0x4240>(uhi),
                s8_pair<0x4341>(uhi), b01, b23);
      }
    }
    __syncwarp();
    if (k + kStages < nt) issue(k + kStages);
  }

#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], off);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int j = 2 * tig + e;
    if (j < G) {
      float *r = rec + j * kRecordFloats;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)  // rows: dim 16cc+2gid (c0/c1) and +1 (c2/c3)
        *reinterpret_cast<float2 *>(r + 16 * cc + 2 * gid) = make_float2(o[cc][e], o[cc][2 + e]);
      if (gid == 0) {
        r[kHeadDim] = m[e] * kLn2;
        r[kHeadDim + 1] = l[e];
      }
    }
  }
}

#ifndef KV4_MIN_BLOCKS
#define KV4_MIN_BLOCKS 4  // CTAs per SM the register budget is sized for
#endif

__global__ void __launch_bounds__(kWarps * 32, KV4_MIN_BLOCKS) attn_kernel(CacheView c, Workspace w,
                                                              const uint16_t *__restrict__ q,
                                                              int32_t *err) {
  extern __shared__ __align__(1024) uint8_t smem[];
  WarpCtx x;
  const int warp = threadIdx.x >> 5;
  x.lane = threadIdx.x & 31;
  x.gid = x.lane >> 2;
  x.tig = x.lane & 3;
  uint8_t *mine = smem + warp * kWarpSmem;
  x.stage0 = mine;
  x.ptile = reinterpret_cast<uint16_t *>(mine + kStages * kStageBytes);
  x.bars = reinterpret_cast<uint64_t *>(mine + kStages * kStageBytes + kPtileBytes);
  x.parity = 0;
  x.dead = false;
  if (x.lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&x.bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const int H = c.num_kv_heads, G = c.gqa;
  const int n_items = *w.n_items;
  for (;;) {
    int item = 0;
    if (x.lane == 0) item = atomicAdd(w.counter, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item >= n_items) break;
    const int pair = item / H;
    const int h = item - pair * H;
    const int2 pr = w.pairs[pair];
    const int b = pr.x, r = pr.y;
    const int L = c.seq_lens[b];
    const Regions rg = regions_of(L, c.num_sinks, c.num_recent, w.chunk_pages);
    float *rec = w.partials +
                 static_cast<size_t>(w.unit_offsets[b * H + h] + r) * G * kRecordFloats;
    if (r < rg.has_prot)
      process_protected(x, c, q, b, h, L, rec, err);
    else
      process_int4(x, c, w, q, b, h, r - rg.has_prot, rg, rec, err);
    if (x.dead) break;
  }
}

// ---------------------------------------------------------------------------
// exact regional merge
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) merge_kernel(const float *__restrict__ partials,
                                                    const int32_t *__restrict__ offs, int n_units,
                                                    int G, uint16_t *__restrict__ out,
                                                    float *__restrict__ out_f32,
                                                    float *__restrict__ lse) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_units * G) return;
  const int u = warp / G, j = warp - u * G;
  const int r0 = offs[u], r1 = offs[u + 1];
  float M = -CUDART_INF_F, lam = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = r0; r < r1; ++r) {
    const float *rec = partials + (static_cast<size_t>(r) * G + j) * kRecordFloats;
    const float mr = rec[kHeadDim], lr = rec[kHeadDim + 1];
    if (!(lr > 0.f)) continue;
    const float4 a = reinterpret_cast<const float4 *>(rec)[lane];
    if (mr > M) {
      const float sc = expf(M - mr);
      acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
      lam *= sc;
      M = mr;
    }
    const float wgt = expf(mr - M);
    acc.x = fmaf(a.x, wgt, acc.x);
    acc.y = fmaf(a.y, wgt, acc.y);
    acc.z = fmaf(a.z, wgt, acc.z);
    acc.w = fmaf(a.w, wgt, acc.w);
    lam = fmaf(lr, wgt, lam);
  }
  const float inv = lam > 0.f ? 1.0f / lam : 0.f;
  const float4 v = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  const size_t o = (static_cast<size_t>(u) * G + j) * kHeadDim + 4 * lane;
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t *>(&lo);
  packed.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(out + o) = packed;
  if (out_f32) *reinterpret_cast<float4 *>(out_f32 + o) = v;
  if (lse && lane == 0) lse[static_cast<size_t>(u) * G + j] = lam > 0.f ? M + logf(lam) : -CUDART_INF_F;
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_plan(const CacheView &c, const Workspace &w, int32_t *err_flag, cudaStream_t s) {
  plan_kernel<<<1, kPlanThreads, 0, s>>>(c, w, err_flag);
  return cudaGetLastError();
}

cudaError_t launch_attention(const CacheView &c, const Workspace &w, const uint16_t *q,
                             int32_t *err_flag, cudaStream_t s) {
  static int configured_device = -1;
  static int grid = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != configured_device) {
    e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCtaSmem);
    if (e != cudaSuccess) return e;
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_kernel, kWarps * 32, kCtaSmem);
    if (e != cudaSuccess) return e;
    grid = sms * (per_sm > 0 ? per_sm : 1);
    configured_device = dev;
  }
  attn_kernel<<<grid, kWarps * 32, kCtaSmem, s>>>(c, w, q, err_flag);
  return cudaGetLastError();
}

cudaError_t launch_merge(const float *partials, const int32_t *unit_offsets, int32_t n_units,
                         int32_t group, uint16_t *out, float *out_f32, float *lse, cudaStream_t s) {
  const long long warps = static_cast<long long>(n_units) * group;
  if (warps == 0) return cudaSuccess;
  const long long blocks = (warps * 32 + 255) / 256;
  merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(partials, unit_offsets, n_units, group,
                                                             out, out_f32, lse);
  return cudaGetLastError();
}

size_t workspace_bytes(int32_t num_seqs, int32_t max_seq_len, int32_t num_kv_heads, int32_t gqa,
                       int32_t chunk_pages, Workspace *carve, void *base) {
  const long long pages = (static_cast<long long>(max_seq_len) + kPage - 1) / kPage + 1;
  const long long per_seq = 1 + (pages + chunk_pages - 1) / chunk_pages;
  const long long cap = static_cast<long long>(num_seqs) * per_seq;
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  size_t off = 256;  // counter, n_items
  const size_t pairs_off = off;
  off = up(off + static_cast<size_t>(cap) * sizeof(int2));
  const size_t units_off = off;
  off = up(off + (static_cast<size_t>(num_seqs) * num_kv_heads + 1) * sizeof(int32_t));
  const size_t part_off = off;
  off = up(off + static_cast<size_t>(cap) * num_kv_heads * gqa * kRecordFloats * sizeof(float));
  if (carve) {
    uint8_t *p = static_cast<uint8_t *>(base);
    carve->counter = reinterpret_cast<int32_t *>(p);
    carve->n_items = reinterpret_cast<int32_t *>(p) + 1;
    carve->pairs = reinterpret_cast<int2 *>(p + pairs_off);
    carve->unit_offsets = reinterpret_cast<int32_t *>(p + units_off);
    carve->partials = reinterpret_cast<float *>(p + part_off);
    carve->cap_pairs = static_cast<int32_t>(cap);
    carve->chunk_pages = chunk_pages;
  }
  return off;
}

}  // namespace kv4
