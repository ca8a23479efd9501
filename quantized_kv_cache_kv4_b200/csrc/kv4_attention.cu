// Decode-step attention over the paged INT4 cache with INT8-protected sinks and recent
// window, split into regions whose partial softmax states are combined by an exact
// log-sum-exp merge (KV4-RL: "integer attention path and an exact regional softmax
// merge", ai4snews summary, "Interpretation" para. 3).
//
// Kernels:
//   plan_kernel  turns seq_lens into a work list. Region 0 of a sequence is its INT8
//                protected set; then the regions of its group's shared INT4 pages (if
//                any); then chunks of `chunk_pages` of its own INT4 pages; one entry per
//                region and one or two kv heads. Entries
//                come in four classes (full chunks, long partial chunks, protected sets,
//                short chunks) so that the longest work starts first.
//   attn_kernel  persistent; every warp repeatedly takes one entry from an atomic counter
//                and computes the partial softmax state of that region for the query
//                heads of its kv head(s). Page tiles stream through a per-warp ring of
//                shared-memory stages filled by bulk async copies (TMA engine, mbarrier
//                completion). Both products run on the tensor cores directly on the
//                integer codes, and the per-group scale/min are applied outside them, so
//                no dequantised K/V is ever materialised:
//                  QK^T  integer MMA (m16n8k32): K codes as bytes times the query in
//                        15-bit fixed point split into a signed high and an unsigned low
//                        byte, exact int32 dot products;
//                  PV    fp16 MMA (m16n8k16, fp32 accumulate): V codes masked into fp16
//                        subnormals (exact, no conversion), P' = p * vscale rounded once
//                        to fp16.
//                With G <= 4 query heads per kv head one warp serves two kv heads: the MMA
//                N dimension (8) holds head A's queries in columns 0-3 and head B's in
//                columns 4-7 (zeros in the other half of each B operand), so every lane's
//                softmax and scaling work is useful.
//   prefix_kernel the shared-prefix read (kv4_config.prefix_mode): consecutive sequences
//                whose page tables map their leading INT4 pages to the same physical pages
//                (the responses of one prompt, ai4snews summary, "Interpretation" para. 3:
//                groups of eight responses) form a group; one warp reads each shared page
//                of a kv head once for up to four members (16 query columns, two MMA N
//                tiles) and writes one partial state per member, merged as an extra
//                region. The members' own chunks start after the shared pages.
//   merge_kernel one warp per (unit, query): fixed-order exact merge -> bf16 out; also
//                the kernel behind kv4_regional_merge.
#include <math_constants.h>

#include "kv4_attn_common.cuh"
#include "kv4_plan.cuh"

namespace kv4 {

// ---------------------------------------------------------------------------
// plan (kv4_plan.cuh): a few CTAs; each scans all sequences and writes its slice.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(CacheView c, Workspace w,
                                                            int32_t *err) {
  plan_block(c, w, err, blockIdx.x, gridDim.x);
}

// How an entry's probability weights are formed (see lift_for_scale):
//   kDecide  attn_kernel, every entry: no lift; when its last page's V scales are small
//            enough to want one (lift >= kLiftMin; checked after the page loop, where it
//            costs the loop nothing), the entry writes nothing and returns kWantLift (it
//            goes on the lift list);
//   kLifted  lift_kernel, for the listed entries: with the lift; returns kOverflow,
//            having written nothing, when a later weight overflowed fp16;
//   kPlain   lift_kernel, after an overflow: no lift and no decision.
// The lifted arithmetic lives in its own kernel because attn_kernel runs at its register
// limit: compiled into it, even unused, it slowed the main path by several percent.
constexpr int kDecide = 0, kLifted = 1, kPlain = 2;
constexpr int kDone = 0, kWantLift = 1, kOverflow = 2;
constexpr float kLiftMin = 6.0f;  // lift only weights whose largest V scale is below 2^-6

// ------------------------- INT8 protected set ----------------------------
// One kv head's protected set: sink tiles then recent-ring tiles, INT8 codes.
// Returns kDone, kWantLift (MODE kDecide) or kOverflow (MODE kLifted).
template <int MODE>
__device__ __forceinline__ int process_protected(WarpCtx &x, const CacheView &c, const uint16_t *__restrict__ q,
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
    return kDone;
  }

  auto issue = [&](int k) {
    const int st = k % kStages;
    if (lane == 0) {
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
  for (int k = 0; k < npre; ++k)
    if (prologue_copy(x, k)) issue(k);

  // query fragments (B operand of QK^T, m16n8k32): lane column gid = query gid; k-step
  // ks: b0 = dims 32ks+4tig..+3, b1 = dims 32ks+16+4tig..+3, as bytes of
  // q / qstep = 256*hi + lo
  uint32_t qh[4][2], ql[4][2];
  float2 kq;  // qstep * log2(e)/sqrt(d) of the C-fragment columns (2tig, 2tig+1)
  {
    const bool live = gid < G;
    const uint16_t *qrow = q + (static_cast<size_t>(b) * H * G + h * G + gid) * kHeadDim;
    float qv[4][2][4];
    float amax = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint2 v = live ? *reinterpret_cast<const uint2 *>(qrow + 32 * ks + 16 * hf + 4 * tig)
                             : make_uint2(0u, 0u);
        qv[ks][hf][0] = __uint_as_float(v.x << 16);
        qv[ks][hf][1] = __uint_as_float(v.x & 0xFFFF0000u);
        qv[ks][hf][2] = __uint_as_float(v.y << 16);
        qv[ks][hf][3] = __uint_as_float(v.y & 0xFFFF0000u);
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(qv[ks][hf][i]));
      }
    const float qstep = query_step(amax);
    const float inv = 1.0f / qstep;  // a power of two: exact
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t hb = 0u, lb = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int qi = __float2int_rn(qv[ks][hf][i] * inv);
          lb |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * i);
          hb |= (static_cast<uint32_t>(qi >> 8) & 0xFFu) << (8 * i);
        }
        qh[ks][hf] = hb;
        ql[ks][hf] = lb;
      }
    kq.x = __shfl_sync(0xffffffffu, qstep, 4 * (2 * tig)) * kScaleLog2;
    kq.y = __shfl_sync(0xffffffffu, qstep, 4 * (2 * tig + 1)) * kScaleLog2;
  }

  float m[2] = {kNegBig, kNegBig}, l[2] = {0.f, 0.f};
  float o[8][4];
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) o[cc][0] = o[cc][1] = o[cc][2] = o[cc][3] = 0.f;
  const int ld_off = ((lane >> 4) * 256) + ((lane >> 3) & 1) * 128 + (lane & 7) * 16;
  const int ring_base = L - R;  // ring slot s holds position ring_base + ((s - ring_base) mod R)
  float lift = 0.f;
  if (MODE == kLifted) {  // the lift from the largest V scale of the first tile
    if (!peek_stage(x, 0, err)) {
      drain_copies(x, 0, npre, 0);
      write_empty(rec, G, lane);
      return kDone;
    }
    const uint16_t *v0 = reinterpret_cast<const uint16_t *>(x.stage0 + kOffVs8);
    lift = lift_for_scale(page_max_scale(max(v0[gid], v0[gid + 8])));
  }

  for (int k = 0; k < nt; ++k) {
    const int st = k % kStages;
    if (!wait_stage(x, st, err)) {
      drain_copies(x, k, min(nt, k + kStages), k);
      write_empty(rec, G, lane);
      return kDone;
    }
    uint8_t *sp = x.stage0 + st * kStageBytes;
    const uint32_t sa = smem_u32(sp);

    int32_t ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t kw[4];  // rows = positions, k = dims 32ks..32ks+31
      ldsm_x4(kw, sa + ks * 512 + ld_off);
      mma_s8s8(ah, kw[0], kw[1], kw[2], kw[3], qh[ks][0], qh[ks][1]);
      mma_s8u8(al, kw[0], kw[1], kw[2], kw[3], ql[ks][0], ql[ks][1]);
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
      // exact integer dot products: |.| < 2^29
      const float d0 = static_cast<float>(ah[2 * hf] * 256 + al[2 * hf]);
      const float d1 = static_cast<float>(ah[2 * hf + 1] * 256 + al[2 * hf + 1]);
      s[hf][0] = valid ? d0 * sk * kq.x : -CUDART_INF_F;
      s[hf][1] = valid ? d1 * sk * kq.y : -CUDART_INF_F;
    }
    float alpha[2];
    softmax_step(s, m, l, alpha, lift);
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
        x.ptile8[j * 16 + gid] = __half_as_ushort(__float2half_rn(s[0][e] * sv0));
        x.ptile8[j * 16 + gid + 8] = __half_as_ushort(__float2half_rn(s[1][e] * sv1));
      }
    }
    __syncwarp();
    uint32_t b01 = 0, b23 = 0;
    if (gid < G) {
      b01 = *reinterpret_cast<const uint32_t *>(&x.ptile8[gid * 16 + 2 * tig]);
      b23 = *reinterpret_cast<const uint32_t *>(&x.ptile8[gid * 16 + 2 * tig + 8]);
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

  if (MODE == kLifted) {
    const float probe[2] = {o[0][0], o[0][1]};
    if (any_not_finite(probe)) return kOverflow;
  }
  if (MODE == kDecide) {  // the last tile's V scales (still staged) ask for the lift?
    const uint16_t *vl = reinterpret_cast<const uint16_t *>(
        x.stage0 + ((nt - 1) % kStages) * kStageBytes + kOffVs8);
    if (lift_for_scale(page_max_scale(max(vl[gid], vl[gid + 8]))) >= kLiftMin) return kWantLift;
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
        st_rec(reinterpret_cast<float2 *>(r + 16 * cc + 2 * gid), make_float2(o[cc][e], o[cc][2 + e]));
      if (gid == 0) {
        st_rec(r + kHeadDim, m[e] * kLn2);
        st_rec(r + kHeadDim + 1, l[e]);
      }
    }
  }
  return kDone;
}


// ------------------- INT8 protected set, two kv heads per warp -------------------
// The protected sets of kv heads h0 and h0+1 (G <= 4) in the column layout of the INT4
// pair path: MMA N columns 0-3 are head slot 0's queries, 4-7 slot 1's. A tile of 16
// positions takes two ring stages: first the K codes and scales of both heads, then their
// V codes and scales, so the K stage is refilled as soon as the logits are taken.
// QK^T on the integer tensor cores: int8 K codes times the query in 15-bit fixed point
// (signed high byte, unsigned low byte), exact int32 dot products; the per-token K scale
// and the query step are applied to the sums in fp32. PV as in the one-head path.
constexpr int kOffScale8P = 2 * kInt8CodeBytes;                       // scales of slot hs at +32 hs
constexpr int kInt8PairBytes = 2 * kInt8CodeBytes + 2 * kInt8ScaleBytes;  // 4160 per stage

// Returns kDone, kWantLift (MODE kDecide) or kOverflow (MODE kLifted).
template <int MODE>
__device__ __forceinline__ int process_protected_pair(WarpCtx &x, const CacheView &c, const Workspace &w,
                                       const uint16_t *__restrict__ q, int b, int h0, int nh,
                                       int L, int r, int32_t *err) {
  constexpr int CPH = 4;  // MMA columns per kv head slot
  const int G = c.gqa, H = c.num_kv_heads;
  const int lane = x.lane, gid = x.gid, tig = x.tig;
  const int S = c.num_sinks, R = c.num_recent;
  const int n_sink = min(S, L);
  const int rec_lo = max(S, L - R);
  const int sink_tiles = (n_sink + kPage - 1) / kPage;
  const int ring_tiles = rec_lo < L ? (R + kPage - 1) / kPage : 0;
  const int nt = sink_tiles + ring_tiles;
  const int nv = 2 * nt;  // copies: the K part, then the V part, of every tile
  // this lane's C-fragment columns 2tig, 2tig+1: head slot and query index
  const int hs_c = (2 * tig) / CPH;
  const int jc0 = (2 * tig) % CPH;
  const bool head_c_live = hs_c < nh;

  const int set = sink_tiles ? (c.sink_idx ? c.sink_idx[b] : b) : 0;
  const int ring = ring_tiles ? (c.ring_idx ? c.ring_idx[b] : b) : 0;
  if ((sink_tiles && (set < 0 || set >= c.num_sink_sets)) ||
      (ring_tiles && (ring < 0 || ring >= c.num_rings))) {
    if (lane == 0) set_err(err, KV4_DEVERR_SIDE_IDX);
    for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
    return kDone;
  }

  // copy k: tile k/2, K part (k even) or V part (k odd), both heads; a spare slot (one
  // head left) gets a copy of head h0
  auto issue = [&](int k) {
    const int st = k % kStages;
    if (lane == 0) {
      uint8_t *dst = x.stage0 + st * kStageBytes;
      const int tile = k >> 1;
      const bool vpart = (k & 1) != 0;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&x.bars[st], kInt8PairBytes);
      for (int hs = 0; hs < 2; ++hs) {
        const int h = h0 + (hs < nh ? hs : 0);
        const int8_t *codes;
        const uint16_t *scales;
        if (tile < sink_tiles) {
          const size_t t = (static_cast<size_t>(set) * H + h) * c.sink_tiles + tile;
          codes = (vpart ? c.sink_v : c.sink_k) + t * kInt8CodeBytes;
          scales = (vpart ? c.sink_vs : c.sink_ks) + t * kPage;
        } else {
          const size_t t =
              (static_cast<size_t>(ring) * H + h) * c.ring_tiles + (tile - sink_tiles);
          codes = (vpart ? c.ring_v : c.ring_k) + t * kInt8CodeBytes;
          scales = (vpart ? c.ring_vs : c.ring_ks) + t * kPage;
        }
        bulk_g2s(dst + hs * kInt8CodeBytes, codes, kInt8CodeBytes, &x.bars[st]);
        bulk_g2s(dst + kOffScale8P + hs * kInt8ScaleBytes, scales, kInt8ScaleBytes, &x.bars[st]);
      }
    }
  };
  int issued = min(nv, kStages);
  for (int k = 0; k < issued; ++k)
    if (prologue_copy(x, k)) issue(k);
  // The bounded wait for copy k gave up: wait for the copies still in flight, write empty
  // states.
  auto give_up = [&](int k) {
    drain_copies(x, k, issued, k);
    for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
  };

  // ---- query fragments (B operand of QK^T, m16n8k32): lane column gid = (slot gid/4,
  // query gid%4); k-step ks: b0 = dims 32ks+4tig..+3, b1 = dims 32ks+16+4tig..+3, as bytes
  // of q / qstep = 256*hi + lo; a slot's fragments are zero outside its columns.
  uint32_t qh[2][4][2], ql[2][4][2];
  float qstep_own;
  {
    const int hs_b = gid / CPH, jb = gid % CPH;
    const bool live = jb < G && hs_b < nh;
    const uint16_t *qrow =
        q + (static_cast<size_t>(b) * H * G + (h0 + hs_b) * G + jb) * kHeadDim;
    float qv[4][2][4];
    float amax = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint2 v = live ? *reinterpret_cast<const uint2 *>(qrow + 32 * ks + 16 * hf + 4 * tig)
                             : make_uint2(0u, 0u);
        qv[ks][hf][0] = __uint_as_float(v.x << 16);
        qv[ks][hf][1] = __uint_as_float(v.x & 0xFFFF0000u);
        qv[ks][hf][2] = __uint_as_float(v.y << 16);
        qv[ks][hf][3] = __uint_as_float(v.y & 0xFFFF0000u);
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(qv[ks][hf][i]));
      }
    qstep_own = query_step(amax);
    const float inv = 1.0f / qstep_own;  // a power of two: exact
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t hb = 0u, lb = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int qi = __float2int_rn(qv[ks][hf][i] * inv);
          lb |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * i);
          hb |= (static_cast<uint32_t>(qi >> 8) & 0xFFu) << (8 * i);
        }
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          qh[hs][ks][hf] = hs == hs_b ? hb : 0u;
          ql[hs][ks][hf] = hs == hs_b ? lb : 0u;
        }
      }
  }
  float2 kq;  // qstep * log2(e)/sqrt(d) of the C-fragment columns (2tig, 2tig+1)
  kq.x = __shfl_sync(0xffffffffu, qstep_own, 4 * (2 * tig)) * kScaleLog2;
  kq.y = __shfl_sync(0xffffffffu, qstep_own, 4 * (2 * tig + 1)) * kScaleLog2;

  float m[2] = {kNegBig, kNegBig}, l[2] = {0.f, 0.f};
  float o[8][4];
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) o[cc][0] = o[cc][1] = o[cc][2] = o[cc][3] = 0.f;
  const int ld_off = ((lane >> 4) * 256) + ((lane >> 3) & 1) * 128 + (lane & 7) * 16;
  const int ring_base = L - R;  // ring slot s holds position ring_base + ((s - ring_base) mod R)
  const bool write_p0 = head_c_live && jc0 < G, write_p1 = head_c_live && jc0 + 1 < G;
  const bool col_live = (gid % CPH) < G && (gid / CPH) < nh;  // this lane's B column
  float lift = 0.f;
  if (MODE == kLifted) {  // the lift from the largest V scale of the first tile (copy 1)
    if (!peek_stage(x, 1 % kStages, err)) {
      drain_copies(x, 0, issued, 1);
      for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
      return kDone;
    }
    const uint16_t *v0 = reinterpret_cast<const uint16_t *>(
        x.stage0 + (1 % kStages) * kStageBytes + kOffScale8P + hs_c * kInt8ScaleBytes);
    uint32_t mx = page_max_scale(max(v0[gid], v0[gid + 8]));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));  // one lift for both head slots
    lift = lift_for_scale(mx);
  }

  for (int j = 0; j < nt; ++j) {
    // ---- K part: logits ----
    const int kk = 2 * j;
    if (!wait_stage(x, kk % kStages, err)) {
      give_up(kk);
      return kDone;
    }
    const uint8_t *spk = x.stage0 + (kk % kStages) * kStageBytes;
    const uint32_t sak = smem_u32(spk);
    int32_t ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        uint32_t kw[4];  // rows = positions, k = dims 32ks..32ks+31
        ldsm_x4(kw, sak + hs * kInt8CodeBytes + ks * 512 + ld_off);
        mma_s8s8(ah, kw[0], kw[1], kw[2], kw[3], qh[hs][ks][0], qh[hs][ks][1]);
        mma_s8u8(al, kw[0], kw[1], kw[2], kw[3], ql[hs][ks][0], ql[hs][ks][1]);
      }
    const uint16_t *ksc =
        reinterpret_cast<const uint16_t *>(spk + kOffScale8P + hs_c * kInt8ScaleBytes);
    const float sk[2] = {__half2float(__ushort_as_half(ksc[gid])),
                         __half2float(__ushort_as_half(ksc[gid + 8]))};
    __syncwarp();
    if (issued < nv) issue(issued++);  // the K stage is free again

    float s[2][2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int slot = gid + 8 * hf;
      bool valid;
      if (j < sink_tiles) {
        valid = j * kPage + slot < n_sink;
      } else {
        const int rs = (j - sink_tiles) * kPage + slot;
        int d = (rs - ring_base) % R;
        if (d < 0) d += R;
        valid = rs < R && ring_base + d >= S;
      }
      // exact integer dot products: |.| < 2^29
      const float d0 = static_cast<float>(ah[2 * hf] * 256 + al[2 * hf]);
      const float d1 = static_cast<float>(ah[2 * hf + 1] * 256 + al[2 * hf + 1]);
      s[hf][0] = valid ? d0 * sk[hf] * kq.x : -CUDART_INF_F;
      s[hf][1] = valid ? d1 * sk[hf] * kq.y : -CUDART_INF_F;
    }
    // ---- online softmax; the rescale is skipped while no running max moves ----
    float a[2];
    bool moved = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float t = fmaxf(s[0][e], s[1][e]);
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 4));
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 8));
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 16));
      const float mn = fmaxf(m[e], t - lift);  // running maximum kept as max - lift
      const bool mv = mn != m[e];
      a[e] = mv ? fast_exp2(m[e] - mn) : 1.0f;
      moved |= mv;
      m[e] = mn;
      s[0][e] = fast_exp2(s[0][e] - mn);
      s[1][e] = fast_exp2(s[1][e] - mn);
      l[e] = fmaf(l[e], a[e], s[0][e] + s[1][e]);
    }
    if (__any_sync(0xffffffffu, moved)) {
      const float2 a2 = make_float2(a[0], a[1]);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const float2 u = fmul2(make_float2(o[cc][0], o[cc][1]), a2);
        const float2 v = fmul2(make_float2(o[cc][2], o[cc][3]), a2);
        o[cc][0] = u.x; o[cc][1] = u.y; o[cc][2] = v.x; o[cc][3] = v.y;
      }
    }

    // ---- V part: P' = p * vscale (fp16), O^T += V^T P' per 16-dim strip and head ----
    const int kvc = 2 * j + 1;
    if (!wait_stage(x, kvc % kStages, err)) {
      give_up(kvc);
      return kDone;
    }
    const uint8_t *spv = x.stage0 + (kvc % kStages) * kStageBytes;
    const uint32_t sav = smem_u32(spv);
    const uint16_t *vsc =
        reinterpret_cast<const uint16_t *>(spv + kOffScale8P + hs_c * kInt8ScaleBytes);
    const float sv0 = __half2float(__ushort_as_half(vsc[gid]));
    const float sv1 = __half2float(__ushort_as_half(vsc[gid + 8]));
    if (write_p0) {
      x.ptile8[(2 * tig) * 16 + gid] = __half_as_ushort(__float2half_rn(s[0][0] * sv0));
      x.ptile8[(2 * tig) * 16 + gid + 8] = __half_as_ushort(__float2half_rn(s[1][0] * sv1));
    }
    if (write_p1) {
      x.ptile8[(2 * tig + 1) * 16 + gid] = __half_as_ushort(__float2half_rn(s[0][1] * sv0));
      x.ptile8[(2 * tig + 1) * 16 + gid + 8] = __half_as_ushort(__float2half_rn(s[1][1] * sv1));
    }
    __syncwarp();
    uint32_t b01 = 0u, b23 = 0u;  // column gid's P' (k = positions 2tig.., 2tig+8..)
    if (col_live) {
      b01 = *reinterpret_cast<const uint32_t *>(&x.ptile8[gid * 16 + 2 * tig]);
      b23 = *reinterpret_cast<const uint32_t *>(&x.ptile8[gid * 16 + 2 * tig + 8]);
    }
#pragma unroll
    for (int pr = 0; pr < 4; ++pr)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        uint32_t vw[4];
        ldsm_x4_t(vw, sav + hs * kInt8CodeBytes + pr * 512 + ld_off);
        const uint32_t c01 = gid / CPH == hs ? b01 : 0u, c23 = gid / CPH == hs ? b23 : 0u;
#pragma unroll
        for (int sp2 = 0; sp2 < 2; ++sp2) {
          const int cc = 2 * pr + sp2;
          const uint32_t ulo = vw[2 * sp2] ^ 0x80808080u, uhi = vw[2 * sp2 + 1] ^ 0x80808080u;
          mma_f16(o[cc], s8_pair<0x4240>(ulo), s8_pair<0x4341>(ulo), s8_pair<0x4240>(uhi),
                  s8_pair<0x4341>(uhi), c01, c23);
        }
      }
    __syncwarp();
    if (issued < nv) issue(issued++);  // the V stage is free again
  }

  // ---- finish: reduce the denominators over the 8 position lanes, write the partials ----
  if (MODE == kLifted) {
    const float probe[2] = {o[0][0], o[0][1]};
    if (any_not_finite(probe)) return kOverflow;
  }
  if (MODE == kDecide) {  // the last tile's V scales (still staged) ask for the lift?
    const uint16_t *vl = reinterpret_cast<const uint16_t *>(
        x.stage0 + ((nv - 1) % kStages) * kStageBytes + kOffScale8P + hs_c * kInt8ScaleBytes);
    uint32_t mx = page_max_scale(max(vl[gid], vl[gid + 8]));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (lift_for_scale(mx) >= kLiftMin) return kWantLift;
  }
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], off);
  if (head_c_live) {
    float *rec = record_of(w, H, G, b, h0 + hs_c, r);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = jc0 + e;
      if (j < G) {
        float *rr = rec + j * kRecordFloats;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)  // rows: dim 16cc+2gid (c0/c1) and +1 (c2/c3)
          st_rec(reinterpret_cast<float2 *>(rr + 16 * cc + 2 * gid),
                 make_float2(o[cc][e], o[cc][2 + e]));
        if (gid == 0) {
          st_rec(rr + kHeadDim, m[e] * kLn2);
          st_rec(rr + kHeadDim + 1, l[e]);
        }
      }
    }
  }
  return kDone;
}

// ---------------------------- INT4 chunk --------------------------------
// Token order of the QK^T M-tile rows: rows 0-7 are tokens 0-7, rows 8-11 tokens 12-15,
// rows 12-15 tokens 8-11. With it a thread's two rows (gid, gid+8) are the tokens whose
// P' values it packs into one 32-bit word, the transposed V loads read those pairs, and
// neither the K nor the V ldmatrix phases hit a shared-memory bank twice.
__device__ __forceinline__ int row_token_hi(int r) { return 8 + ((r + 4) & 7); }

// One chunk of INT4 pages for HPW kv heads (h0 .. h0+nh-1, nh <= HPW). MMA column
// col (0..7) belongs to head slot col / CPH and query j = col % CPH of that head.
// Returns kDone, kWantLift (MODE kDecide) or kOverflow (MODE kLifted).
template <int HPW, int MODE>
__device__ __forceinline__ int process_int4(WarpCtx &x, const CacheView &c, const Workspace &w,
                             const uint16_t *__restrict__ q, int b, int h0, int nh, int r,
                             int chunk, const Regions &rg, int32_t *err) {
  constexpr int CPH = 8 / HPW;  // MMA columns per kv head slot
  const int G = c.gqa, H = c.num_kv_heads;
  const int lane = x.lane, gid = x.gid, tig = x.tig;
  const int p0 = rg.first_page + chunk * w.chunk_pages;
  const int last = (rg.int4_hi - 1) / kPage;
  const int np = min(w.chunk_pages, last - p0 + 1);
  if (np < 1 || chunk < 0) {  // only with a reused work list whose lengths have changed
    if (lane == 0) set_err(err, KV4_DEVERR_WORKSPACE);
    for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
    return kDone;
  }
  // this lane's C-fragment columns 2tig, 2tig+1: head slot and query index
  const int hs_c = (2 * tig) / CPH;
  const int jc0 = (2 * tig) % CPH;
  const bool head_c_live = hs_c < nh;

  // page ids of the chunk: page k in lane k (k < 32) or in the second register of lane
  // k - 32 (chunks of up to 64 pages)
  const int *pt = c.page_table + static_cast<size_t>(b) * c.max_pages + p0;
  int pid = 0, pid2 = 0;
  if (lane < np) pid = pt[lane];
  if (lane + 32 < np) pid2 = pt[lane + 32];
  const bool bad = (lane < np && (pid < 0 || pid >= c.num_pages)) ||
                   (lane + 32 < np && (pid2 < 0 || pid2 >= c.num_pages));
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) set_err(err, KV4_DEVERR_PAGE_ID);
    for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
    return kDone;
  }

  // stage layout: K codes [HPW][1024] | V codes [HPW][1024] | K params [HPW][256] | V params
  constexpr int kOffVc = HPW * kInt4CodeBytes;
  constexpr int kOffKp = 2 * HPW * kInt4CodeBytes;
  constexpr int kOffVp = kOffKp + HPW * kInt4ParamBytes;
  auto issue = [&](int k) {
    const int pk = __shfl_sync(0xffffffffu, k < 32 ? pid : pid2, k & 31);
    const int st = k % kStages;
    if (lane == 0) {
      uint8_t *dst = x.stage0 + st * kStageBytes;
      const size_t blk = static_cast<size_t>(pk) * H + h0;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&x.bars[st], HPW * (2 * kInt4CodeBytes + 2 * kInt4ParamBytes));
      if (nh == HPW) {  // the kv heads of one page are adjacent: one copy per array
        bulk_g2s(dst, c.k_codes + blk * kInt4CodeBytes, HPW * kInt4CodeBytes, &x.bars[st]);
        bulk_g2s(dst + kOffVc, c.v_codes + blk * kInt4CodeBytes, HPW * kInt4CodeBytes, &x.bars[st]);
        bulk_g2s(dst + kOffKp, reinterpret_cast<const uint8_t *>(c.k_params) + blk * kInt4ParamBytes,
                 HPW * kInt4ParamBytes, &x.bars[st]);
        bulk_g2s(dst + kOffVp, reinterpret_cast<const uint8_t *>(c.v_params) + blk * kInt4ParamBytes,
                 HPW * kInt4ParamBytes, &x.bars[st]);
      } else {  // fewer heads than slots: fill the spare slots with a copy of head h0
        for (int hs = 0; hs < HPW; ++hs) {
          bulk_g2s(dst + hs * kInt4CodeBytes, c.k_codes + blk * kInt4CodeBytes, kInt4CodeBytes,
                   &x.bars[st]);
          bulk_g2s(dst + kOffVc + hs * kInt4CodeBytes, c.v_codes + blk * kInt4CodeBytes,
                   kInt4CodeBytes, &x.bars[st]);
          bulk_g2s(dst + kOffKp + hs * kInt4ParamBytes,
                   reinterpret_cast<const uint8_t *>(c.k_params) + blk * kInt4ParamBytes,
                   kInt4ParamBytes, &x.bars[st]);
          bulk_g2s(dst + kOffVp + hs * kInt4ParamBytes,
                   reinterpret_cast<const uint8_t *>(c.v_params) + blk * kInt4ParamBytes,
                   kInt4ParamBytes, &x.bars[st]);
        }
      }
    }
  };
  const int npre = min(np, kStages);
  for (int k = 0; k < npre; ++k)
    if (prologue_copy(x, k)) issue(k);

  // ---- query fragments (B operand of QK^T). Lane column gid = (slot gid/CPH, query
  // gid%CPH); slot hs's fragments are zero unless the column is in slot hs.
  // q = qstep * (256*hi + lo) with qstep = 2^e chosen per query so that
  // |256*hi + lo| < 2^14; b0 holds dims 8tig+{0,2,4,6} and b1 dims 8tig+{1,3,5,7} of a
  // group (the low and high nibbles of the lane's K word), as bytes.
  uint32_t qh[HPW][4][2], ql[HPW][4][2];
  float qsum_own[4];
  float qstep_own;
  {
    const int hs_b = gid / CPH, jb = gid % CPH;
    const bool live = jb < G && hs_b < nh;
    const uint16_t *qrow =
        q + (static_cast<size_t>(b) * H * G + (h0 + hs_b) * G + jb) * kHeadDim;
    float qv[4][8];
    float amax = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint4 v = load_q8(qrow, 32 * g + 8 * tig, live);  // bf16 dims +0..+7
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        qv[g][2 * i] = __uint_as_float(w4[i] << 16);
        qv[g][2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
        sum += qv[g][2 * i] + qv[g][2 * i + 1];
        amax = fmaxf(amax, fmaxf(fabsf(qv[g][2 * i]), fabsf(qv[g][2 * i + 1])));
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      qsum_own[g] = sum;  // sum over the group's 32 dims for column gid
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int ex = 0;
    if (amax > 0.f) {
      frexpf(amax, &ex);  // amax < 2^ex
      ex -= 14;
    }
    const float inv = ldexpf(1.0f, -ex);
    qstep_own = ldexpf(1.0f, ex);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t hb[2] = {0u, 0u}, lb[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int qi = __float2int_rn(qv[g][i] * inv);  // exact scaling by 2^-ex
        const int sel = i & 1, byte = i >> 1;           // dim 8tig+i -> b[i&1], byte i>>1
        lb[sel] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * byte);
        hb[sel] |= (static_cast<uint32_t>(qi >> 8) & 0xFFu) << (8 * byte);
      }
#pragma unroll
      for (int hs = 0; hs < HPW; ++hs) {
        const bool mine = hs == hs_b;
        qh[hs][g][0] = mine ? hb[0] : 0u;
        qh[hs][g][1] = mine ? hb[1] : 0u;
        ql[hs][g][0] = mine ? lb[0] : 0u;
        ql[hs][g][1] = mine ? lb[1] : 0u;
      }
    }
  }
  float2 kq;  // qstep * log2(e)/sqrt(d) of the C-fragment columns (2tig, 2tig+1)
  kq.x = __shfl_sync(0xffffffffu, qstep_own, 4 * (2 * tig)) * kScaleLog2;
  kq.y = __shfl_sync(0xffffffffu, qstep_own, 4 * (2 * tig + 1)) * kScaleLog2;
  float2 qs[4];  // column (2tig, 2tig+1) sums, matching the C-fragment columns
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    qs[g].x = __shfl_sync(0xffffffffu, qsum_own[g], 4 * (2 * tig));
    qs[g].y = __shfl_sync(0xffffffffu, qsum_own[g], 4 * (2 * tig + 1));
  }

  float m[2] = {kNegBig, kNegBig}, l[2] = {0.f, 0.f};
  float o[4][2][4];  // [group][m-tile]: rows dim 32g+4gid+2mt (c0,c1) and +1 (c2,c3)
  float mt[4][2];    // sum p * vmin per group and column
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    mt[g][0] = mt[g][1] = 0.f;
#pragma unroll
    for (int t = 0; t < 2; ++t) o[g][t][0] = o[g][t][1] = o[g][t][2] = o[g][t][3] = 0.f;
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
  const int kp_off = kOffKp + hs_c * kInt4ParamBytes;
  const int vp_off = kOffVp + hs_c * kInt4ParamBytes;
  const bool write_p0 = head_c_live && jc0 < G, write_p1 = head_c_live && jc0 + 1 < G;
  uint32_t *pt_mine = x.ptile + (hs_c * 4 * 8 + 2 * tig) * kPWordsPerCol + gid;
  // the largest V scale of the page staged at `st` over the warp (both head slots)
  auto page_scale = [&](int st) {
    const uint8_t *sp = x.stage0 + st * kStageBytes;
    const uint4 v0 = *reinterpret_cast<const uint4 *>(sp + vp_off + t0 * 16);
    const uint4 v1 = *reinterpret_cast<const uint4 *>(sp + vp_off + t1 * 16);
    uint32_t mx = page_max_scale(__vmaxu2(__vmaxu2(__vmaxu2(v0.x, v0.y), __vmaxu2(v0.z, v0.w)),
                                          __vmaxu2(__vmaxu2(v1.x, v1.y), __vmaxu2(v1.z, v1.w))));
    if (HPW == 2) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    return mx;
  };
  float lift = 0.f;
  if (MODE == kLifted) {  // the lift from the largest V scale of the first page
    if (!peek_stage(x, 0, err)) {
      drain_copies(x, 0, npre, 0);
      for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
      return kDone;
    }
    lift = lift_for_scale(page_scale(0));
  }

  for (int k = 0; k < np; ++k) {
    const int st = k % kStages;
    if (!wait_stage(x, st, err)) {
      drain_copies(x, k, min(np, k + kStages), k);
      for (int hs = 0; hs < nh; ++hs) write_empty(record_of(w, H, G, b, h0 + hs, r), G, lane);
      return kDone;
    }
    uint8_t *sp = x.stage0 + st * kStageBytes;
    const uint32_t sa = smem_u32(sp);

    // ---- logits: s = sum_g scale_g * (q . c)_g + min_g * sum_g(q), log2 units ----
    const uint4 kp[2] = {*reinterpret_cast<const uint4 *>(sp + kp_off + t0 * 16),
                         *reinterpret_cast<const uint4 *>(sp + kp_off + t1 * 16)};
    // sc*: sum_g scale_g * (q . c)_g in units of the query step;
    // mn*: sum_g min_g * sum_g(q)
    float2 sc0 = make_float2(0.f, 0.f), sc1 = make_float2(0.f, 0.f);
    float2 mn0 = make_float2(0.f, 0.f), mn1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {  // group pairs (2gp, 2gp+1): one ldmatrix.x4 per head
      uint32_t kw[HPW][4];
#pragma unroll
      for (int hs = 0; hs < HPW; ++hs) ldsm_x4(kw[hs], sa + hs * kInt4CodeBytes + gp * 512 + ld_k);
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = 2 * gp + gg;
        int32_t ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
        for (int hs = 0; hs < HPW; ++hs) {
          const uint32_t wlo = kw[hs][2 * gg], whi = kw[hs][2 * gg + 1];
          const uint32_t a0 = wlo & 0x0F0F0F0Fu, a1 = whi & 0x0F0F0F0Fu;
          const uint32_t a2 = (wlo >> 4) & 0x0F0F0F0Fu, a3 = (whi >> 4) & 0x0F0F0F0Fu;
          mma_u8s8(ah, a0, a1, a2, a3, qh[hs][g][0], qh[hs][g][1]);
          mma_u8u8(al, a0, a1, a2, a3, ql[hs][g][0], ql[hs][g][1]);
        }
        float acc[4];  // exact integer dot products, |.| < 2^24
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = static_cast<float>(ah[i] * 256 + al[i]);
        const uint32_t w0 = g == 0 ? kp[0].x : g == 1 ? kp[0].y : g == 2 ? kp[0].z : kp[0].w;
        const uint32_t w1 = g == 0 ? kp[1].x : g == 1 ? kp[1].y : g == 2 ? kp[1].z : kp[1].w;
        const float2 f0 = h2_to_f2(w0), f1 = h2_to_f2(w1);
        sc0 = ffma2(make_float2(f0.x, f0.x), make_float2(acc[0], acc[1]), sc0);
        mn0 = ffma2(make_float2(f0.y, f0.y), qs[g], mn0);
        sc1 = ffma2(make_float2(f1.x, f1.x), make_float2(acc[2], acc[3]), sc1);
        mn1 = ffma2(make_float2(f1.y, f1.y), qs[g], mn1);
      }
    }
    const float2 k512 = kq;  // the integer dot products are in units of qstep
    const float2 k1 = make_float2(kScaleLog2, kScaleLog2);
    const float2 sl0 = ffma2(sc0, k512, fmul2(mn0, k1));
    const float2 sl1 = ffma2(sc1, k512, fmul2(mn1, k1));
    float s[2][2];
    s[0][0] = sl0.x;
    s[0][1] = sl0.y;
    s[1][0] = sl1.x;
    s[1][1] = sl1.y;
    const int tok0 = (p0 + k) * kPage;
    if (tok0 < tok_lo || tok0 + kPage > tok_hi) {  // ragged first/last page of the range
      if (!(tok0 + t0 >= tok_lo && tok0 + t0 < tok_hi)) s[0][0] = s[0][1] = -CUDART_INF_F;
      if (!(tok0 + t1 >= tok_lo && tok0 + t1 < tok_hi)) s[1][0] = s[1][1] = -CUDART_INF_F;
    }
    // ---- online softmax; the rescale is skipped while no running max moves ----
    float a[2];
    bool moved = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float t = fmaxf(s[0][e], s[1][e]);
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 4));
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 8));
      t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, 16));
      const float mn = fmaxf(m[e], t - lift);  // running maximum kept as max - lift
      const bool mv = mn != m[e];
      a[e] = mv ? fast_exp2(m[e] - mn) : 1.0f;
      moved |= mv;
      m[e] = mn;
      s[0][e] = fast_exp2(s[0][e] - mn);
      s[1][e] = fast_exp2(s[1][e] - mn);
      l[e] = fmaf(l[e], a[e], s[0][e] + s[1][e]);
    }
    if (__any_sync(0xffffffffu, moved)) {
      const float2 a2 = make_float2(a[0], a[1]);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        mt[g][0] *= a[0];
        mt[g][1] *= a[1];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const float2 u = fmul2(make_float2(o[g][t][0], o[g][t][1]), a2);
          const float2 v = fmul2(make_float2(o[g][t][2], o[g][t][3]), a2);
          o[g][t][0] = u.x; o[g][t][1] = u.y; o[g][t][2] = v.x; o[g][t][3] = v.y;
        }
      }
    }
    // ---- P'_g = p * vscale_g as fp16 token pairs; sum p * vmin_g on the side ----
    const uint4 vp[2] = {*reinterpret_cast<const uint4 *>(sp + vp_off + t0 * 16),
                         *reinterpret_cast<const uint4 *>(sp + vp_off + t1 * 16)};
    const float2 pe0 = make_float2(s[0][0], s[1][0]), pe1 = make_float2(s[0][1], s[1][1]);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t w0 = g == 0 ? vp[0].x : g == 1 ? vp[0].y : g == 2 ? vp[0].z : vp[0].w;
      const uint32_t w1 = g == 0 ? vp[1].x : g == 1 ? vp[1].y : g == 2 ? vp[1].z : vp[1].w;
      const float2 f0 = h2_to_f2(w0), f1 = h2_to_f2(w1);
      const float2 sv = make_float2(f0.x, f1.x);
      const float2 q0 = fmul2(pe0, sv), q1 = fmul2(pe1, sv);
      if (write_p0) pt_mine[(g * 8) * kPWordsPerCol] = pack_h2(q0.x, q0.y);
      if (write_p1) pt_mine[(g * 8 + 1) * kPWordsPerCol] = pack_h2(q1.x, q1.y);
      mt[g][0] = fmaf(pe0.x, f0.y, fmaf(pe0.y, f1.y, mt[g][0]));
      mt[g][1] = fmaf(pe1.x, f0.y, fmaf(pe1.y, f1.y, mt[g][1]));
    }
    __syncwarp();
    // ---- O^T += V^T P' per group and head slot: A = V codes, B = P'_g of that slot ----
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {
      uint32_t vw[HPW][4];
#pragma unroll
      for (int hs = 0; hs < HPW; ++hs)
        ldsm_x4_t(vw[hs], sa + kOffVc + hs * kInt4CodeBytes + gp * 512 + ld_v);
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = 2 * gp + gg;
#pragma unroll
        for (int hs = 0; hs < HPW; ++hs) {
          uint32_t vl[4], vh[4];
          nib_pairs_v_sub(vw[hs][2 * gg], vl);
          nib_pairs_v_sub(vw[hs][2 * gg + 1], vh);
          const uint32_t *pb = x.ptile + ((hs * 4 + g) * 8 + gid) * kPWordsPerCol + tig;
          const uint32_t b01 = pb[0], b23 = pb[4];
          mma_f16(o[g][0], vl[0], vl[1], vh[0], vh[1], b01, b23);
          mma_f16(o[g][1], vl[2], vl[3], vh[2], vh[3], b01, b23);
        }
      }
    }
    __syncwarp();
    if (k + kStages < np) issue(k + kStages);
  }

  // ---- finish: reduce per-thread sums over the 8 token lanes, write the partial ----
  if (MODE == kLifted) {
    const float probe[8] = {o[0][0][0], o[0][0][1], o[1][0][0], o[1][0][1],
                            o[2][0][0], o[2][0][1], o[3][0][0], o[3][0][1]};
    if (any_not_finite(probe)) return kOverflow;
  }
  // the last page's V scales (still staged) ask for the lift?
  if (MODE == kDecide && lift_for_scale(page_scale((np - 1) % kStages)) >= kLiftMin)
    return kWantLift;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], off);
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int off = 4; off < 32; off <<= 1)
        mt[g][e] += __shfl_xor_sync(0xffffffffu, mt[g][e], off);
  }
  if (head_c_live) {
    float *rec = record_of(w, H, G, b, h0 + hs_c, r);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = jc0 + e;
      if (j < G) {
        float *rr = rec + j * kRecordFloats;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          // rows gid (dims +0, +2) and gid+8 (dims +1, +3) carry their code scale
          const float4 v = make_float4(fmaf(o[g][0][e], kUnscaleV, mt[g][e]),
                                       fmaf(o[g][0][2 + e], kUnscaleV1, mt[g][e]),
                                       fmaf(o[g][1][e], kUnscaleV, mt[g][e]),
                                       fmaf(o[g][1][2 + e], kUnscaleV1, mt[g][e]));
          st_rec(reinterpret_cast<float4 *>(rr + 32 * g + 4 * gid), v);
        }
        if (gid == 0) {
          st_rec(rr + kHeadDim, m[e] * kLn2);
          st_rec(rr + kHeadDim + 1, l[e]);
        }
      }
    }
  }
  return kDone;
}

// ---------------------------------------------------------------------------
// shared-prefix read
// ---------------------------------------------------------------------------
// One entry = one chunk of a group's shared INT4 pages, one kv head, up to
// kPrefixCols / G consecutive member sequences. Column c of the 16 query columns (MMA N
// tiles c / 8) is query c % G of member c / G. Every page is copied into shared memory
// once and its K and V codes are unpacked once for all members; the arithmetic per column
// is that of process_int4 (integer QK^T on the fixed-point query, online softmax,
// P' = p * vscale in fp16 against the V codes as fp16 subnormals, sum p * vmin in fp32).
// Member m's tokens outside its INT4 range [S, L_m - R) are masked, so a member whose
// recent window starts inside the shared pages reads those positions from its ring only.
// The entries run in prefix_kernel, whose warps have the attention kernel's shared-memory
// layout: a ring of kStages one-head page blocks and the per-lane query operands in the
// stage area, the P' tile of both N tiles in the INT4 tile. (A separate kernel rather than
// a class of attn_kernel: compiled into one kernel, the two paths share one register
// allocation, and the INT4 path lost 8-10 % to it.)
constexpr int kPfxOffVc = kInt4CodeBytes;
constexpr int kPfxOffKp = 2 * kInt4CodeBytes;
constexpr int kPfxOffVp = 2 * kInt4CodeBytes + kInt4ParamBytes;
constexpr int kPfxStageBytes = 2 * kInt4CodeBytes + 2 * kInt4ParamBytes;  // 2560: one kv head
// per-lane query operands: [N tile][group][lane] uint4 (hi b0, hi b1, lo b0, lo b1) and
// float2 group sums of the lane's C-fragment columns
constexpr int kPfxOffQ = kStages * kPfxStageBytes;
constexpr int kPfxOffQs = kPfxOffQ + 2 * 4 * 32 * 16;
static_assert(kPfxOffQs + 2 * 4 * 32 * 8 <= kStages * kStageBytes,
              "the shared-prefix ring and query operands fit the warp's stage area");
static_assert(2 * 4 * 8 * kPWordsPerCol * 4 == kPtileBytes, "two N tiles of P'");

// Prompt chunk ci of kv head h for the nmem group members b0 .. b0+nmem-1. Returns true
// when the lift chosen on the first page overflowed a later weight: the entry is then to
// be redone with LIFT = false (nothing was written).
template <bool LIFT>
__device__ __forceinline__ bool process_prefix(WarpCtx &x, const CacheView &c, const Workspace &w,
                               const uint16_t *__restrict__ q, int b0, int ci, int h, int nmem,
                               int32_t *err) {
  const int G = c.gqa, H = c.num_kv_heads;
  const int S = c.num_sinks, R = c.num_recent;
  const int lane = x.lane, gid = x.gid, tig = x.tig;
  const int p0 = S / kPage + ci * w.chunk_pages;
  const int np = min(w.chunk_pages, w.prefix_end[b0] - p0);
  uint4 *qop = reinterpret_cast<uint4 *>(x.stage0 + kPfxOffQ);
  float2 *qsum_t = reinterpret_cast<float2 *>(x.stage0 + kPfxOffQs);

  // this thread's C-fragment columns (N tile t, 2tig + e): the end of the member's INT4
  // range (0 for a column without a member)
  int hi[2][2];
  int hi_min = 0x7fffffff;
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int mi = (8 * t + 2 * tig + e) / G;
      hi[t][e] = mi < nmem ? c.seq_lens[b0 + mi] - R : 0;
    }
  for (int mi = 0; mi < nmem; ++mi) hi_min = min(hi_min, c.seq_lens[b0 + mi] - R);

  auto write_empty_all = [&]() {
    for (int mi = 0; mi < nmem; ++mi) {
      const int L = c.seq_lens[b0 + mi];
      const int r = regions_of(L, S, R, w.chunk_pages).has_prot + ci;
      write_empty(record_of(w, H, G, b0 + mi, h, r), G, lane);
    }
  };
  if (np <= 0 || p0 + np > c.max_pages) {  // a reused work list that is not this batch's
    if (lane == 0) set_err(err, KV4_DEVERR_WORKSPACE);
    write_empty_all();
    return false;
  }
  const int *pt = c.page_table + static_cast<size_t>(b0) * c.max_pages + p0;
  int pid = 0, pid2 = 0;
  if (lane < np) pid = pt[lane];
  if (lane + 32 < np) pid2 = pt[lane + 32];
  const bool bad = (lane < np && (pid < 0 || pid >= c.num_pages)) ||
                   (lane + 32 < np && (pid2 < 0 || pid2 >= c.num_pages));
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) set_err(err, KV4_DEVERR_PAGE_ID);
    write_empty_all();
    return false;
  }

  auto issue = [&](int k) {
    const int pk = __shfl_sync(0xffffffffu, k < 32 ? pid : pid2, k & 31);
    const int st = k % kStages;
    if (lane == 0) {
      uint8_t *dst = x.stage0 + st * kPfxStageBytes;
      const size_t blk = static_cast<size_t>(pk) * H + h;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&x.bars[st], kPfxStageBytes);
      bulk_g2s(dst, c.k_codes + blk * kInt4CodeBytes, kInt4CodeBytes, &x.bars[st]);
      bulk_g2s(dst + kPfxOffVc, c.v_codes + blk * kInt4CodeBytes, kInt4CodeBytes, &x.bars[st]);
      bulk_g2s(dst + kPfxOffKp, reinterpret_cast<const uint8_t *>(c.k_params) + blk * kInt4ParamBytes,
               kInt4ParamBytes, &x.bars[st]);
      bulk_g2s(dst + kPfxOffVp, reinterpret_cast<const uint8_t *>(c.v_params) + blk * kInt4ParamBytes,
               kInt4ParamBytes, &x.bars[st]);
    }
  };
  const int npre = min(np, kStages);
  for (int k = 0; k < npre; ++k)
    if (prologue_copy(x, k)) issue(k);

  // ---- query fragments (B operand of QK^T) of column 8t + gid of N tile t, as in
  // process_int4: q = qstep * (256*hi + lo), b0 = dims 8tig+{0,2,4,6}, b1 = 8tig+{1,3,5,7}
  float2 kq[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int col = 8 * t + gid, mb = col / G, jb = col - mb * G;
    const bool live = mb < nmem;
    const uint16_t *qrow = q + (static_cast<size_t>(b0 + (live ? mb : 0)) * H * G + h * G + jb) * kHeadDim;
    float qv[4][8];
    float qsum[4];
    float amax = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint4 v = load_q8(qrow, 32 * g + 8 * tig, live);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        qv[g][2 * i] = __uint_as_float(w4[i] << 16);
        qv[g][2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
        sum += qv[g][2 * i] + qv[g][2 * i + 1];
        amax = fmaxf(amax, fmaxf(fabsf(qv[g][2 * i]), fabsf(qv[g][2 * i + 1])));
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      qsum[g] = sum;
    }
    const float qstep = query_step(amax);
    const float inv = 1.0f / qstep;  // a power of two: exact
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t hb[2] = {0u, 0u}, lb[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int qi = __float2int_rn(qv[g][i] * inv);
        const int sel = i & 1, byte = i >> 1;
        lb[sel] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * byte);
        hb[sel] |= (static_cast<uint32_t>(qi >> 8) & 0xFFu) << (8 * byte);
      }
      qop[(t * 4 + g) * 32 + lane] = make_uint4(hb[0], hb[1], lb[0], lb[1]);
      qsum_t[(t * 4 + g) * 32 + lane] = make_float2(__shfl_sync(0xffffffffu, qsum[g], 4 * (2 * tig)),
                                                    __shfl_sync(0xffffffffu, qsum[g], 4 * (2 * tig + 1)));
    }
    kq[t].x = __shfl_sync(0xffffffffu, qstep, 4 * (2 * tig)) * kScaleLog2;
    kq[t].y = __shfl_sync(0xffffffffu, qstep, 4 * (2 * tig + 1)) * kScaleLog2;
  }

  float m[2][2], l[2][2];
  float o[4][2][2][4];  // [group][m-tile][N tile]
  float mt[4][2][2];    // sum p * vmin per group, N tile and column
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    m[t][0] = m[t][1] = kNegBig;
    l[t][0] = l[t][1] = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      mt[g][t][0] = mt[g][t][1] = 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u) o[g][u][t][0] = o[g][u][t][1] = o[g][u][t][2] = o[g][u][t][3] = 0.f;
    }
  }

  const int r8 = lane & 7;
  const int mhalf = (lane >> 3) & 1;
  const int strip_off = (lane >> 4) * 256;
  const int ld_k = strip_off + (mhalf ? row_token_hi(r8) : r8) * 16;
  const int ld_v = strip_off + (mhalf ? ((r8 & 1) ? 8 + (r8 >> 1) : 4 + (r8 >> 1))
                                      : ((r8 & 1) ? 12 + (r8 >> 1) : (r8 >> 1))) * 16;
  const int t0 = gid, t1 = row_token_hi(gid);
  uint32_t *pt_mine = x.ptile + (2 * tig) * kPWordsPerCol + gid;
  float lift = 0.f;
  if (LIFT) {  // the lift from the largest V scale of the first page
    if (!peek_stage(x, 0, err)) {
      drain_copies(x, 0, npre, 0);
      write_empty_all();
      return false;
    }
    const uint4 v0 = *reinterpret_cast<const uint4 *>(x.stage0 + kPfxOffVp + t0 * 16);
    const uint4 v1 = *reinterpret_cast<const uint4 *>(x.stage0 + kPfxOffVp + t1 * 16);
    lift = lift_for_scale(page_max_scale(__vmaxu2(__vmaxu2(__vmaxu2(v0.x, v0.y), __vmaxu2(v0.z, v0.w)),
                                                  __vmaxu2(__vmaxu2(v1.x, v1.y), __vmaxu2(v1.z, v1.w)))));
  }

  for (int k = 0; k < np; ++k) {
    const int st = k % kStages;
    if (!wait_stage(x, st, err)) {
      drain_copies(x, k, min(np, k + kStages), k);
      write_empty_all();
      return false;
    }
    const uint8_t *sp = x.stage0 + st * kPfxStageBytes;
    const uint32_t sa = smem_u32(sp);

    // ---- logits of both N tiles ----
    const uint4 kp[2] = {*reinterpret_cast<const uint4 *>(sp + kPfxOffKp + t0 * 16),
                         *reinterpret_cast<const uint4 *>(sp + kPfxOffKp + t1 * 16)};
    float2 sc0[2], sc1[2], mn0[2], mn1[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) sc0[t] = sc1[t] = mn0[t] = mn1[t] = make_float2(0.f, 0.f);
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {
      uint32_t kw[4];
      ldsm_x4(kw, sa + gp * 512 + ld_k);
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = 2 * gp + gg;
        const uint32_t wlo = kw[2 * gg], whi = kw[2 * gg + 1];
        const uint32_t a0 = wlo & 0x0F0F0F0Fu, a1 = whi & 0x0F0F0F0Fu;
        const uint32_t a2 = (wlo >> 4) & 0x0F0F0F0Fu, a3 = (whi >> 4) & 0x0F0F0F0Fu;
        const uint32_t w0 = g == 0 ? kp[0].x : g == 1 ? kp[0].y : g == 2 ? kp[0].z : kp[0].w;
        const uint32_t w1 = g == 0 ? kp[1].x : g == 1 ? kp[1].y : g == 2 ? kp[1].z : kp[1].w;
        const float2 f0 = h2_to_f2(w0), f1 = h2_to_f2(w1);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint4 qo = qop[(t * 4 + g) * 32 + lane];
          const float2 qs = qsum_t[(t * 4 + g) * 32 + lane];
          int32_t ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
          mma_u8s8(ah, a0, a1, a2, a3, qo.x, qo.y);
          mma_u8u8(al, a0, a1, a2, a3, qo.z, qo.w);
          float acc[4];  // exact integer dot products, |.| < 2^24
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = static_cast<float>(ah[i] * 256 + al[i]);
          sc0[t] = ffma2(make_float2(f0.x, f0.x), make_float2(acc[0], acc[1]), sc0[t]);
          mn0[t] = ffma2(make_float2(f0.y, f0.y), qs, mn0[t]);
          sc1[t] = ffma2(make_float2(f1.x, f1.x), make_float2(acc[2], acc[3]), sc1[t]);
          mn1[t] = ffma2(make_float2(f1.y, f1.y), qs, mn1[t]);
        }
      }
    }
    const float2 k1 = make_float2(kScaleLog2, kScaleLog2);
    float s[2][2][2];  // [N tile][token t0 / t1][column e]
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const float2 sl0 = ffma2(sc0[t], kq[t], fmul2(mn0[t], k1));
      const float2 sl1 = ffma2(sc1[t], kq[t], fmul2(mn1[t], k1));
      s[t][0][0] = sl0.x;
      s[t][0][1] = sl0.y;
      s[t][1][0] = sl1.x;
      s[t][1][1] = sl1.y;
    }
    const int tok0 = (p0 + k) * kPage;
    if (tok0 < S || tok0 + kPage > hi_min) {  // some member does not read all 16 tokens
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          if (!(tok0 + t0 >= S && tok0 + t0 < hi[t][e])) s[t][0][e] = -CUDART_INF_F;
          if (!(tok0 + t1 >= S && tok0 + t1 < hi[t][e])) s[t][1][e] = -CUDART_INF_F;
        }
    }
    // ---- online softmax per column; the rescale is skipped while no running max moves ----
    float a[2][2];
    bool moved = false;
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = fmaxf(s[t][0][e], s[t][1][e]);
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        const float mn = fmaxf(m[t][e], v - lift);  // running maximum kept as max - lift
        const bool mv = mn != m[t][e];
        a[t][e] = mv ? fast_exp2(m[t][e] - mn) : 1.0f;
        moved |= mv;
        m[t][e] = mn;
        s[t][0][e] = fast_exp2(s[t][0][e] - mn);
        s[t][1][e] = fast_exp2(s[t][1][e] - mn);
        l[t][e] = fmaf(l[t][e], a[t][e], s[t][0][e] + s[t][1][e]);
      }
    if (__any_sync(0xffffffffu, moved)) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float2 a2 = make_float2(a[t][0], a[t][1]);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          mt[g][t][0] *= a[t][0];
          mt[g][t][1] *= a[t][1];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float2 x0 = fmul2(make_float2(o[g][u][t][0], o[g][u][t][1]), a2);
            const float2 x1 = fmul2(make_float2(o[g][u][t][2], o[g][u][t][3]), a2);
            o[g][u][t][0] = x0.x; o[g][u][t][1] = x0.y; o[g][u][t][2] = x1.x; o[g][u][t][3] = x1.y;
          }
        }
      }
    }
    // ---- P'_g = p * vscale_g as fp16 token pairs per column; sum p * vmin_g on the side ----
    const uint4 vp[2] = {*reinterpret_cast<const uint4 *>(sp + kPfxOffVp + t0 * 16),
                         *reinterpret_cast<const uint4 *>(sp + kPfxOffVp + t1 * 16)};
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t w0 = g == 0 ? vp[0].x : g == 1 ? vp[0].y : g == 2 ? vp[0].z : vp[0].w;
      const uint32_t w1 = g == 0 ? vp[1].x : g == 1 ? vp[1].y : g == 2 ? vp[1].z : vp[1].w;
      const float2 f0 = h2_to_f2(w0), f1 = h2_to_f2(w1);
      const float2 sv = make_float2(f0.x, f1.x);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const float2 pe0 = make_float2(s[t][0][0], s[t][1][0]), pe1 = make_float2(s[t][0][1], s[t][1][1]);
        const float2 q0 = fmul2(pe0, sv), q1 = fmul2(pe1, sv);
        pt_mine[((t * 4 + g) * 8) * kPWordsPerCol] = pack_h2(q0.x, q0.y);
        pt_mine[((t * 4 + g) * 8 + 1) * kPWordsPerCol] = pack_h2(q1.x, q1.y);
        mt[g][t][0] = fmaf(pe0.x, f0.y, fmaf(pe0.y, f1.y, mt[g][t][0]));
        mt[g][t][1] = fmaf(pe1.x, f0.y, fmaf(pe1.y, f1.y, mt[g][t][1]));
      }
    }
    __syncwarp();
    // ---- O^T += V^T P' per group and N tile ----
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {
      uint32_t vw[4];
      ldsm_x4_t(vw, sa + kPfxOffVc + gp * 512 + ld_v);
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = 2 * gp + gg;
        uint32_t vl[4], vh[4];
        nib_pairs_v_sub(vw[2 * gg], vl);
        nib_pairs_v_sub(vw[2 * gg + 1], vh);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint32_t *pb = x.ptile + ((t * 4 + g) * 8 + gid) * kPWordsPerCol + tig;
          const uint32_t b01 = pb[0], b23 = pb[4];
          mma_f16(o[g][0][t], vl[0], vl[1], vh[0], vh[1], b01, b23);
          mma_f16(o[g][1][t], vl[2], vl[3], vh[2], vh[3], b01, b23);
        }
      }
    }
    __syncwarp();
    if (k + kStages < np) issue(k + kStages);
  }

  // ---- finish: reduce over the 8 token lanes, write each member's partial ----
  if (LIFT) {
    const float probe[16] = {o[0][0][0][0], o[0][0][0][1], o[0][0][1][0], o[0][0][1][1],
                             o[1][0][0][0], o[1][0][0][1], o[1][0][1][0], o[1][0][1][1],
                             o[2][0][0][0], o[2][0][0][1], o[2][0][1][0], o[2][0][1][1],
                             o[3][0][0][0], o[3][0][0][1], o[3][0][1][0], o[3][0][1][1]};
    if (any_not_finite(probe)) return true;
  }
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) l[t][e] += __shfl_xor_sync(0xffffffffu, l[t][e], off);
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)
          mt[g][t][e] += __shfl_xor_sync(0xffffffffu, mt[g][t][e], off);
    }
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int col = 8 * t + 2 * tig + e, mi = col / G, j = col - mi * G;
      if (mi >= nmem) continue;
      const int r = regions_of(c.seq_lens[b0 + mi], S, R, w.chunk_pages).has_prot + ci;
      float *rr = record_of(w, H, G, b0 + mi, h, r) + j * kRecordFloats;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 v = make_float4(fmaf(o[g][0][t][e], kUnscaleV, mt[g][t][e]),
                                     fmaf(o[g][0][t][2 + e], kUnscaleV1, mt[g][t][e]),
                                     fmaf(o[g][1][t][e], kUnscaleV, mt[g][t][e]),
                                     fmaf(o[g][1][t][2 + e], kUnscaleV1, mt[g][t][e]));
        st_rec(reinterpret_cast<float4 *>(rr + 32 * g + 4 * gid), v);
      }
      if (gid == 0) {
        st_rec(rr + kHeadDim, m[t][e] * kLn2);
        st_rec(rr + kHeadDim + 1, l[t][e]);
      }
    }
  return false;
}

__global__ void __launch_bounds__(kWarps * 32, KV4_MIN_BLOCKS) prefix_kernel(CacheView c, Workspace w,
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
  x.ptile = reinterpret_cast<uint32_t *>(mine + kStages * kStageBytes);
  x.ptile8 = reinterpret_cast<uint16_t *>(mine + kStages * kStageBytes + kPtileBytes);
  x.bars = reinterpret_cast<uint64_t *>(mine + kStages * kStageBytes + kPtileBytes + kPtile8Bytes);
  init_warp<false>(x, w);
  if (x.lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&x.bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (w.check_plan && !plan_matches(c, w)) {  // a reused list of another batch: read none
    if (x.lane == 0) set_err(err, KV4_DEVERR_WORKSPACE);
    return;
  }
  const int base = *w.n_items;  // the prefix entries follow the attention kernel's
  const int n_items = *w.pn_items;
  for (;;) {
    int item = 0;
    if (x.lane == 0) item = atomicAdd(w.pcounter, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item >= n_items) break;
    const int4 en = w.entries[base + item];
    if (process_prefix<true>(x, c, w, q, en.x, -1 - en.y, en.z, en.w, err))
      process_prefix<false>(x, c, w, q, en.x, -1 - en.y, en.z, en.w, err);
    if (x.dead) break;
  }
}

// ---------------------------------------------------------------------------
// exact regional merge
// ---------------------------------------------------------------------------
// One warp merges query j of unit u over its regions r0 .. r0+n-1:
//   M = max m_r, Lambda = sum l_r e^(m_r - M), O = sum acc_r e^(m_r - M) / Lambda,
//   lse = M + ln Lambda, over live regions (l_r > 0); no live region gives O = 0,
//   lse = -inf.
// Regions are taken in batches of 4: every lane loads its 4 dims of each record of the
// batch and, with one broadcast load per record, the record's (m, l); each lane then
// forms the batch's maximum and weights itself (no shuffles) and adds the records in
// region order. The arithmetic order is fixed, so the result is deterministic; M is the
// running maximum over the batches (with a rescale between batches, as in the online
// softmax). e^x is evaluated as 2^(x log2 e) with x = m_r - M formed first, so the
// rounding of the scaling is relative to the difference (weights and Lambda to a few
// 1e-7 relative for the differences that carry weight); 1/Lambda and ln Lambda use the
// hardware reciprocal and base-2 logarithm (1-2 ulp). Against per-lane gathers with
// shuffle reductions, IEEE division and the library exp/log (292 instructions per row)
// this takes a third of the instructions. Batches of 4 rather than 8 keep the registers
// low enough for 40 resident warps per SM.
__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float fast_rcp(float x) {
  float y;
  asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(256, 5) merge_kernel(const float *__restrict__ partials,
                                                    const int32_t *__restrict__ offs, int n_units,
                                                    int G, int g_shift, Outputs o, int32_t *reset,
                                                    PlanSig want, int check) {
  constexpr int kBatch = 4;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (check) {  // a reused work list must be this call's (see plan_signature)
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) ok &= reset[8 + i] == want.v[i];
    if (!ok) {
      if (warp < n_units * G) {  // write zero outputs, lse = -inf; read no partial state
        const size_t row = static_cast<size_t>(warp);
        *reinterpret_cast<uint2 *>(o.out + row * kHeadDim + 4 * lane) = make_uint2(0u, 0u);
        if (o.out_f32)
          *reinterpret_cast<float4 *>(o.out_f32 + row * kHeadDim + 4 * lane) =
              make_float4(0.f, 0.f, 0.f, 0.f);
        if (o.lse && lane == 0) o.lse[row] = -CUDART_INF_F;
      }
      return;
    }
  }
  if (reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    // the call's attention kernels are done: zero the work counters of the work list
    // (counter, prefix counter, lift list count and counter) for a call that reuses it
    reset[0] = 0;
    reset[2] = 0;
    reset[4] = 0;
    reset[5] = 0;
  }
  if (warp >= n_units * G) return;
  const int u = g_shift >= 0 ? warp >> g_shift : warp / G;
  const int j = warp - u * G;
  const int r0 = offs[u], n = offs[u + 1] - r0;
  const int stride = G * kRecordFloats;  // floats from one region's record to the next
  const float *rec = partials + (static_cast<size_t>(r0) * G + j) * kRecordFloats;
  float M = -CUDART_INF_F, lam = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int base = 0; base < n; base += kBatch, rec += kBatch * stride) {
    const int cnt = min(kBatch, n - base);
    float4 a[kBatch];
    float2 ml[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      a[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      ml[i] = make_float2(-CUDART_INF_F, 0.f);
      if (i < cnt) {
        a[i] = __ldcs(reinterpret_cast<const float4 *>(rec + i * stride) + lane);
        ml[i] = __ldcs(reinterpret_cast<const float2 *>(rec + i * stride + kHeadDim));
      }
    }
    float mr[kBatch];
    float bm = -CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      mr[i] = ml[i].y > 0.f ? ml[i].x : -CUDART_INF_F;  // only live regions carry weight
      bm = fmaxf(bm, mr[i]);
    }
    if (bm == -CUDART_INF_F) continue;  // no live region in this batch
    const float Mn = fmaxf(M, bm);
    if (Mn != M) {  // rescale what was accumulated under the old maximum (0 at the start)
      const float sc = fast_exp2((M - Mn) * kLog2e);
      acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
      lam *= sc;
      M = Mn;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const float wgt = fast_exp2((mr[i] - M) * kLog2e);  // 0 for a dead or absent region
      if (wgt > 0.f) {  // a skipped region's acc is never read into the sum
        lam = fmaf(ml[i].y, wgt, lam);
        acc.x = fmaf(a[i].x, wgt, acc.x);
        acc.y = fmaf(a[i].y, wgt, acc.y);
        acc.z = fmaf(a[i].z, wgt, acc.z);
        acc.w = fmaf(a[i].w, wgt, acc.w);
      }
    }
  }
  const float inv = lam > 0.f ? fast_rcp(lam) : 0.f;
  const float4 v = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  const size_t row = static_cast<size_t>(u) * G + j;
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t *>(&lo);
  packed.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(o.out + row * kHeadDim + 4 * lane) = packed;
  if (o.out_f32) *reinterpret_cast<float4 *>(o.out_f32 + row * kHeadDim + 4 * lane) = v;
  if (o.lse && lane == 0) o.lse[row] = lam > 0.f ? M + fast_log2(lam) * kLn2 : -CUDART_INF_F;
}


template <int HPW, bool HOOK>
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
  x.ptile = reinterpret_cast<uint32_t *>(mine + kStages * kStageBytes);
  x.ptile8 = reinterpret_cast<uint16_t *>(mine + kStages * kStageBytes + kPtileBytes);
  x.bars = reinterpret_cast<uint64_t *>(mine + kStages * kStageBytes + kPtileBytes + kPtile8Bytes);
  init_warp<HOOK>(x, w);
  // the INT4 P' tile's unused columns stay zero for the whole kernel
  for (int i = x.lane; i < kPtileBytes / 4; i += 32) x.ptile[i] = 0u;
  if (x.lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&x.bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const int H = c.num_kv_heads, G = c.gqa;
  if (w.check_plan && !plan_matches(c, w)) {  // a reused list of another batch: read none
    if (x.lane == 0) set_err(err, KV4_DEVERR_WORKSPACE);
    return;
  }
  const int n_items = *w.n_items;
  for (;;) {
    int item = 0;
    if (x.lane == 0) item = atomicAdd(w.counter, 1);
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item >= n_items) break;
    x.fault = withheld_item<HOOK>(w, item);
    const int4 en = w.entries[item];
    const int b = en.x, r = en.y, h0 = en.z, nh = en.w;
    const int L = c.seq_lens[b];
    if (L < 0 || L > c.max_pages * kPage) {  // (a reused list whose lengths have changed)
      if (x.lane == 0) set_err(err, KV4_DEVERR_SEQ_LEN);
      continue;
    }
    const int pe = w.prefix_end ? w.prefix_end[b] : 0;
    const Regions rg = regions_of(L, c.num_sinks, c.num_recent, w.chunk_pages, pe);
    int res;
    if (r < rg.has_prot) {
      if constexpr (HPW == 2)
        res = process_protected_pair<kDecide>(x, c, w, q, b, h0, nh, L, r, err);
      else
        res = process_protected<kDecide>(x, c, q, b, h0, L, record_of(w, H, G, b, h0, r), err);
    } else {
      res = process_int4<HPW, kDecide>(x, c, w, q, b, h0, nh, r, r - rg.has_prot - rg.n_prompt,
                                       rg, err);
    }
    if (res == kWantLift && x.lane == 0) w.lift_items[atomicAdd(w.lift_count, 1)] = item;
    if (x.dead) break;
  }
}

// The entries of the lift list (small V scales): redone with the lift of their weights,
// and again without it if a later weight overflowed fp16 under the lift.
template <int HPW>
__global__ void __launch_bounds__(kWarps * 32, KV4_MIN_BLOCKS) lift_kernel(CacheView c, Workspace w,
                                                                           const uint16_t *__restrict__ q,
                                                                           int32_t *err) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (w.check_plan && !plan_matches(c, w)) return;  // flagged by the attention kernel
  const int n_items = *w.lift_count;
  if (n_items == 0) return;
  WarpCtx x;
  const int warp = threadIdx.x >> 5;
  x.lane = threadIdx.x & 31;
  x.gid = x.lane >> 2;
  x.tig = x.lane & 3;
  uint8_t *mine = smem + warp * kWarpSmem;
  x.stage0 = mine;
  x.ptile = reinterpret_cast<uint32_t *>(mine + kStages * kStageBytes);
  x.ptile8 = reinterpret_cast<uint16_t *>(mine + kStages * kStageBytes + kPtileBytes);
  x.bars = reinterpret_cast<uint64_t *>(mine + kStages * kStageBytes + kPtileBytes + kPtile8Bytes);
  init_warp<false>(x, w);
  for (int i = x.lane; i < kPtileBytes / 4; i += 32) x.ptile[i] = 0u;
  if (x.lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&x.bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
  const int H = c.num_kv_heads, G = c.gqa;
  for (;;) {
    int i = 0;
    if (x.lane == 0) i = atomicAdd(w.lift_counter, 1);
    i = __shfl_sync(0xffffffffu, i, 0);
    if (i >= n_items) break;
    const int4 en = w.entries[w.lift_items[i]];
    const int b = en.x, r = en.y, h0 = en.z, nh = en.w;
    const int L = c.seq_lens[b];
    const int pe = w.prefix_end ? w.prefix_end[b] : 0;
    const Regions rg = regions_of(L, c.num_sinks, c.num_recent, w.chunk_pages, pe);
    if (r < rg.has_prot) {
      if constexpr (HPW == 2) {
        if (process_protected_pair<kLifted>(x, c, w, q, b, h0, nh, L, r, err) == kOverflow)
          process_protected_pair<kPlain>(x, c, w, q, b, h0, nh, L, r, err);
      } else {
        float *rec = record_of(w, H, G, b, h0, r);
        if (process_protected<kLifted>(x, c, q, b, h0, L, rec, err) == kOverflow)
          process_protected<kPlain>(x, c, q, b, h0, L, rec, err);
      }
    } else {
      const int chunk = r - rg.has_prot - rg.n_prompt;
      if (process_int4<HPW, kLifted>(x, c, w, q, b, h0, nh, r, chunk, rg, err) == kOverflow)
        process_int4<HPW, kPlain>(x, c, w, q, b, h0, nh, r, chunk, rg, err);
    }
    if (x.dead) break;
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_plan(const CacheView &c, const Workspace &w, int32_t *err_flag,
                        cudaStream_t s) {
  int ctas = 0, threads = 0;
  plan_shape(c.num_seqs, &ctas, &threads);
  plan_kernel<<<ctas, threads, 0, s>>>(c, w, err_flag);
  return cudaGetLastError();
}

template <int HPW, bool HOOK>
static cudaError_t launch_attn_t(const CacheView &c, const Workspace &w, const uint16_t *q,
                                 int32_t *err_flag, cudaStream_t s) {
  static PerDevice grids;  // persistent grid per device
  int grid = 0;
  cudaError_t e = once_per_device(grids, [](int dev, int *g) {
    cudaError_t r = cudaFuncSetAttribute(attn_kernel<HPW, HOOK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kCtaSmem);
    int sms = 0, per_sm = 0;
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_kernel<HPW, HOOK>,
                                                        kWarps * 32, kCtaSmem);
    *g = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  }, &grid);
  if (e != cudaSuccess) return e;
  attn_kernel<HPW, HOOK><<<grid, kWarps * 32, kCtaSmem, s>>>(c, w, q, err_flag);
  return cudaGetLastError();
}

cudaError_t launch_prefix(const CacheView &c, const Workspace &w, const uint16_t *q,
                          int32_t *err_flag, cudaStream_t s) {
  if (w.prefix_end == nullptr) return cudaSuccess;
  static PerDevice grids;  // persistent grid per device
  int grid = 0;
  cudaError_t e = once_per_device(grids, [](int dev, int *g) {
    cudaError_t r = cudaFuncSetAttribute(prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kCtaSmem);
    int sms = 0, per_sm = 0;
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefix_kernel, kWarps * 32,
                                                        kCtaSmem);
    *g = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  }, &grid);
  if (e != cudaSuccess) return e;
  prefix_kernel<<<grid, kWarps * 32, kCtaSmem, s>>>(c, w, q, err_flag);
  return cudaGetLastError();
}

int heads_per_warp_for(int gqa) { return gqa <= 4 ? 2 : 1; }

PlanSig plan_signature_host(const CacheView &c, const Workspace &w) {
  PlanSig p;
  p.v[0] = 0x4b563450;
  p.v[1] = c.num_seqs;
  p.v[2] = c.num_kv_heads;
  p.v[3] = c.gqa | (w.heads_per_warp << 8) | (w.prefix_end != nullptr ? 1 << 16 : 0);
  p.v[4] = w.chunk_pages;
  p.v[5] = c.num_sinks | (c.num_recent << 16);
  p.v[6] = w.cap_entries;
  p.v[7] = w.cap_pairs;
  return p;
}

// The persistent grid of the attention kernel: an empty list costs a launch whose CTAs
// end at once (about 3 us), a long one (small values everywhere) runs at full width.
template <int HPW>
static cudaError_t launch_lift_t(const CacheView &c, const Workspace &w, const uint16_t *q,
                                 int32_t *err_flag, cudaStream_t s) {
  static PerDevice grids;
  int grid = 0;
  cudaError_t e = once_per_device(grids, [](int dev, int *g) {
    cudaError_t r = cudaFuncSetAttribute(lift_kernel<HPW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kCtaSmem);
    int sms = 0, per_sm = 0;
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lift_kernel<HPW>, kWarps * 32,
                                                        kCtaSmem);
    *g = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  }, &grid);
  if (e != cudaSuccess) return e;
  lift_kernel<HPW><<<grid, kWarps * 32, kCtaSmem, s>>>(c, w, q, err_flag);
  return cudaGetLastError();
}

cudaError_t launch_attention(const CacheView &c, const Workspace &w, const uint16_t *q,
                             int32_t *err_flag, cudaStream_t s) {
  cudaError_t e;
  if (w.fault_item >= 0)  // the testing hook is armed for this call
    e = w.heads_per_warp == 2 ? launch_attn_t<2, true>(c, w, q, err_flag, s)
                              : launch_attn_t<1, true>(c, w, q, err_flag, s);
  else
    e = w.heads_per_warp == 2 ? launch_attn_t<2, false>(c, w, q, err_flag, s)
                              : launch_attn_t<1, false>(c, w, q, err_flag, s);
  if (e != cudaSuccess) return e;
  return w.heads_per_warp == 2 ? launch_lift_t<2>(c, w, q, err_flag, s)
                               : launch_lift_t<1>(c, w, q, err_flag, s);
}

cudaError_t launch_merge(const float *partials, const int32_t *unit_offsets, int32_t n_units,
                         int32_t group, uint16_t *out, float *out_f32, float *lse,
                         const int32_t *reset, const PlanSig *want, cudaStream_t s) {
  const long long warps = static_cast<long long>(n_units) * group;
  if (warps == 0) return cudaSuccess;
  const long long blocks = (warps * 32 + 255) / 256;
  const int g_shift = (group & (group - 1)) == 0 ? __builtin_ctz(group) : -1;
  merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      partials, unit_offsets, n_units, group, g_shift, Outputs{out, out_f32, lse},
      const_cast<int32_t *>(reset), want ? *want : PlanSig{}, want && reset ? 1 : 0);
  return cudaGetLastError();
}

size_t workspace_bytes(int32_t num_seqs, int32_t max_seq_len, int32_t num_kv_heads, int32_t gqa,
                       int32_t chunk_pages, bool prefix, Workspace *carve, void *base) {
  const long long pages = (static_cast<long long>(max_seq_len) + kPage - 1) / kPage + 1;
  // regions per sequence: the protected set and the INT4 chunks; with the shared-prefix
  // read the INT4 pages are cut once more (shared pages | own pages): one region more
  const long long per_seq = (prefix ? 2 : 1) + (pages + chunk_pages - 1) / chunk_pages;
  const long long cap = static_cast<long long>(num_seqs) * per_seq;
  const long long cap_e = cap * num_kv_heads;
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  size_t off = 256;  // counters and counts (work, prefix work, lift list)
  const size_t ent_off = off;
  off = up(off + static_cast<size_t>(cap_e) * sizeof(int4));
  const size_t units_off = off;
  off = up(off + (static_cast<size_t>(num_seqs) * num_kv_heads + 1) * sizeof(int32_t));
  const size_t lift_off = off;  // the lift list: at most one per entry
  off = up(off + static_cast<size_t>(cap_e) * sizeof(int32_t));
  size_t pend_off = 0;
  if (prefix) {
    pend_off = off;
    off = up(off + static_cast<size_t>(num_seqs) * sizeof(int32_t));
  }
  const size_t part_off = off;
  off = up(off + static_cast<size_t>(cap) * num_kv_heads * gqa * kRecordFloats * sizeof(float));
  if (carve) {
    uint8_t *p = static_cast<uint8_t *>(base);
    carve->counter = reinterpret_cast<int32_t *>(p);
    carve->n_items = reinterpret_cast<int32_t *>(p) + 1;
    carve->pcounter = reinterpret_cast<int32_t *>(p) + 2;
    carve->pn_items = reinterpret_cast<int32_t *>(p) + 3;
    carve->lift_count = reinterpret_cast<int32_t *>(p) + 4;
    carve->lift_counter = reinterpret_cast<int32_t *>(p) + 5;
    carve->lift_items = reinterpret_cast<int32_t *>(p + lift_off);
    carve->entries = reinterpret_cast<int4 *>(p + ent_off);
    carve->unit_offsets = reinterpret_cast<int32_t *>(p + units_off);
    carve->prefix_end = prefix ? reinterpret_cast<int32_t *>(p + pend_off) : nullptr;
    carve->partials = reinterpret_cast<float *>(p + part_off);
    carve->cap_pairs = static_cast<int32_t>(cap);
    carve->cap_entries = static_cast<int32_t>(cap_e);
    carve->chunk_pages = chunk_pages;
    carve->heads_per_warp = heads_per_warp_for(gqa);
    carve->wait_limit = kWaitLimit;
    carve->fault_item = -1;
    carve->check_plan = 0;
  }
  return off;
}

}  // namespace kv4
