// Comparison baselines: the same paged decode attention over an unquantised BF16 cache
// and over an all-INT8 (KV8) cache. The pages measure KV4 against both (KV8 "tracks
// BF16 closely", and the replay throughputs are quoted against BF16: ai4snews summary,
// "Interpretation" paras. 1-2); these kernels reproduce the bytes-per-position side of
// that comparison with the same harness as the KV4-RL path (plan, persistent grid,
// per-warp copy ring, exact merge).
//
//   baseline_append_kernel<F>  one warp per (new token, kv head): BF16 copies the row into
//                              its page slot; KV8 quantises it with the INT8 quantiser of
//                              the protected set (symmetric, per token and head, fp16 scale).
//   baseline_attn_kernel<F>    persistent; every warp takes (sequence, chunk of pages, kv
//                              head) entries and computes the partial softmax state over
//                              those pages for the head's G queries. A page takes two ring
//                              stages: its K part, then its V part.
//                                BF16: QK^T and PV on the bf16 tensor cores (P split into
//                                      a bf16 high and low part, two MMAs, so P keeps ~16
//                                      bits); K/V pages in octet-major layout for ldmatrix.
//                                KV8:  QK^T on the integer tensor cores (int8 codes x the
//                                      fixed-point query), PV with int8 -> fp16 codes and
//                                      P' = p * vscale in fp16, as for the protected set.
// The work list (plan_kernel, with no protected set) and the merge are the KV4-RL ones.
#include "kv4_attn_common.cuh"

namespace kv4 {

constexpr int kFmtBf16 = KV4_BASELINE_BF16;
constexpr int kFmtKv8 = KV4_BASELINE_KV8;
constexpr int kBf16PartBytes = kPage * kHeadDim * 2;              // 4096: K or V of a page
constexpr int kKv8PartBytes = kInt8CodeBytes + kInt8ScaleBytes;  // 2080: codes + scales

// ---------------------------------------------------------------------------
// append
// ---------------------------------------------------------------------------
template <int F>
__global__ void __launch_bounds__(256) baseline_append_kernel(CacheView c,
                                                              const uint16_t *__restrict__ k_new,
                                                              const uint16_t *__restrict__ v_new,
                                                              const int32_t *__restrict__ new_indptr,
                                                              int32_t total_new, int32_t *err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int H = c.num_kv_heads;
  if (warp >= total_new * H) return;
  const int row = warp / H;
  const int h = warp - row * H;
  int b, pos, L;
  locate_new_token(c.seq_lens, c.num_seqs, new_indptr, row, b, pos, L);
  if (pos < 0 || pos >= L || L > c.max_pages * kPage) {
    if (lane == 0) set_err(err, KV4_DEVERR_SEQ_LEN);
    return;
  }
  const int page = c.page_table[static_cast<size_t>(b) * c.max_pages + pos / kPage];
  if (page < 0 || page >= c.num_pages) {
    if (lane == 0) set_err(err, KV4_DEVERR_PAGE_ID);
    return;
  }
  const int slot = pos % kPage;
  const size_t blk = static_cast<size_t>(page) * H + h;
  const size_t rowoff = (static_cast<size_t>(row) * H + h) * kHeadDim + 4 * lane;  // dims 4l..4l+3
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const uint2 raw = *reinterpret_cast<const uint2 *>((which == 0 ? k_new : v_new) + rowoff);
    uint8_t *dst = which == 0 ? c.k_codes : c.v_codes;
    if constexpr (F == kFmtBf16) {
      // [16 octets of dims][16 slots][8 dims]: lane l holds half (l & 1) of octet l / 2
      *reinterpret_cast<uint2 *>(dst + ((blk * 16 + (lane >> 1)) * kPage + slot) * 16 +
                                 8 * (lane & 1)) = raw;
    } else {
      float x[4];
      x[0] = bf16_bits_to_f32(static_cast<uint16_t>(raw.x & 0xFFFFu));
      x[1] = bf16_bits_to_f32(static_cast<uint16_t>(raw.x >> 16));
      x[2] = bf16_bits_to_f32(static_cast<uint16_t>(raw.y & 0xFFFFu));
      x[3] = bf16_bits_to_f32(static_cast<uint16_t>(raw.y >> 16));
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
      for (int off = 1; off < 32; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const __half s8h = f16_sat(quotient_rn(amax, 127.0f, kRcp127));
      const float s8 = __half2float(s8h);
      const float r8 = s8 == 0.0f ? 0.0f : __frcp_rn(s8);
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float qv = rintf(quotient_rn(x[i], s8, r8));  // r8 = 0 when s8 = 0: 0
        qv = fminf(fmaxf(qv, -127.0f), 127.0f);
        word |= (static_cast<uint32_t>(static_cast<int32_t>(qv)) & 0xFFu) << (8 * i);
      }
      // [8 strips of 16 dims][16 slots][16 bytes]: lane l -> strip l / 4, bytes 4 (l % 4)
      *reinterpret_cast<uint32_t *>(dst + blk * kInt8CodeBytes + (lane >> 2) * (kPage * 16) +
                                    slot * 16 + 4 * (lane & 3)) = word;
      if (lane == 0) (which == 0 ? c.k_params : c.v_params)[blk * kPage + slot] = __half_as_ushort(s8h);
    }
  }
}

// ---------------------------------------------------------------------------
// attention: one kv head per warp, MMA N columns = the head's G queries
// ---------------------------------------------------------------------------
template <int F>
__device__ __forceinline__ void process_baseline(WarpCtx &x, const CacheView &c, const Workspace &w,
                                 const uint16_t *__restrict__ q, int b, int h, int r,
                                 const Regions &rg, int32_t *err) {
  const int G = c.gqa, H = c.num_kv_heads;
  const int lane = x.lane, gid = x.gid, tig = x.tig;
  const int L = rg.int4_hi;  // no protected set: the region is [0, L)
  const int p0 = r * w.chunk_pages;
  const int last = (L - 1) / kPage;
  const int np = min(w.chunk_pages, last - p0 + 1);
  const int nv = 2 * np;  // copies: K part, then V part, of every page
  float *rec = record_of(w, H, G, b, h, r);
  if (np < 1) {  // only with a reused work list whose lengths have changed
    if (lane == 0) set_err(err, KV4_DEVERR_WORKSPACE);
    write_empty(rec, G, lane);
    return;
  }

  const int *pt = c.page_table + static_cast<size_t>(b) * c.max_pages + p0;
  int pid = 0, pid2 = 0;
  if (lane < np) pid = pt[lane];
  if (lane + 32 < np) pid2 = pt[lane + 32];
  const bool bad = (lane < np && (pid < 0 || pid >= c.num_pages)) ||
                   (lane + 32 < np && (pid2 < 0 || pid2 >= c.num_pages));
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) set_err(err, KV4_DEVERR_PAGE_ID);
    write_empty(rec, G, lane);
    return;
  }

  auto issue = [&](int k) {
    const int page = k >> 1;
    const int pk = __shfl_sync(0xffffffffu, page < 32 ? pid : pid2, page & 31);
    const int st = k % kStages;
    if (lane == 0) {
      uint8_t *dst = x.stage0 + st * kStageBytes;
      const size_t blk = static_cast<size_t>(pk) * H + h;
      const bool vpart = (k & 1) != 0;
      fence_proxy_async_smem();
      if constexpr (F == kFmtBf16) {
        mbar_arrive_expect_tx(&x.bars[st], kBf16PartBytes);
        bulk_g2s(dst, (vpart ? c.v_codes : c.k_codes) + blk * kBf16PartBytes, kBf16PartBytes,
                 &x.bars[st]);
      } else {
        mbar_arrive_expect_tx(&x.bars[st], kKv8PartBytes);
        bulk_g2s(dst, (vpart ? c.v_codes : c.k_codes) + blk * kInt8CodeBytes, kInt8CodeBytes,
                 &x.bars[st]);
        bulk_g2s(dst + kInt8CodeBytes, (vpart ? c.v_params : c.k_params) + blk * kPage,
                 kInt8ScaleBytes, &x.bars[st]);
      }
    }
  };
  int issued = min(nv, kStages);
  for (int k = 0; k < issued; ++k)
    if (prologue_copy(x, k)) issue(k);
  auto give_up = [&](int k) {
    drain_copies(x, k, issued, k);
    write_empty(rec, G, lane);
  };

  // ---- query fragments (B operand of QK^T); lane column gid = query gid ----
  const bool live = gid < G;
  const uint16_t *qrow = q + (static_cast<size_t>(b) * H * G + h * G + gid) * kHeadDim;
  uint32_t qb[8][2];       // BF16: k-step kk: dims 16kk+2tig..+1 and 16kk+8+2tig..+1
  uint32_t qh[4][2], ql[4][2];  // KV8: 15-bit fixed point, hi / lo bytes
  float2 kq;
  if constexpr (F == kFmtBf16) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qb[kk][0] = live ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 2 * tig) : 0u;
      qb[kk][1] = live ? *reinterpret_cast<const uint32_t *>(qrow + 16 * kk + 8 + 2 * tig) : 0u;
    }
    kq = make_float2(kScaleLog2, kScaleLog2);
  } else {
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
  // ldmatrix lane addresses
  const int mi = lane >> 3, r8 = lane & 7;
  const int ld8 = ((lane >> 4) * 256) + ((lane >> 3) & 1) * 128 + r8 * 16;  // KV8 strips
  // BF16 K (rows = positions): matrices (octet 2kk | slots 0-7), (2kk | 8-15), (2kk+1 | 0-7),
  // (2kk+1 | 8-15); V transposed: (2cc | 0-7), (2cc+1 | 0-7), (2cc | 8-15), (2cc+1 | 8-15)
  const int ldk16 = ((mi >> 1) * kPage + (mi & 1) * 8 + r8) * 16;
  const int ldv16 = ((mi & 1) * kPage + (mi >> 1) * 8 + r8) * 16;
  uint16_t *pt_hi = reinterpret_cast<uint16_t *>(x.ptile);  // BF16 P: [2][8 cols][16 pos]
  const bool write_p0 = 2 * tig < G, write_p1 = 2 * tig + 1 < G;

  for (int j = 0; j < np; ++j) {
    // ---- K part: logits ----
    const int kk_ = 2 * j;
    if (!wait_stage(x, kk_ % kStages, err)) {
      give_up(kk_);
      return;
    }
    const uint8_t *spk = x.stage0 + (kk_ % kStages) * kStageBytes;
    const uint32_t sak = smem_u32(spk);
    float d[4];
    float sk[2] = {1.f, 1.f};
    if constexpr (F == kFmtBf16) {
      d[0] = d[1] = d[2] = d[3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, sak + 2 * kk * kPage * 16 + ldk16);
        mma_bf16(d, a[0], a[1], a[2], a[3], qb[kk][0], qb[kk][1]);
      }
    } else {
      int32_t ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t kw[4];  // rows = positions, k = dims 32ks..32ks+31
        ldsm_x4(kw, sak + ks * 512 + ld8);
        mma_s8s8(ah, kw[0], kw[1], kw[2], kw[3], qh[ks][0], qh[ks][1]);
        mma_s8u8(al, kw[0], kw[1], kw[2], kw[3], ql[ks][0], ql[ks][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] = static_cast<float>(ah[i] * 256 + al[i]);  // exact
      const uint16_t *ks = reinterpret_cast<const uint16_t *>(spk + kInt8CodeBytes);
      sk[0] = __half2float(__ushort_as_half(ks[gid]));
      sk[1] = __half2float(__ushort_as_half(ks[gid + 8]));
    }
    __syncwarp();
    if (issued < nv) issue(issued++);  // the K stage is free again
    float s[2][2];
    const int tok0 = (p0 + j) * kPage;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const bool valid = tok0 + gid + 8 * hf < L;
      s[hf][0] = valid ? d[2 * hf] * sk[hf] * kq.x : -CUDART_INF_F;
      s[hf][1] = valid ? d[2 * hf + 1] * sk[hf] * kq.y : -CUDART_INF_F;
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
      const float mn = fmaxf(m[e], t);
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

    // ---- V part: P into shared memory, O^T += V^T P per 16-dim strip ----
    const int kv_ = 2 * j + 1;
    if (!wait_stage(x, kv_ % kStages, err)) {
      give_up(kv_);
      return;
    }
    const uint8_t *spv = x.stage0 + (kv_ % kStages) * kStageBytes;
    const uint32_t sav = smem_u32(spv);
    uint32_t b01 = 0u, b23 = 0u, c01 = 0u, c23 = 0u;
    if constexpr (F == kFmtBf16) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (e == 0 ? !write_p0 : !write_p1) continue;
        const int col = 2 * tig + e;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float p = s[hf][e];
          const __nv_bfloat16 hi = __float2bfloat16_rn(p);
          const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
          pt_hi[col * kPage + gid + 8 * hf] = __bfloat16_as_ushort(hi);
          pt_hi[8 * kPage + col * kPage + gid + 8 * hf] = __bfloat16_as_ushort(lo);
        }
      }
      __syncwarp();
      if (live) {
        b01 = *reinterpret_cast<const uint32_t *>(pt_hi + gid * kPage + 2 * tig);
        b23 = *reinterpret_cast<const uint32_t *>(pt_hi + gid * kPage + 2 * tig + 8);
        c01 = *reinterpret_cast<const uint32_t *>(pt_hi + 8 * kPage + gid * kPage + 2 * tig);
        c23 = *reinterpret_cast<const uint32_t *>(pt_hi + 8 * kPage + gid * kPage + 2 * tig + 8);
      }
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t v4[4];
        ldsm_x4_t(v4, sav + 2 * cc * kPage * 16 + ldv16);
        mma_bf16(o[cc], v4[0], v4[1], v4[2], v4[3], b01, b23);
        mma_bf16(o[cc], v4[0], v4[1], v4[2], v4[3], c01, c23);
      }
    } else {
      const uint16_t *vs = reinterpret_cast<const uint16_t *>(spv + kInt8CodeBytes);
      const float sv0 = __half2float(__ushort_as_half(vs[gid]));
      const float sv1 = __half2float(__ushort_as_half(vs[gid + 8]));
      if (write_p0) {
        x.ptile8[(2 * tig) * 16 + gid] = __half_as_ushort(__float2half_rn(s[0][0] * sv0));
        x.ptile8[(2 * tig) * 16 + gid + 8] = __half_as_ushort(__float2half_rn(s[1][0] * sv1));
      }
      if (write_p1) {
        x.ptile8[(2 * tig + 1) * 16 + gid] = __half_as_ushort(__float2half_rn(s[0][1] * sv0));
        x.ptile8[(2 * tig + 1) * 16 + gid + 8] = __half_as_ushort(__float2half_rn(s[1][1] * sv1));
      }
      __syncwarp();
      if (live) {
        b01 = *reinterpret_cast<const uint32_t *>(&x.ptile8[gid * 16 + 2 * tig]);
        b23 = *reinterpret_cast<const uint32_t *>(&x.ptile8[gid * 16 + 2 * tig + 8]);
      }
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        uint32_t vw[4];
        ldsm_x4_t(vw, sav + pr * 512 + ld8);
#pragma unroll
        for (int sp2 = 0; sp2 < 2; ++sp2) {
          const int cc = 2 * pr + sp2;
          const uint32_t ulo = vw[2 * sp2] ^ 0x80808080u, uhi = vw[2 * sp2 + 1] ^ 0x80808080u;
          mma_f16(o[cc], s8_pair<0x4240>(ulo), s8_pair<0x4341>(ulo), s8_pair<0x4240>(uhi),
                  s8_pair<0x4341>(uhi), b01, b23);
        }
      }
    }
    __syncwarp();
    if (issued < nv) issue(issued++);  // the V stage is free again
  }

  // ---- finish: reduce the denominators over the 8 position lanes, write the partials ----
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], off);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int jq = 2 * tig + e;
    if (jq >= G) continue;
    float *rr = rec + jq * kRecordFloats;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      if constexpr (F == kFmtBf16) {  // rows: dim 16cc+gid (c0/c1) and 16cc+8+gid (c2/c3)
        rr[16 * cc + gid] = o[cc][e];
        rr[16 * cc + 8 + gid] = o[cc][2 + e];
      } else {  // rows: dim 16cc+2gid (c0/c1) and +1 (c2/c3)
        *reinterpret_cast<float2 *>(rr + 16 * cc + 2 * gid) = make_float2(o[cc][e], o[cc][2 + e]);
      }
    }
    if (gid == 0) {
      rr[kHeadDim] = m[e] * kLn2;
      rr[kHeadDim + 1] = l[e];
    }
  }
}

template <int F, bool HOOK>
__global__ void __launch_bounds__(kWarps * 32, KV4_MIN_BLOCKS) baseline_attn_kernel(
    CacheView c, Workspace w, const uint16_t *__restrict__ q, int32_t *err) {
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
  if (x.lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&x.bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
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
    const int b = en.x, r = en.y, h = en.z;
    const int L = c.seq_lens[b];
    if (L < 0 || L > c.max_pages * kPage) {  // (a reused list whose lengths have changed)
      if (x.lane == 0) set_err(err, KV4_DEVERR_SEQ_LEN);
      continue;
    }
    const Regions rg = regions_of(L, 0, 0, w.chunk_pages);
    process_baseline<F>(x, c, w, q, b, h, r, rg, err);
    if (x.dead) break;
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_baseline_append(int fmt, const CacheView &c, const uint16_t *k_new,
                                   const uint16_t *v_new, const int32_t *new_indptr,
                                   int32_t total_new, int32_t *err_flag, cudaStream_t s) {
  if (total_new == 0) return cudaSuccess;
  const long long warps = static_cast<long long>(total_new) * c.num_kv_heads;
  const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
  if (fmt == kFmtBf16)
    baseline_append_kernel<kFmtBf16><<<blocks, 256, 0, s>>>(c, k_new, v_new, new_indptr,
                                                           total_new, err_flag);
  else
    baseline_append_kernel<kFmtKv8><<<blocks, 256, 0, s>>>(c, k_new, v_new, new_indptr, total_new,
                                                          err_flag);
  return cudaGetLastError();
}

template <int F, bool HOOK>
static cudaError_t launch_baseline_attn_t(const CacheView &c, const Workspace &w,
                                          const uint16_t *q, int32_t *err_flag, cudaStream_t s) {
  static PerDevice grids;  // persistent grid per device
  int grid = 0;
  cudaError_t e = once_per_device(grids, [](int dev, int *g) {
    cudaError_t r = cudaFuncSetAttribute(baseline_attn_kernel<F, HOOK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kCtaSmem);
    int sms = 0, per_sm = 0;
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, baseline_attn_kernel<F, HOOK>,
                                                        kWarps * 32, kCtaSmem);
    *g = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  }, &grid);
  if (e != cudaSuccess) return e;
  baseline_attn_kernel<F, HOOK><<<grid, kWarps * 32, kCtaSmem, s>>>(c, w, q, err_flag);
  return cudaGetLastError();
}

cudaError_t launch_baseline_attention(int fmt, const CacheView &c, const Workspace &w,
                                      const uint16_t *q, int32_t *err_flag, cudaStream_t s) {
  if (w.fault_item >= 0)  // the testing hook is armed for this call
    return fmt == kFmtBf16 ? launch_baseline_attn_t<kFmtBf16, true>(c, w, q, err_flag, s)
                           : launch_baseline_attn_t<kFmtKv8, true>(c, w, q, err_flag, s);
  return fmt == kFmtBf16 ? launch_baseline_attn_t<kFmtBf16, false>(c, w, q, err_flag, s)
                         : launch_baseline_attn_t<kFmtKv8, false>(c, w, q, err_flag, s);
}

}  // namespace kv4
