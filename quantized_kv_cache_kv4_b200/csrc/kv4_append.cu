// Quantise-append: writes each new token's K/V into its INT4 page slot and, for
// protected positions, an INT8 copy into the sink set or the recent-window ring.
// Writing ring slot (p mod R) overwrites the INT8 copy of position p-R, which from then
// on is read from its INT4 copy: that is the demotion out of the recent window.
//
// KV4-RL pages: "keeps the whole context in paged INT4 and retains INT8 copies only for
// a fixed set of attention-sink and recent positions" (ai4snews summary,
// "Interpretation" para. 3); INT8 side cache (aimodeling article, "INT4 as the base").
//
// Demotion reading B (kv4_config.demotion = 1): the INT4 copy is quantised from the
// token's INT8 copy (code * scale) instead of its bf16 values, which is what demotion out
// of the recent window would write; the attention reads the same regions either way.
//
// Two kernels, the same arithmetic:
//   append_kernel       one warp per (new token, kv head); lane i owns dims 4i..4i+3, so an
//                       INT4 group of 32 dims is 8 lanes and its min/max a 3-step shuffle
//                       reduction. Used for one token per sequence (decode steps), where
//                       the launch, not the arithmetic, sets the time.
//   append_rows_kernel  bulk appends (CSR rows, e.g. prefill of prompts): one thread per
//                       (new token, kv head), a warp = 32 consecutive rows of one head.
//                       No shuffles; consecutive rows are consecutive page slots, so each
//                       16-byte code and parameter store of the warp lands in contiguous
//                       256-byte runs of a page block (full sectors).
// The code decisions are taken in IEEE fp32 (subtraction, division, nearest-even
// rounding) so they are unique and reproducible bit for bit; the correctly rounded
// quotients come from a reciprocal multiply and one fma correction (quotient_rn), exact
// for the fp16 scales.
#include "kv4_device.cuh"
#include "kv4_internal.h"
#include "kv4_plan.cuh"


namespace kv4 {

// The quantise-append of one token (sequence b, position pos of L) and kv head h; every
// lane holds 4 dims of the token's K (kraw) and V (vraw).
__device__ __forceinline__ void append_token(const CacheView &c, int h, int b, int pos, int L,
                                             uint2 kraw, uint2 vraw, int lane, int32_t *err) {
  const int H = c.num_kv_heads;
  const int page = c.page_table[static_cast<size_t>(b) * c.max_pages + pos / kPage];
  const bool page_ok = page >= 0 && page < c.num_pages;
  if (!page_ok && lane == 0) set_err(err, KV4_DEVERR_PAGE_ID);
  const int slot = pos % kPage;

  const int S = c.num_sinks, R = c.num_recent;
  int8_t *side_k = nullptr, *side_v = nullptr;
  uint16_t *side_ks = nullptr, *side_vs = nullptr;
  size_t tile_base = 0, scale_idx = 0;
  int side_slot = 0;
  if (pos < S) {
    const int set = c.sink_idx ? c.sink_idx[b] : b;
    if (set >= 0 && set < c.num_sink_sets) {
      const size_t sh = static_cast<size_t>(set) * H + h;
      tile_base = (sh * c.sink_tiles + pos / kPage) * kInt8CodeBytes;
      scale_idx = sh * c.sink_tiles * kPage + pos;
      side_k = c.sink_k; side_v = c.sink_v; side_ks = c.sink_ks; side_vs = c.sink_vs;
      side_slot = pos % kPage;
    } else if (lane == 0) {
      set_err(err, KV4_DEVERR_SIDE_IDX);
    }
  } else if (R > 0 && pos >= L - R) {
    const int ring = c.ring_idx ? c.ring_idx[b] : b;
    if (ring >= 0 && ring < c.num_rings) {
      const int rs = pos % R;
      const size_t rh = static_cast<size_t>(ring) * H + h;
      tile_base = (rh * c.ring_tiles + rs / kPage) * kInt8CodeBytes;
      scale_idx = rh * c.ring_tiles * kPage + rs;
      side_k = c.ring_k; side_v = c.ring_v; side_ks = c.ring_ks; side_vs = c.ring_vs;
      side_slot = rs % kPage;
    } else if (lane == 0) {
      set_err(err, KV4_DEVERR_SIDE_IDX);
    }
  }

#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const uint2 raw = which == 0 ? kraw : vraw;
    float x[4];
    x[0] = bf16_bits_to_f32(static_cast<uint16_t>(raw.x & 0xFFFFu));
    x[1] = bf16_bits_to_f32(static_cast<uint16_t>(raw.x >> 16));
    x[2] = bf16_bits_to_f32(static_cast<uint16_t>(raw.y & 0xFFFFu));
    x[3] = bf16_bits_to_f32(static_cast<uint16_t>(raw.y >> 16));

    // ---- INT8 (symmetric, per token and head): the protected copy, and in demotion
    // reading B also the values the INT4 copy is quantised from ----
    const bool need8 = side_k != nullptr || c.int4_from_int8;  // uniform over the warp
    float q8[4] = {0.f, 0.f, 0.f, 0.f};
    __half s8h = __float2half(0.f);
    float s8 = 0.f;
    if (need8) {
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
      for (int off = 1; off < 32; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      s8h = f16_sat(quotient_rn(amax, 127.0f, kRcp127));
      s8 = __half2float(s8h);
      const float r8 = s8 == 0.0f ? 0.0f : __frcp_rn(s8);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float qv = rintf(quotient_rn(x[i], s8, r8));  // r8 = 0 when s8 = 0: 0
        q8[i] = fminf(fmaxf(qv, -127.0f), 127.0f);
      }
    }
    if (c.int4_from_int8) {
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = q8[i] * s8;  // code * fp16 scale: exact in fp32
    }

    // ---- INT4: per 32-dim group (8 lanes), asymmetric, fp16 scale and min ----
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    const __half min_h = f16_sat(mn);
    const __half scale_h = f16_sat(quotient_rn(__fsub_rn(mx, mn), 15.0f, kRcp15));
    const float minf = __half2float(min_h);
    const float sf = __half2float(scale_h);
    const float rf = sf == 0.0f ? 0.0f : __frcp_rn(sf);
    uint32_t code4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float q = rintf(quotient_rn(__fsub_rn(x[i], minf), sf, rf));  // rf = 0 when sf = 0: 0
      code4[i] = static_cast<uint32_t>(fminf(fmaxf(q, 0.0f), 15.0f));
    }
    if (page_ok) {
      const int g = lane >> 3;
      const size_t blk = static_cast<size_t>(page) * H + h;
      uint8_t *codes = which == 0 ? c.k_codes : c.v_codes;
      uint16_t *params = which == 0 ? c.k_params : c.v_params;
      const uint16_t packed = static_cast<uint16_t>(code4[0] | (code4[1] << 4) | (code4[2] << 8) |
                                                    (code4[3] << 12));
      *reinterpret_cast<uint16_t *>(codes + (blk * 4 + g) * (kPage * 16) + slot * 16 +
                                    2 * (lane & 7)) = packed;
      if ((lane & 7) == 0) {
        const uint32_t pv = static_cast<uint32_t>(__half_as_ushort(scale_h)) |
                            (static_cast<uint32_t>(__half_as_ushort(min_h)) << 16);
        *reinterpret_cast<uint32_t *>(params + ((blk * kPage + slot) * 4 + g) * 2) = pv;
      }
    }

    // ---- INT8 copy of a protected position ----
    if (side_k != nullptr) {
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        word |= (static_cast<uint32_t>(static_cast<int32_t>(q8[i])) & 0xFFu) << (8 * i);
      int8_t *dst = (which == 0 ? side_k : side_v) + tile_base;
      // lane i holds dims 4i..4i+3: strip i/4, byte offset 4*(i%4)
      *reinterpret_cast<uint32_t *>(dst + (lane >> 2) * (kPage * 16) + side_slot * 16 +
                                    4 * (lane & 3)) = word;
      if (lane == 0) (which == 0 ? side_ks : side_vs)[scale_idx] = __half_as_ushort(s8h);
    }
  }
}

// Largest b in [0, num_seqs) with indptr[b] <= row, by the whole warp: each round the 32
// lanes probe 32 evenly spaced entries of the remaining range (ranges of 1M sequences
// resolve in 4 rounds of dependent loads instead of 20).
__device__ __forceinline__ int find_seq_warp(const int32_t *__restrict__ indptr, int num_seqs,
                                             int row, int lane) {
  int lo = 0, hi = num_seqs;  // indptr[lo] <= row holds throughout (indptr[0] = 0)
  while (hi - lo > 1) {
    const int step = (hi - lo + 31) / 32;
    const int idx = lo + lane * step;
    const bool le = idx < hi && indptr[idx] <= row;
    const int k = max(__popc(__ballot_sync(0xffffffffu, le)) - 1, 0);
    lo += k * step;
    hi = min(hi, lo + step);
  }
  return lo;
}

// Warp `warp` of the single-token append: (new token, kv head) = (warp / H, warp % H); the
// token's 256 bytes of K and of V are one coalesced load per warp.
__device__ __forceinline__ void append_warp(const CacheView &c, const uint16_t *__restrict__ k_new,
                                            const uint16_t *__restrict__ v_new,
                                            const int32_t *__restrict__ new_indptr,
                                            int32_t total_new, int32_t *err, int warp, int lane) {
  const int H = c.num_kv_heads;
  if (warp >= total_new * H) return;
  const int h = warp % H;
  const int row = warp / H;
  const size_t rowoff = (static_cast<size_t>(row) * H + h) * kHeadDim + 4 * lane;
  const uint2 kr = *reinterpret_cast<const uint2 *>(k_new + rowoff);
  const uint2 vr = *reinterpret_cast<const uint2 *>(v_new + rowoff);
  int b, pos, L;
  if (new_indptr == nullptr) {
    b = row;
    L = c.seq_lens[b];
    pos = L - 1;
  } else {
    b = find_seq_warp(new_indptr, c.num_seqs, row, lane);
    const int n = new_indptr[b + 1] - new_indptr[b];
    const int i = row - new_indptr[b];
    L = c.seq_lens[b];
    pos = (i >= 0 && i < n) ? L - n + i : -1;  // rows outside the CSR ranges are rejected
  }
  if (pos < 0 || pos >= L || L > c.max_pages * kPage) {
    if (lane == 0) set_err(err, KV4_DEVERR_SEQ_LEN);
    return;
  }
  append_token(c, h, b, pos, L, kr, vr, lane, err);
}

__global__ void __launch_bounds__(256) append_kernel(CacheView c, const uint16_t *__restrict__ k_new,
                                                     const uint16_t *__restrict__ v_new,
                                                     const int32_t *__restrict__ new_indptr,
                                                     int32_t total_new, int32_t *err) {
  append_warp(c, k_new, v_new, new_indptr, total_new, err,
              (blockIdx.x * blockDim.x + threadIdx.x) >> 5, threadIdx.x & 31);
}

// A decode step's two independent first launches as one: blocks [0, n_plan) build the
// work list (plan_block; it reads the lengths and page tables, which the append does not
// write), the blocks after them append one token per sequence, blockDim / 32 (token, kv
// head) warps per block. The block size is the plan's (32 to 1024 threads by batch size).
__global__ void __launch_bounds__(kPlanThreads) plan_append_kernel(
    CacheView c, Workspace w, const uint16_t *__restrict__ k_new,
    const uint16_t *__restrict__ v_new, int32_t *err, int n_plan) {
  if (static_cast<int>(blockIdx.x) < n_plan) {
    plan_block(c, w, err, blockIdx.x, n_plan);
    return;
  }
  const int warp = (static_cast<int>(blockIdx.x) - n_plan) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  append_warp(c, k_new, v_new, nullptr, c.num_seqs, err, warp, threadIdx.x & 31);
}

// ---------------------------------------------------------------------------
// bulk appends: one thread per (new token, kv head)
// ---------------------------------------------------------------------------
// y = v + 1.5*2^23 (|v| < 2^22) is rounded by the add to an integer in round-to-nearest-
// even, which y's low mantissa bits then hold: y_bits - 0x4B400000 (two's complement for
// negative integers, so the low byte of y_bits is an int8 code and the low nibble an
// INT4 code).
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

// rint(clamp(RN(a / b), lo, hi)) as y = result + 1.5*2^23 (see kRoundMagic); the integer
// bounds make clamping before rounding equal to rounding before clamping.
__device__ __forceinline__ uint32_t round_clamped(float a, float b, float y_rcp, float lo,
                                                  float hi) {
  const float q = fminf(fmaxf(quotient_rn(a, b, y_rcp), lo), hi);
  return __float_as_uint(__fadd_rn(q, kRoundMagic));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ __nv_bfloat162 bf2(uint32_t w) {
  return *reinterpret_cast<__nv_bfloat162 *>(&w);
}

// Byte 0 of each of four words, packed into one word (byte 0 = a's).
__device__ __forceinline__ uint32_t low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Where one row's INT4 record and (when protected) INT8 copy go.
struct RowDst {
  uint8_t *codes;    // the (page, head) code block: [4 groups][16 slots][16 B]
  uint16_t *params;  // the slot's [4 groups][scale, min]
  int slot;
  int8_t *side;      // INT8 tile (nullptr: not protected)
  uint16_t *side_scale;
  int side_slot;
};

// Staging of the rows in shared memory: per thread one row (256 B: its K row, then its V
// row) and 16 B of padding, then two mbarriers per warp. The thread stride of 272 B (68
// words = 4 mod 32) makes the 16-byte reads of 8 consecutive threads fall in distinct
// banks; 34 KB per block of 128 threads lets 6 blocks (24 warps) share an SM.
constexpr int kRowsThreads = 128;
constexpr int kRowStageStride = 272;
constexpr int kRowsSmem = kRowsThreads * kRowStageStride + (kRowsThreads / 32) * 16;

// The 16 words (dims 32g..32g+31, two per word) of group g of a staged row.
__device__ __forceinline__ void group_words(const uint8_t *row, int g, uint32_t (&w)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = *reinterpret_cast<const uint4 *>(row + 64 * g + 16 * i);
    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
}

// quotient_rn on a pair (nb = -b, y = RN(1/b) in both lanes), rounded to integers as
// y = RN(a/b) + 1.5*2^23: callers know every quotient lies where no clamp is needed.
__device__ __forceinline__ float2 round_quotient_pair(float2 a, float2 nb, float2 y) {
  const float2 q0 = fmul2(a, y);
  const float2 q = ffma2(ffma2(q0, nb, a), y, q0);
  return fadd2(q, make_float2(kRoundMagic, kRoundMagic));
}

// INT8 codes of one group (words w: dims 2i, 2i+1 in word i), packed 4 per word (dim
// 4j+i of the group in byte i of c8[j]); with FROM8 also the codes as floats (x8).
// fast: RN(amax / s8) < 127.5, so every code lies in [-127, 127] without the clamp.
template <bool FROM8>
__device__ __forceinline__ void int8_group(const uint32_t (&w)[16], float s8, float r8, bool fast,
                                           uint32_t (&c8)[8], float (&x8)[32]) {
  if (fast) {
    const float2 nb = make_float2(-s8, -s8), yr = make_float2(r8, r8);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 y0 =
          round_quotient_pair(make_float2(bf16_lo(w[2 * j]), bf16_hi(w[2 * j])), nb, yr);
      const float2 y1 = round_quotient_pair(
          make_float2(bf16_lo(w[2 * j + 1]), bf16_hi(w[2 * j + 1])), nb, yr);
      c8[j] = low_bytes(__float_as_uint(y0.x), __float_as_uint(y0.y), __float_as_uint(y1.x),
                        __float_as_uint(y1.y));
      if (FROM8) {
        x8[4 * j] = y0.x - kRoundMagic;
        x8[4 * j + 1] = y0.y - kRoundMagic;
        x8[4 * j + 2] = y1.x - kRoundMagic;
        x8[4 * j + 3] = y1.y - kRoundMagic;
      }
    }
  } else {  // a saturated fp16 scale: clamp every code
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t y[4] = {round_clamped(bf16_lo(w[2 * j]), s8, r8, -127.f, 127.f),
                             round_clamped(bf16_hi(w[2 * j]), s8, r8, -127.f, 127.f),
                             round_clamped(bf16_lo(w[2 * j + 1]), s8, r8, -127.f, 127.f),
                             round_clamped(bf16_hi(w[2 * j + 1]), s8, r8, -127.f, 127.f)};
      c8[j] = low_bytes(y[0], y[1], y[2], y[3]);
      if (FROM8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) x8[4 * j + i] = __uint_as_float(y[i]) - kRoundMagic;
      }
    }
  }
}

// Quantise one staged row (one new token and kv head, 128 bf16 values) into its INT4
// record and, when protected, its INT8 copy. FROM8: demotion reading B (the INT4 copy
// quantised from the INT8 copy). The group loop is not unrolled: the code stays small
// enough for the instruction cache. next (or nullptr): the global row staged into this
// slot next; each of its groups is requested as soon as this row's group has been used.
template <bool FROM8>
__device__ __forceinline__ void quantize_row(uint8_t *row, const RowDst &d,
                                             const uint8_t *next, uint64_t *next_bar) {
  const bool need8 = FROM8 || d.side != nullptr;
  float s8 = 0.f, r8 = 0.f;
  uint16_t s8_bits = 0;
  bool fast8 = false;
  if (need8) {  // symmetric INT8: amax over the 128 dims (|x| of bf16 = clear the sign bit)
    __nv_bfloat162 m2 = bf2(0u);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint4 v = *reinterpret_cast<const uint4 *>(row + 16 * i);
      m2 = __hmax2(m2, bf2(v.x & 0x7FFF7FFFu));
      m2 = __hmax2(m2, bf2(v.y & 0x7FFF7FFFu));
      m2 = __hmax2(m2, bf2(v.z & 0x7FFF7FFFu));
      m2 = __hmax2(m2, bf2(v.w & 0x7FFF7FFFu));
    }
    const float amax = fmaxf(__low2float(m2), __high2float(m2));
    const __half s8h = f16_sat(quotient_rn(amax, 127.0f, kRcp127));
    s8_bits = __half_as_ushort(s8h);
    s8 = __half2float(s8h);
    r8 = s8 == 0.0f ? 0.0f : __frcp_rn(s8);
    fast8 = quotient_rn(amax, s8, r8) < 127.5f;  // |x| <= amax: every quotient below it
  }
  uint32_t pv[4];
#pragma unroll 1
  for (int g = 0; g < 4; ++g) {
    uint32_t w[16];
    group_words(row, g, w);
    uint32_t c8[8];
    float x8[32];  // FROM8: the group's INT8 codes; the INT4 copy is quantised from x8 * s8
    if (need8) {
      int8_group<FROM8>(w, s8, r8, fast8, c8, x8);
      if (d.side != nullptr) {  // strips 2g, 2g+1 (16 dims each) of the INT8 tile
        int8_t *dst = d.side + 2 * g * (kPage * 16) + d.side_slot * 16;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(c8[0], c8[1], c8[2], c8[3]);
        *reinterpret_cast<uint4 *>(dst + kPage * 16) = make_uint4(c8[4], c8[5], c8[6], c8[7]);
      }
    }
    // ---- INT4 group: min/max, fp16 scale and min, codes ----
    auto xval = [&](int k) {  // dim 32g+k of the values the INT4 copy is quantised from
      if (FROM8) return x8[k] * s8;  // INT8 code * fp16 scale: exact in fp32
      return (k & 1) ? bf16_hi(w[k >> 1]) : bf16_lo(w[k >> 1]);
    };
    float mn, mx;
    if (FROM8) {
      mn = mx = xval(0);
#pragma unroll
      for (int k = 1; k < 32; ++k) {
        mn = fminf(mn, xval(k));
        mx = fmaxf(mx, xval(k));
      }
    } else {  // bf16 min/max are exact: pairwise on bf16x2, then the two halves
      __nv_bfloat162 lo2 = bf2(w[0]), hi2 = lo2;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        lo2 = __hmin2(lo2, bf2(w[i]));
        hi2 = __hmax2(hi2, bf2(w[i]));
      }
      mn = fminf(__low2float(lo2), __high2float(lo2));
      mx = fmaxf(__low2float(hi2), __high2float(hi2));
    }
    const __half min_h = f16_sat(mn);
    const __half scale_h = f16_sat(quotient_rn(__fsub_rn(mx, mn), 15.0f, kRcp15));
    const float minf = __half2float(min_h);
    const float sf = __half2float(scale_h);
    const float rf = sf == 0.0f ? 0.0f : __frcp_rn(sf);  // scale 0: every quotient 0
    // RN(RN(x - min) / scale) is monotone in x, so the group's quotients lie between
    // those of mn and mx; within [-1/2, 15.5) they round into [0, 15] without the clamp
    const bool fast = quotient_rn(__fsub_rn(mn, minf), sf, rf) >= -0.5f &&
                      quotient_rn(__fsub_rn(mx, minf), sf, rf) < 15.5f;
    // byte i of the group's 16 = code(2i) | code(2i+1) << 4. A rounded y's low nibble is
    // the code and its next 4 bits are zero, so y_even + (y_odd << 4) has the byte in
    // its low 8 bits.
    uint32_t words[4];
    if (fast) {
      const float2 m2 = make_float2(minf, minf), nb = make_float2(-sf, -sf);
      const float2 yr = make_float2(rf, rf);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = 8 * j + 2 * i;
          const float2 y =
              round_quotient_pair(fsub2(make_float2(xval(k), xval(k + 1)), m2), nb, yr);
          pb[i] = __float_as_uint(y.x) + (__float_as_uint(y.y) << 4);
        }
        words[j] = low_bytes(pb[0], pb[1], pb[2], pb[3]);
      }
    } else {  // a min far from the group (|min| >> range) or a saturated scale: clamp
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = 8 * j + 2 * i;
          pb[i] = round_clamped(__fsub_rn(xval(k), minf), sf, rf, 0.f, 15.f) +
                  (round_clamped(__fsub_rn(xval(k + 1), minf), sf, rf, 0.f, 15.f) << 4);
        }
        words[j] = low_bytes(pb[0], pb[1], pb[2], pb[3]);
      }
    }
    if (d.codes != nullptr)
      *reinterpret_cast<uint4 *>(d.codes + g * (kPage * 16) + d.slot * 16) =
          make_uint4(words[0], words[1], words[2], words[3]);
    pv[g] = static_cast<uint32_t>(__half_as_ushort(scale_h)) |
            (static_cast<uint32_t>(__half_as_ushort(min_h)) << 16);
    if (next != nullptr) {  // group g of this slot is consumed: fetch the next row's
      fence_proxy_async_smem();  // the reads above come before the async write
      bulk_g2s(row + 64 * g, next + 64 * g, 64, next_bar);
    }
  }
  if (d.codes != nullptr)
    *reinterpret_cast<uint4 *>(d.params) = make_uint4(pv[0], pv[1], pv[2], pv[3]);
  if (d.side != nullptr) *d.side_scale = s8_bits;
}


// A warp = 32 consecutive CSR rows (lane = row) of one kv head; consecutive warps are
// the heads of the same rows, so the rows' lookups hit the same L1 lines. Each thread
// first stages its row's K (256 B) into shared memory with one bulk copy (TMA engine,
// completion on the warp's mbarrier) and prefetches its V into L2, then finds where the
// row goes while they land; V is staged into the same slot, group by group, as K's
// groups are consumed (a second mbarrier). One bulk copy per row instead of sixteen
// 16-byte copies keeps the memory-instruction queue free for the arithmetic.
template <bool FROM8>
__global__ void __launch_bounds__(kRowsThreads) append_rows_kernel(CacheView c,
                                                         const uint16_t *__restrict__ k_new,
                                                         const uint16_t *__restrict__ v_new,
                                                         const int32_t *__restrict__ new_indptr,
                                                         int32_t total_new, int32_t *err) {
  extern __shared__ __align__(16) uint8_t rows_smem[];
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int H = c.num_kv_heads;
  const int tiles = (total_new + 31) / 32;
  if (warp >= tiles * H) return;  // whole warps
  const int h = warp % H;
  const int r0 = (warp / H) * 32;
  const int row = r0 + lane;
  bool live = row < total_new;

  uint8_t *stage = rows_smem + threadIdx.x * kRowStageStride;
  uint64_t *bars = reinterpret_cast<uint64_t *>(rows_smem + kRowsThreads * kRowStageStride) +
                   2 * (threadIdx.x >> 5);  // this warp's: K rows, V rows
  const size_t rowoff = (static_cast<size_t>(live ? row : r0) * H + h) * kHeadDim;
  const int n_k = __popc(__ballot_sync(0xffffffffu, live));
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(&bars[0], n_k * 256u);
  }
  __syncwarp();
  if (live) {  // one bulk copy per K row; V is prefetched into L2 and staged after K
    const uint8_t *vs = reinterpret_cast<const uint8_t *>(v_new + rowoff);
    bulk_g2s(stage, k_new + rowoff, 256, &bars[0]);
    asm volatile("prefetch.global.L2 [%0];" ::"l"(vs));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(vs + 128));
  }

  // the row's sequence: the warp finds the first row's sequence b0, then reads the CSR
  // offsets, lengths and side-set indices of sequences b0 .. b0+31 in one round, and each
  // lane picks its own sequence from them by a shuffle search (largest j with
  // indptr[b0 + j] <= row)
  const int B = c.num_seqs;
  const int b0 = find_seq_warp(new_indptr, B, r0, lane);
  const int wb = min(b0 + lane, B);
  const int w_off = new_indptr[wb];
  const int w_end = new_indptr[min(b0 + 32, B)];
  const bool w_ok = b0 + lane < B;
  const int w_len = w_ok ? c.seq_lens[wb] : 0;
  const int w_sink = (w_ok && c.sink_idx) ? c.sink_idx[wb] : wb;
  const int w_ring = (w_ok && c.ring_idx) ? c.ring_idx[wb] : wb;
  int j = 0;
#pragma unroll
  for (int step = 16; step; step >>= 1)
    if (__shfl_sync(0xffffffffu, w_off, j + step) <= row) j += step;
  // every lane takes part in every shuffle (none sits inside a conditional expression)
  const int off_b = __shfl_sync(0xffffffffu, w_off, j);
  const int off_after = __shfl_sync(0xffffffffu, w_off, min(j + 1, 31));
  const int off_next = j == 31 ? w_end : off_after;
  int b = b0 + j;
  int L = __shfl_sync(0xffffffffu, w_len, j);
  int sink_set = __shfl_sync(0xffffffffu, w_sink, j);
  int ring_id = __shfl_sync(0xffffffffu, w_ring, j);
  int n = off_next - off_b, first = off_b;
  if (live && j == 31 && w_end <= row && b0 + 32 < B) {
    // rare: the row's sequence lies beyond the window (more than 32 sequences start in
    // these 32 rows, i.e. empty ones): per-lane binary search
    int lo = b0 + 32, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (new_indptr[mid] <= row) lo = mid; else hi = mid - 1;
    }
    b = lo;
    first = new_indptr[b];
    n = new_indptr[b + 1] - first;
    L = c.seq_lens[b];
    sink_set = c.sink_idx ? c.sink_idx[b] : b;
    ring_id = c.ring_idx ? c.ring_idx[b] : b;
  }
  int pos = -1;
  if (live) {
    const int i = row - first;
    pos = (b < B && i >= 0 && i < n) ? L - n + i : -1;  // rows outside the CSR ranges
    if (pos < 0 || pos >= L || L > c.max_pages * kPage) {
      set_err(err, KV4_DEVERR_SEQ_LEN);
      live = false;
    }
  }
  RowDst dk{}, dv{};
  if (live) {
    const int page = c.page_table[static_cast<size_t>(b) * c.max_pages + pos / kPage];
    if (page >= 0 && page < c.num_pages) {
      const size_t blk = static_cast<size_t>(page) * H + h;
      dk.codes = c.k_codes + blk * 4 * (kPage * 16);
      dv.codes = c.v_codes + blk * 4 * (kPage * 16);
      dk.params = c.k_params + (blk * kPage + pos % kPage) * 8;
      dv.params = c.v_params + (blk * kPage + pos % kPage) * 8;
    } else {
      set_err(err, KV4_DEVERR_PAGE_ID);
    }
    dk.slot = dv.slot = pos % kPage;
    const int S = c.num_sinks, R = c.num_recent;
    if (pos < S) {
      const int set = sink_set;
      if (set >= 0 && set < c.num_sink_sets) {
        const size_t sh = static_cast<size_t>(set) * H + h;
        const size_t tile = (sh * c.sink_tiles + pos / kPage) * kInt8CodeBytes;
        const size_t sidx = sh * c.sink_tiles * kPage + pos;
        dk.side = c.sink_k + tile; dk.side_scale = c.sink_ks + sidx;
        dv.side = c.sink_v + tile; dv.side_scale = c.sink_vs + sidx;
        dk.side_slot = dv.side_slot = pos % kPage;
      } else {
        set_err(err, KV4_DEVERR_SIDE_IDX);
      }
    } else if (R > 0 && pos >= L - R) {
      const int ring = ring_id;
      if (ring >= 0 && ring < c.num_rings) {
        const int rs = pos % R;
        const size_t rh = static_cast<size_t>(ring) * H + h;
        const size_t tile = (rh * c.ring_tiles + rs / kPage) * kInt8CodeBytes;
        const size_t sidx = rh * c.ring_tiles * kPage + rs;
        dk.side = c.ring_k + tile; dk.side_scale = c.ring_ks + sidx;
        dv.side = c.ring_v + tile; dv.side_scale = c.ring_vs + sidx;
        dk.side_slot = dv.side_slot = rs % kPage;
      } else {
        set_err(err, KV4_DEVERR_SIDE_IDX);
      }
    }
  }
  // the V rows the warp will stage: those still live after the lookups
  const int n_v = __popc(__ballot_sync(0xffffffffu, live));
  if (lane == 0) mbar_arrive_expect_tx(&bars[1], n_v * 256u);
  // every lane waits for the warp's K copies (none may exit with one in flight); the
  // waits are bounded, and a wait that gives up waits once more before returning
  if (!mbar_wait_bounded(&bars[0], 0)) {
    if (lane == 0) set_err(err, KV4_DEVERR_TIMEOUT);
    mbar_wait_bounded(&bars[0], 0);
    return;
  }
  if (!live) return;
  quantize_row<FROM8>(stage, dk, reinterpret_cast<const uint8_t *>(v_new + rowoff), &bars[1]);
  if (!mbar_wait_bounded(&bars[1], 0)) {
    set_err(err, KV4_DEVERR_TIMEOUT);
    mbar_wait_bounded(&bars[1], 0);
    return;
  }
  quantize_row<FROM8>(stage, dv, nullptr, nullptr);
}

cudaError_t launch_append(const CacheView &c, const uint16_t *k_new, const uint16_t *v_new,
                          const int32_t *new_indptr, int32_t total_new, int32_t *err_flag,
                          cudaStream_t s) {
  if (total_new == 0) return cudaSuccess;
  const int threads = 256;
  if (new_indptr != nullptr) {  // CSR rows: one thread per (row, kv head)
    static PerDevice configured;
    int done = 0;
    cudaError_t e = once_per_device(configured, [](int, int *v) {
      cudaError_t r = cudaFuncSetAttribute(append_rows_kernel<false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kRowsSmem);
      if (r == cudaSuccess)
        r = cudaFuncSetAttribute(append_rows_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kRowsSmem);
      *v = 1;
      return r;
    }, &done);
    if (e != cudaSuccess) return e;
    const long long warps = static_cast<long long>((total_new + 31) / 32) * c.num_kv_heads;
    const unsigned blocks =
        static_cast<unsigned>((warps * 32 + kRowsThreads - 1) / kRowsThreads);
    if (c.int4_from_int8)
      append_rows_kernel<true><<<blocks, kRowsThreads, kRowsSmem, s>>>(c, k_new, v_new, new_indptr,
                                                                       total_new, err_flag);
    else
      append_rows_kernel<false><<<blocks, kRowsThreads, kRowsSmem, s>>>(c, k_new, v_new, new_indptr,
                                                                        total_new, err_flag);
  } else {  // one token per sequence: one warp per (token, kv head)
    const long long warps = static_cast<long long>(total_new) * c.num_kv_heads;
    const unsigned blocks = static_cast<unsigned>((warps * 32 + threads - 1) / threads);
    append_kernel<<<blocks, threads, 0, s>>>(c, k_new, v_new, new_indptr, total_new, err_flag);
  }
  return cudaGetLastError();
}

cudaError_t launch_plan_append(const CacheView &c, const Workspace &w, const uint16_t *k_new,
                               const uint16_t *v_new, int32_t *err_flag, cudaStream_t s) {
  int n_plan = 0, threads = 0;
  plan_shape(c.num_seqs, &n_plan, &threads);
  const long long warps = static_cast<long long>(c.num_seqs) * c.num_kv_heads;
  const long long per_block = threads / 32;
  const unsigned blocks = static_cast<unsigned>(n_plan + (warps + per_block - 1) / per_block);
  plan_append_kernel<<<blocks, threads, 0, s>>>(c, w, k_new, v_new, err_flag, n_plan);
  return cudaGetLastError();
}

}  // namespace kv4
