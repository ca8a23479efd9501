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
// One warp per (new token, kv head); lane i owns dims 4i..4i+3, so an INT4 group of 32
// dims is 8 lanes and its min/max is a 3-step shuffle reduction. The code decisions are
// taken in IEEE fp32 (__fsub_rn / __fdiv_rn / rintf = nearest-even) so they are unique
// and reproducible bit for bit; the quotients of the code decisions go through
// rint_quotient (a reciprocal multiply, with the IEEE division near half-integers).
#include "kv4_device.cuh"
#include "kv4_internal.h"

#ifndef KV4_APPEND_ROWS
#define KV4_APPEND_ROWS 4  // new-token rows per warp in bulk appends
#endif

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
      s8h = f16_sat(__fdiv_rn(amax, 127.0f));
      s8 = __half2float(s8h);
      const float r8 = s8 == 0.0f ? 0.0f : __frcp_rn(s8);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float qv = s8 == 0.0f ? 0.0f : rint_quotient(x[i], s8, r8);
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
    const __half scale_h = f16_sat(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
    const float minf = __half2float(min_h);
    const float sf = __half2float(scale_h);
    const float rf = sf == 0.0f ? 0.0f : __frcp_rn(sf);
    uint32_t code4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float q = sf == 0.0f ? 0.0f : rint_quotient(__fsub_rn(x[i], minf), sf, rf);
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

// One warp per (block of T consecutive new-token rows, kv head); the loads of all T rows
// are issued before the first is quantised. T = 1 for decode steps (one row per sequence).
template <int T>
__global__ void __launch_bounds__(256) append_kernel(CacheView c, const uint16_t *__restrict__ k_new,
                                                     const uint16_t *__restrict__ v_new,
                                                     const int32_t *__restrict__ new_indptr,
                                                     int32_t total_new, int32_t *err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int H = c.num_kv_heads;
  const int blocks = (total_new + T - 1) / T;
  if (warp >= blocks * H) return;
  const int h = warp % H;
  const int r0 = (warp / H) * T;
  uint2 kr[T], vr[T];
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int row = r0 + t;
    if (row < total_new) {
      const size_t rowoff = (static_cast<size_t>(row) * H + h) * kHeadDim + 4 * lane;
      kr[t] = *reinterpret_cast<const uint2 *>(k_new + rowoff);
      vr[t] = *reinterpret_cast<const uint2 *>(v_new + rowoff);
    }
  }
  int b = new_indptr ? find_seq_warp(new_indptr, c.num_seqs, r0, lane) : r0;
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int row = r0 + t;
    if (row >= total_new) break;
    int pos, L;
    if (new_indptr == nullptr) {
      b = row;
      L = c.seq_lens[b];
      pos = L - 1;
    } else {
      while (b + 1 < c.num_seqs && new_indptr[b + 1] <= row) ++b;  // next sequence's rows
      const int n = new_indptr[b + 1] - new_indptr[b];
      const int i = row - new_indptr[b];
      L = c.seq_lens[b];
      pos = (i >= 0 && i < n) ? L - n + i : -1;  // rows outside the CSR ranges are rejected
    }
    if (pos < 0 || pos >= L || L > c.max_pages * kPage) {
      if (lane == 0) set_err(err, KV4_DEVERR_SEQ_LEN);
      continue;
    }
    append_token(c, h, b, pos, L, kr[t], vr[t], lane, err);
  }
}

cudaError_t launch_append(const CacheView &c, const uint16_t *k_new, const uint16_t *v_new,
                          const int32_t *new_indptr, int32_t total_new, int32_t *err_flag,
                          cudaStream_t s) {
  if (total_new == 0) return cudaSuccess;
  const int threads = 256;
  // bulk appends (prefill): KV4_APPEND_ROWS rows per warp; decode-sized appends: one
  constexpr int TB = KV4_APPEND_ROWS;
  const bool bulk = new_indptr != nullptr && total_new >= TB * 148 * 64;
  const int T = bulk ? TB : 1;
  const long long warps = static_cast<long long>((total_new + T - 1) / T) * c.num_kv_heads;
  const unsigned blocks = static_cast<unsigned>((warps * 32 + threads - 1) / threads);
  if (bulk)
    append_kernel<TB><<<blocks, threads, 0, s>>>(c, k_new, v_new, new_indptr, total_new, err_flag);
  else
    append_kernel<1><<<blocks, threads, 0, s>>>(c, k_new, v_new, new_indptr, total_new, err_flag);
  return cudaGetLastError();
}

}  // namespace kv4
