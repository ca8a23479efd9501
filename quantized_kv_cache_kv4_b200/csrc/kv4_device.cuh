// Device-side building blocks shared by the kv4 kernels: shared-memory async bulk
// copies with mbarrier completion, warp-level tensor-core MMA and ldmatrix, and the
// nibble/byte -> fp16 unpack used on integer KV codes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/kv4.h"

namespace kv4 {

constexpr int kHeadDim = 128;
constexpr int kPage = 16;       // tokens per INT4 page and per INT8 tile
constexpr int kGroup = 32;      // INT4 group length along head_dim
constexpr int kMaxChunkPages = 64;  // INT4 pages per work entry (page ids in two registers)
constexpr int kMaxGqa = 8;      // query heads per kv head handled by one warp (MMA N = 8)
constexpr int kRecordFloats = kHeadDim + 4;  // partial record: acc[128], m, l, pad, pad

// Bytes of one (page, kv head) INT4 block and one (tile, kv head) INT8 block.
constexpr int kInt4CodeBytes = kPage * kHeadDim / 2;  // 1024
constexpr int kInt4ParamBytes = kPage * 4 * 2 * 2;    // 256: 16 slots x 4 groups x (scale,min)
constexpr int kInt8CodeBytes = kPage * kHeadDim;      // 2048
constexpr int kInt8ScaleBytes = kPage * 2;            // 32

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier + bulk async copy (global -> shared), completion counted in bytes
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One attempt; returns true once the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after `limit` attempts (each attempt itself blocks for a
// hardware-chosen interval). Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint32_t limit = (1u << 22)) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from global to
// this CTA's shared memory; completes `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Stores of partial records: written by the attention kernels and read back by the merge
// (with evict-first loads) right after, so they are stored with the L2 evict_last
// priority and stay in L2 while the pages stream past (measured: the call 1.5-2 us
// faster on every batch; an evict_first hint on the page copies was slower).
__device__ __forceinline__ uint64_t l2_keep_policy() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_rec(float *p, float v) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(l2_keep_policy())
               : "memory");
}
__device__ __forceinline__ void st_rec(float2 *p, float2 v) {
  asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v.x), "f"(v.y),
               "l"(l2_keep_policy())
               : "memory");
}
__device__ __forceinline__ void st_rec(float4 *p, float4 v) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w), "l"(l2_keep_policy())
               : "memory");
}

// ---------------------------------------------------------------------------
// warp-level tensor cores: D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col)
// Fragment ownership, lane = 4*gid + tig:
//   A: a01 = (row gid, k 2tig..+1), a23 = (row gid+8, k 2tig..+1),
//      a45 = (row gid, k 2tig+8..+9), a67 = (row gid+8, k 2tig+8..+9)
//   B: b01 = (k 2tig..+1, col gid), b23 = (k 2tig+8..+9, col gid)
//   C: c0,c1 = (row gid, col 2tig..+1), c2,c3 = (row gid+8, col 2tig..+1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a01, uint32_t a23, uint32_t a45,
                                        uint32_t a67, uint32_t b01, uint32_t b23) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a01), "r"(a23), "r"(a45), "r"(a67), "r"(b01), "r"(b23));
}

// D(16x8, s32) += A(16x32, u8, row) * B(32x8, s8 or u8, col). Fragments, lane = 4*gid+tig:
//   A: a0 = (row gid, k 4tig..+3), a1 = (row gid+8, k 4tig..+3),
//      a2 = (row gid, k 16+4tig..+3), a3 = (row gid+8, k 16+4tig..+3)
//   B: b0 = (k 4tig..+3, col gid), b1 = (k 16+4tig..+3, col gid); C as for mma_f16.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a01, uint32_t a23, uint32_t a45,
                                         uint32_t a67, uint32_t b01, uint32_t b23) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a01), "r"(a23), "r"(a45), "r"(a67), "r"(b01), "r"(b23));
}

__device__ __forceinline__ void mma_u8s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_s8s8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_s8u8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8u8(int32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// ---------------------------------------------------------------------------
// int8 code -> fp16 without conversion instructions.
// binary16 with exponent field 25 (bits 0x6400) is 1024 + mantissa, so OR-ing a small
// unsigned integer u <= 1023 into the mantissa gives exactly 1024 + u; subtracting
// 1024 (or 1024 + 128 for offset-binary int8) is exact.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t h2_sub(uint32_t x, uint32_t y) {
  __half2 r = __hsub2(*reinterpret_cast<__half2 *>(&x), *reinterpret_cast<__half2 *>(&y));
  return *reinterpret_cast<uint32_t *>(&r);
}

constexpr uint32_t kMagic1152x2 = 0x64806480u;  // (1152.0, 1152.0)

// V word from a transposed ldmatrix (token t0's nibbles d0..d3 in bits 0-15, token t1's
// in bits 16-31) as fp16 subnormals, without any conversion: a 16-bit half holding a
// nibble c in bits 0-3 (exponent field 0) is exactly c * 2^-24, one in bits 4-7 exactly
// 16c * 2^-24. So p[k] = (t0 dim k, t1 dim k) is a mask for k = 0, 1 and a shift and a
// mask for k = 2, 3; dims 1 and 3 carry an extra factor 16. The products with P' are
// exact in the fp32 accumulators; the factors 2^24 (dims 0, 2) and 2^20 (dims 1, 3) are
// applied once to the output.
constexpr float kSubUnscale = 16777216.0f;  // 2^24
constexpr float kSubUnscale16 = 1048576.0f;  // 2^20
__device__ __forceinline__ void nib_pairs_v_sub(uint32_t x, uint32_t (&p)[4]) {
  p[0] = x & 0x000F000Fu;
  p[1] = x & 0x00F000F0u;
  const uint32_t y = x >> 8;
  p[2] = y & 0x000F000Fu;
  p[3] = y & 0x00F000F0u;
}

// ---------------------------------------------------------------------------
// packed fp32 pairs (sm_100 f32x2 FMA pipe operations; each lane rounds to nearest-even
// exactly as the scalar operation does)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// Two int8 codes (bytes SEL0 and SEL1 of w) as an fp16 pair.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// sel picks [byte, 0x64, byte, 0x64] from (w ^ 0x80808080, 0x64646464)
template <uint32_t SEL>
__device__ __forceinline__ uint32_t s8_pair(uint32_t w_offset_binary) {
  return h2_sub(prmt(w_offset_binary, 0x64646464u, SEL), kMagic1152x2);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t x) {
  return __half22float2(*reinterpret_cast<__half2 *>(&x));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// fp16 round-to-nearest-even with saturation to +-65504.
__device__ __forceinline__ __half f16_sat(float x) {
  return __float2half_rn(fminf(fmaxf(x, -65504.0f), 65504.0f));
}

// The sequence and position of new-token row `row` of an append call: one row per
// sequence (indptr == nullptr: position L-1), or CSR ranges (the rows of sequence b are
// the last indptr[b+1]-indptr[b] positions before its length L). pos = -1 when the row
// lies outside every range.
__device__ __forceinline__ void locate_new_token(const int32_t *__restrict__ seq_lens,
                                                 int num_seqs,
                                                 const int32_t *__restrict__ indptr, int row,
                                                 int &b, int &pos, int &L) {
  if (indptr == nullptr) {
    b = row;
    L = seq_lens[b];
    pos = L - 1;
    return;
  }
  int lo = 0, hi = num_seqs - 1;  // largest b with indptr[b] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (indptr[mid] <= row) lo = mid; else hi = mid - 1;
  }
  b = lo;
  const int n = indptr[b + 1] - indptr[b];
  const int i = row - indptr[b];
  L = seq_lens[b];
  pos = (i >= 0 && i < n) ? L - n + i : -1;
}

// RN(a / b), the IEEE binary32 quotient, without a division, for a divisor b with at most
// 11 significant bits (an fp16 value, or the constants 15 and 127) and y = RN(1/b):
//   q0 = RN(a*y) lies within 2 ulp(a/b) of a/b (|b*y - 1| <= 2^-24);
//   r = a - q0*b is exact (a multiple of 2^(e_q + e_b - 34) below 2^14 of those units),
//   so the fma returns it exactly;
//   q0 + r*y = a/b + (a/b - q0)(b*y - 1) = a/b + delta with |delta| <= 2^-23 ulp(a/b),
//   and RN(q0 + r*y) is taken by the second fma in one rounding.
// RN(a/b + delta) = RN(a/b) unless a rounding midpoint lies between a/b and a/b + delta.
// a - m*b is a multiple of 2^(e_q + e_b - 34) for every midpoint m at a/b's exponent
// (b has <= 11 bits, m <= 25), so a nonzero distance |a/b - m| is at least 2^-12 ulp(a/b);
// and a/b = m exactly would need 25 significant bits in a. Hence the result is RN(a/b)
// (a/b and a in the normal range; tiny quotients only decide codes that are 0 either way).
// b = 0 with y = 0 gives 0.
__device__ __forceinline__ float quotient_rn(float a, float b, float y) {
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-q0, b, a);
  return __fmaf_rn(r, y, q0);
}
constexpr float kRcp15 = 1.0f / 15.0f;    // RN(1/15), folded by the compiler in binary32
constexpr float kRcp127 = 1.0f / 127.0f;  // RN(1/127)

__device__ __forceinline__ void set_err(int32_t *flag, uint32_t bit) {
  if (flag) atomicOr(reinterpret_cast<unsigned int *>(flag), bit);
}

}  // namespace kv4
