// The plan of a decode-attention call: the work list (entries in classes, unit offsets of
// the partial records, the shared-prefix groups and the list's signature) built on the
// device from the sequence lengths and, for the shared-prefix read, the page tables.
// Included by the attention translation unit (plan_kernel) and the append one (the fused
// plan-and-append kernel of a decode step), so every function here is inline.
#pragma once

#include <climits>

#include "kv4_attn_common.cuh"

namespace kv4 {

// ---------------------------------------------------------------------------
// plan: a few CTAs of 1024 threads. Every CTA scans all sequences (a few KB of lengths)
// to get the same offsets, then writes the entries of its own slice of sequences only,
// so the scattered 16-byte entry stores are spread over several SMs.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kPlanSeqsPerCta = 32;  // sequences per CTA, until kPlanMaxCtas is reached
constexpr int kPlanMaxCtas = 148;
constexpr int kScanN = 6;            // values scanned together per sequence
constexpr int kPrefixCols = 16;      // query columns of one prefix entry (two MMA N tiles)
constexpr int kMaxPrefixPages = 256;  // leading INT4 pages compared for sharing

// The plan's launch shape for a batch: one CTA per kPlanSeqsPerCta sequences (at most
// kPlanMaxCtas) and, for small batches, fewer threads (the scans and barriers span only
// the warps in use).
inline void plan_shape(int num_seqs, int *ctas, int *threads) {
  *ctas = max(1, min(kPlanMaxCtas, (num_seqs + kPlanSeqsPerCta - 1) / kPlanSeqsPerCta));
  *threads = min(kPlanThreads, max(32, (num_seqs + 31) / 32 * 32));
}

// Exclusive block-wide scan of kScanN values at once (warp shuffles + one warp per value
// over the warp totals); totals returned in tot. Blocks of 32 to 1024 threads.
__device__ inline void block_scan_n(int (&v)[kScanN], int (&tot)[kScanN], int (*warp_sums)[32]) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x[kScanN];
#pragma unroll
  for (int i = 0; i < kScanN; ++i) {
    x[i] = v[i];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x[i], off);
      if (lane >= off) x[i] += y;
    }
    if (lane == 31) warp_sums[i][wid] = x[i];
  }
  __syncthreads();
  for (int i = wid; i < kScanN; i += nw) {
    int t = lane < nw ? warp_sums[i][lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t += y;
    }
    warp_sums[i][lane] = t;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kScanN; ++i) {
    const int base = wid ? warp_sums[i][wid - 1] : 0;
    tot[i] = warp_sums[i][31];
    v[i] = base + x[i] - v[i];
  }
  __syncthreads();
}

// Ranks of the threads' keys within one block of 1024 sequences, stable in sequence
// order: rank = earlier threads with the same key. Keys are in [0, 32) or -1 (none).
// cnt: shared scratch; chunk_tot[k] receives the block's count of key k.
__device__ inline int key_rank(int key, int (*cnt)[33], int *chunk_tot) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 32 * 33; i += blockDim.x) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const unsigned same = __match_any_sync(0xffffffffu, key);
  const int lr = __popc(same & ((1u << lane) - 1u));
  if (key >= 0 && lr == 0) cnt[key][wid] = __popc(same);
  __syncthreads();
  if (threadIdx.x < 32) {  // per key: exclusive scan over the 32 warps
    int sum = 0;
    for (int wi = 0; wi < 32; ++wi) {
      const int v = cnt[threadIdx.x][wi];
      cnt[threadIdx.x][wi] = sum;
      sum += v;
    }
    chunk_tot[threadIdx.x] = sum;
  }
  __syncthreads();
  const int rank = key >= 0 ? cnt[key][wid] + lr : 0;
  __syncthreads();
  return rank;
}

// Inclusive block-wide max-scan of v (32 to 1024 threads); warp_max: shared scratch [32].
__device__ inline int block_max_scan(int v, int *warp_max) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v = max(v, y);
  }
  if (lane == 31) warp_max[wid] = v;
  __syncthreads();
  if (wid == 0) {
    int t = lane < nw ? warp_max[lane] : INT_MIN;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t = max(t, y);
    }
    warp_max[lane] = t;
  }
  __syncthreads();
  if (wid > 0) v = max(v, warp_max[wid - 1]);
  __syncthreads();
  return v;
}

// Pages at the head of sequence b's INT4 range that hold the same physical pages as in
// sequence b-1's page table: returns p0 plus the number of equal page ids from page p0 on,
// compared over the pages holding positions of both sequences (at most kMaxPrefixPages).
__device__ inline int pages_shared_with_prev(const CacheView &c, int b, int p0) {
  const int cap = c.max_pages * kPage;
  int L1 = c.seq_lens[b], L0 = c.seq_lens[b - 1];
  if (L1 < 0 || L1 > cap) L1 = 0;
  if (L0 < 0 || L0 > cap) L0 = 0;
  const int np = min((min(L1, L0) + kPage - 1) / kPage, p0 + kMaxPrefixPages);
  const int32_t *r1 = c.page_table + static_cast<size_t>(b) * c.max_pages;
  const int32_t *r0 = r1 - c.max_pages;
  // eight pages per round, their loads issued together (one memory latency per round)
  for (int k = p0; k < np; k += 8) {
    int a[8], z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool in = k + i < np;
      a[i] = in ? r1[k + i] : 0;
      z[i] = in ? r0[k + i] : 1;
    }
    int first = 8;
#pragma unroll
    for (int i = 7; i >= 0; --i)
      if (a[i] != z[i]) first = i;
    if (first < 8) return k + first;
  }
  return max(p0, np);
}

struct PrefixRun {
  int pe = 0;    // end page of the group's shared INT4 pages (0: not in a group)
  int nmem = 0;  // members of the prefix entry this sequence leads (0: it leads none)
};

// Groups of the sequences base .. base+1023 (one per thread): maximal runs of consecutive
// sequences each sharing at least one INT4 page with its predecessor (the run's first
// sequence, or the block's first, starts it). The group's shared pages are [S/16, pe) with
// pe the smallest shared count of its members; groups of one sequence read nothing
// together. Members are taken kPrefixCols / G at a time into prefix entries. All threads
// of the block call this together (it synchronises the block).
__device__ inline PrefixRun prefix_runs(const CacheView &c, const Workspace &w, int base, int *run_min,
                                 int *run_len, int *warp_max) {
  const int t = threadIdx.x, b = base + t;
  const int p0 = c.num_sinks / kPage;
  int k = 0;
  bool share = false;
  if (b < c.num_seqs && t > 0) {
    k = pages_shared_with_prev(c, b, p0);
    share = k > p0;
  }
  const int lead = block_max_scan(share ? -1 : t, warp_max);
  run_min[t] = 0x7fffffff;
  run_len[t] = 0;
  __syncthreads();
  if (b < c.num_seqs) {
    atomicAdd(&run_len[lead], 1);
    if (share) atomicMin(&run_min[lead], k);
  }
  __syncthreads();
  PrefixRun pr;
  if (b < c.num_seqs) {
    const int n = run_len[lead];
    if (n >= 2) {
      pr.pe = run_min[lead];
      const int pos = t - lead;
      const int M = max(1, kPrefixCols / c.gqa);
      if (pos % M == 0) pr.nmem = min(M, n - pos);
    }
  }
  __syncthreads();
  return pr;
}

struct SeqPlan {
  Regions g;
  PrefixRun pr;
  int pages;   // pages of the sequence's own INT4 chunks
  int nfull;   // own INT4 chunks of exactly chunk_pages pages
  int key = -1;  // short last chunk: 31 - its pages (sort key), else -1
  bool last_long;  // the shorter last chunk (if any) has at least half the pages
  // scanned values: regions (protected set, shared-prefix regions, own INT4 chunks), then
  // entries per class: full chunks, long partial chunks, protected sets, short chunks (the
  // attention kernel's), then shared-prefix chunks (led by the first member of each prefix
  // entry; the prefix kernel's, at the end of the list)
  int n[kScanN];
};

// The plan of one CTA, `cta` of `nctas`: each CTA scans all sequences and writes the work
// entries of its own slice of them. Run by plan_kernel and, in a decode step, by the plan
// blocks of the fused plan-and-append kernel.
__device__ inline void plan_block(const CacheView &c, const Workspace &w, int32_t *err, int cta,
                                  int nctas) {
  __shared__ int warp_sums[kScanN][32];
  // the short class is ordered by decreasing chunk length (key = 31 - pages), so that
  // the last entries of the kernel are the shortest
  __shared__ int key_cnt[32][33];
  __shared__ int key_chunk[32], key_tot[32], key_run[32];
  __shared__ int run_min[kPlanThreads], run_len[kPlanThreads], warp_max[32];
  const bool prefix = w.prefix_end != nullptr;
  const int B = c.num_seqs, H = c.num_kv_heads, C = w.chunk_pages;
  const int S = c.num_sinks, R = c.num_recent;
  const int hpw = w.heads_per_warp;
  const int nslots = (H + hpw - 1) / hpw;
  const int per = (B + nctas - 1) / nctas;  // sequences written by this CTA
  const int my_lo = cta * per;
  const int my_hi = min(B, my_lo + per);

  auto plan_of = [&](int b, const PrefixRun &pr) {
    SeqPlan sp{};
    if (b >= B) return sp;
    int L = c.seq_lens[b];
    if (L < 0 || L > c.max_pages * kPage) {
      if (b >= my_lo && b < my_hi) set_err(err, KV4_DEVERR_SEQ_LEN);
      L = 0;
    }
    sp.pr = pr;
    sp.g = regions_of(L, S, R, C, pr.pe);
    sp.pages = sp.g.n_chunks ? (sp.g.int4_hi - 1) / kPage - sp.g.first_page + 1 : 0;
    sp.nfull = sp.pages / C;
    const bool has_last = sp.g.n_chunks > sp.nfull;
    sp.last_long = 2 * (sp.pages - sp.nfull * C) >= C;
    sp.n[0] = sp.g.has_prot + sp.g.n_prompt + sp.g.n_chunks;
    sp.n[1] = sp.nfull * nslots;
    sp.n[2] = has_last && sp.last_long ? nslots : 0;
    sp.n[3] = sp.g.has_prot * nslots;
    sp.n[4] = has_last && !sp.last_long ? nslots : 0;
    sp.n[5] = pr.nmem ? sp.g.n_prompt * H : 0;
    sp.key = sp.n[4] ? 31 - (sp.pages - sp.nfull * C) : -1;
    return sp;
  };
  auto runs_of = [&](int base) {
    return prefix ? prefix_runs(c, w, base, run_min, run_len, warp_max) : PrefixRun{};
  };

  // pass 1: totals over every sequence. A batch of at most one block of sequences is
  // one block-wide pass, whose exclusive offsets and key ranks are kept for pass 2.
  // Blocks have min(1024, num_seqs rounded up to a warp) threads.
  const int T = blockDim.x;
  const bool single = B <= T;
  int tot[kScanN] = {0, 0, 0, 0, 0, 0};
  SeqPlan keep{};
  int keep_off[kScanN] = {0, 0, 0, 0, 0, 0};
  int keep_rank = 0;
  if (threadIdx.x < 32) key_tot[threadIdx.x] = 0;
  for (int base = 0; base < B; base += T) {
    SeqPlan sp = plan_of(base + threadIdx.x, runs_of(base));
    int off[kScanN], t[kScanN];
#pragma unroll
    for (int i = 0; i < kScanN; ++i) off[i] = sp.n[i];
    block_scan_n(off, t, warp_sums);
#pragma unroll
    for (int i = 0; i < kScanN; ++i) tot[i] += t[i];
    const int krank = key_rank(sp.key, key_cnt, key_chunk);
    if (threadIdx.x < 32) key_tot[threadIdx.x] += key_chunk[threadIdx.x];
    if (single) {
      keep = sp;
#pragma unroll
      for (int i = 0; i < kScanN; ++i) keep_off[i] = off[i];
      keep_rank = krank;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // first rank of every key: exclusive scan over the keys
    int sum = 0;
    for (int k = 0; k < 32; ++k) {
      key_run[k] = sum;
      sum += key_tot[k];
    }
  }
  __syncthreads();
  const int te_all = tot[1] + tot[2] + tot[3] + tot[4] + tot[5];
  const bool fits = tot[0] <= w.cap_pairs && te_all <= w.cap_entries;

  // pass 2: offsets up to this CTA's slice; entries of the slice (every unit empty if
  // the workspace is too small)
  // class bases: full chunks at 0, then long partial chunks, protected sets, short chunks
  int class_base[kScanN] = {0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int i = 2; i < kScanN; ++i) class_base[i] = class_base[i - 1] + tot[i - 1];
  auto write_seq = [&](int b, const SeqPlan &sp, const int (&off)[kScanN], int short_rank) {
    const int pairs = sp.n[0];
    for (int h = 0; h < H; ++h) w.unit_offsets[b * H + h] = H * off[0] + h * pairs;
    if (prefix) w.prefix_end[b] = sp.pr.pe;
    if (pairs == 0) return;
    const Regions &g = sp.g;
    int ef = off[1], el = off[2], epr = off[3], ep = off[5];
    const int es = class_base[4] + short_rank * nslots;
    const int own = g.has_prot + g.n_prompt;  // region index of the first own chunk
    if (g.has_prot)
      for (int s = 0; s < nslots; ++s)
        w.entries[epr++] = make_int4(b, 0, s * hpw, min(hpw, H - s * hpw));
    // this sequence leads a prefix entry: one per prompt chunk ci and kv head, encoded
    // with region -1 - ci and the member count in place of the head count
    if (sp.n[5])
      for (int ci = 0; ci < g.n_prompt; ++ci)
        for (int h = 0; h < H; ++h) w.entries[ep++] = make_int4(b, -1 - ci, h, sp.pr.nmem);
    for (int ch = 0; ch < sp.nfull; ++ch)
      for (int s = 0; s < nslots; ++s)
        w.entries[ef++] = make_int4(b, own + ch, s * hpw, min(hpw, H - s * hpw));
    if (g.n_chunks > sp.nfull) {
      int e = sp.last_long ? el : es;
      for (int s = 0; s < nslots; ++s)
        w.entries[e++] = make_int4(b, own + sp.nfull, s * hpw, min(hpw, H - s * hpw));
    }
  };
  if (single) {  // the kept pass-1 offsets are final
    const int b = threadIdx.x;
    if (b >= my_lo && b < my_hi) {
      int off[kScanN];
      SeqPlan sp = fits ? keep : SeqPlan{};
#pragma unroll
      for (int i = 0; i < kScanN; ++i) off[i] = (fits ? keep_off[i] : 0) + class_base[i];
      write_seq(b, sp, off, sp.key >= 0 ? key_run[sp.key] + keep_rank : 0);
    }
  } else {
    int run[kScanN];
#pragma unroll
    for (int i = 0; i < kScanN; ++i) run[i] = class_base[i];
    for (int base = 0; base < my_hi; base += T) {
      const int b = base + threadIdx.x;
      const PrefixRun pr = runs_of(base);
      SeqPlan sp = fits ? plan_of(b, pr) : SeqPlan{};
      int off[kScanN], t[kScanN];
#pragma unroll
      for (int i = 0; i < kScanN; ++i) off[i] = sp.n[i];
      block_scan_n(off, t, warp_sums);
#pragma unroll
      for (int i = 0; i < kScanN; ++i) {
        off[i] += run[i];
        run[i] += t[i];
      }
      const int krank = key_rank(sp.key, key_cnt, key_chunk);
      const int short_rank = sp.key >= 0 ? key_run[sp.key] + krank : 0;
      __syncthreads();
      if (threadIdx.x < 32) key_run[threadIdx.x] += key_chunk[threadIdx.x];
      __syncthreads();
      if (b >= my_lo && b < my_hi) write_seq(b, sp, off, short_rank);
    }
  }
  if (cta == 0 && threadIdx.x == 0) {
    // a workspace too small leaves every unit empty (all offsets 0): the merge then
    // reads no partial state and writes zero outputs with lse = -inf
    w.unit_offsets[B * H] = fits ? H * tot[0] : 0;
    int32_t sig[8];
    plan_signature(c, w, sig);
    for (int i = 0; i < 8; ++i) w.counter[8 + i] = sig[i];
    *w.n_items = fits ? te_all - tot[5] : 0;  // the attention kernel's entries
    *w.counter = 0;
    *w.pn_items = fits ? tot[5] : 0;          // then the prefix kernel's
    *w.pcounter = 0;
    *w.lift_count = 0;
    *w.lift_counter = 0;
    if (!fits) set_err(err, KV4_DEVERR_WORKSPACE);
  }
}

}  // namespace kv4
