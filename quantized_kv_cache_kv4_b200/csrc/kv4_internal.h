// Internal launch interfaces between the C-ABI layer (kv4_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "../../include/kv4.h"

namespace kv4 {

constexpr int kMaxDevices = 64;

// Per-device launch set-up done once: `configure(dev)` (kernel attributes, the persistent
// grid size) runs under the table's lock the first time a device is seen, and its
// positive result is kept for that device; later calls only read it. Safe for host
// threads driving different devices at once.
struct PerDevice {
  std::mutex mu;
  int value[kMaxDevices] = {};
};

template <class F>
cudaError_t once_per_device(PerDevice &t, F configure, int *value) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(t.mu);
  if (t.value[dev] <= 0) {
    int v = 0;
    e = configure(dev, &v);
    if (e != cudaSuccess) return e;
    t.value[dev] = v > 0 ? v : 1;
  }
  *value = t.value[dev];
  return cudaSuccess;
}

// Everything a kernel needs about the cache and the batch, by value.
struct CacheView {
  uint8_t *k_codes, *v_codes;
  uint16_t *k_params, *v_params;
  int32_t num_pages;
  int8_t *sink_k, *sink_v;
  uint16_t *sink_ks, *sink_vs;
  int32_t num_sink_sets, sink_tiles;
  int8_t *ring_k, *ring_v;
  uint16_t *ring_ks, *ring_vs;
  int32_t num_rings, ring_tiles;
  const int32_t *page_table;
  int32_t max_pages;
  const int32_t *seq_lens;
  const int32_t *sink_idx;
  const int32_t *ring_idx;
  int32_t num_seqs;
  int32_t num_kv_heads;
  int32_t gqa;  // query heads per kv head
  int32_t num_sinks, num_recent;
  bool int4_from_int8;  // demotion reading B: INT4 copies quantised from the INT8 copy
};

// Workspace carve-up for one decode-attention call.
struct Workspace {
  int32_t *counter;       // [1] dynamic work counter (reset by the plan kernel)
  int32_t *n_items;       // [1] number of work entries
  int4 *entries;          // [cap_entries] (sequence, region, first kv head, kv heads)
  int32_t *unit_offsets;  // [num_seqs*Hkv + 1] first partial record row of each (b, h)
  float *partials;        // [cap_pairs*Hkv][gqa][kRecordFloats]
  int32_t cap_pairs;      // (sequence, region) pairs the partial area holds
  int32_t cap_entries;    // work entries the entry list holds
  int32_t chunk_pages;
  int32_t heads_per_warp;  // kv heads one warp serves in an INT4 region entry (1 or 2)
  // shared-prefix read (nullptr prefix_end: off): pages shared by consecutive sequences
  // are read once per group of up to 16 / gqa members, in entries (first member,
  // -1 - prompt chunk, kv head, members)
  int32_t *prefix_end;     // [num_seqs] end page of the group's shared INT4 pages, 0 = none
  int32_t *pcounter;       // [1] dynamic work counter of the prefix kernel
  int32_t *pn_items;       // [1] shared-prefix entries (listed after the n_items others)
  int32_t *lift_count;     // [1] entries on the lift list (small V scales)
  int32_t *lift_counter;   // [1] dynamic work counter of the lift kernel
  int32_t *lift_items;     // [cap_entries] work items on the lift list
  int32_t check_plan;      // the call reuses a work list: kernels check its signature first
  uint32_t wait_limit;     // attempts of one bounded wait for a copy (kWaitLimit)
  int32_t fault_item;      // testing hook: work item whose first copy is withheld, -1 none
};

constexpr uint32_t kWaitLimit = 1u << 22;  // bounded-wait attempts in normal operation

// Where the merged attention output goes.
struct Outputs {
  uint16_t *out;   // bf16 [B][Hq][128]
  float *out_f32;  // optional fp32 [B][Hq][128]
  float *lse;      // optional fp32 [B][Hq]
};

// kv heads one attention warp serves for a GQA ratio (2 when G <= 4).
int heads_per_warp_for(int gqa);

size_t workspace_bytes(int32_t num_seqs, int32_t max_seq_len, int32_t num_kv_heads,
                       int32_t gqa, int32_t chunk_pages, bool prefix, Workspace *carve,
                       void *base);

cudaError_t launch_append(const CacheView &c, const uint16_t *k_new, const uint16_t *v_new,
                          const int32_t *new_indptr, int32_t total_new, int32_t *err_flag,
                          cudaStream_t s);

cudaError_t launch_plan(const CacheView &c, const Workspace &w, int32_t *err_flag,
                        cudaStream_t s);

// The work list of w and the append of one token per sequence (k_new, v_new: bf16
// [num_seqs][num_kv_heads][128]) in one launch; the two are independent.
cudaError_t launch_plan_append(const CacheView &c, const Workspace &w, const uint16_t *k_new,
                               const uint16_t *v_new, int32_t *err_flag, cudaStream_t s);

cudaError_t launch_attention(const CacheView &c, const Workspace &w, const uint16_t *q,
                             int32_t *err_flag, cudaStream_t s);

// The shared-prefix read (launches nothing when w.prefix_end is nullptr).
cudaError_t launch_prefix(const CacheView &c, const Workspace &w, const uint16_t *q,
                          int32_t *err_flag, cudaStream_t s);


// The signature a work list of (c, w) carries (plan_signature in the kernels; the host
// copy is what the merge compares with).
struct PlanSig {
  int32_t v[8];
};
PlanSig plan_signature_host(const CacheView &c, const Workspace &w);

// reset: the workspace's counter block (nullptr for a bare merge); the merge, the last
// kernel of an attention call, zeroes its work counters there, so that a following call
// can reuse the work list without the plan kernel. want: the call's signature when it
// reuses a work list (nullptr otherwise); the merge then checks the list's signature
// first and writes zero outputs if it is another batch's.
cudaError_t launch_merge(const float *partials, const int32_t *unit_offsets, int32_t n_units,
                         int32_t group, uint16_t *out, float *out_f32, float *lse,
                         const int32_t *reset, const PlanSig *want, cudaStream_t s);

// Comparison baselines (kv4_baseline.cu): fmt is a kv4_baseline_format. The view's
// k_codes / v_codes hold the BF16 or INT8 pages, k_params / v_params the KV8 scales.
cudaError_t launch_baseline_append(int fmt, const CacheView &c, const uint16_t *k_new,
                                   const uint16_t *v_new, const int32_t *new_indptr,
                                   int32_t total_new, int32_t *err_flag, cudaStream_t s);
cudaError_t launch_baseline_attention(int fmt, const CacheView &c, const Workspace &w,
                                      const uint16_t *q, int32_t *err_flag, cudaStream_t s);

}  // namespace kv4
