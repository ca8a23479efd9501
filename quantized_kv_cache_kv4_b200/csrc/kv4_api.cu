// C-ABI entry points declared in include/kv4.h: host-side argument checks, workspace
// carve-up, and kernel launches on the caller's stream. No allocation, no sync.
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/kv4.h"
#include "kv4_device.cuh"
#include "kv4_internal.h"

namespace {

kv4_status check_config(const kv4_config *cfg) {
  if (cfg == nullptr) return KV4_ERR_INVALID_ARG;
  if (cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 || cfg->num_sinks < 0 ||
      cfg->num_recent < 0 || cfg->chunk_pages < 0 || cfg->demotion < 0 || cfg->demotion > 1 ||
      cfg->prefix_mode < 0 || cfg->prefix_mode > 1)
    return KV4_ERR_INVALID_ARG;
  if (cfg->head_dim != kv4::kHeadDim || cfg->page_size != kv4::kPage ||
      cfg->group_size != kv4::kGroup)
    return KV4_ERR_UNSUPPORTED_SHAPE;
  if (cfg->num_q_heads % cfg->num_kv_heads != 0 ||
      cfg->num_q_heads / cfg->num_kv_heads > kv4::kMaxGqa)
    return KV4_ERR_UNSUPPORTED_SHAPE;
  if (cfg->chunk_pages > kv4::kMaxChunkPages) return KV4_ERR_UNSUPPORTED_SHAPE;
  if (cfg->num_sinks + cfg->num_recent > KV4_MAX_PROTECTED) return KV4_ERR_PROTECTED_TOO_LARGE;
  return KV4_OK;
}

// Automatic chunk length (chunk_pages == 0), from num_seqs and max_seq_len only (the
// lengths themselves are on the device): the C in [8, 64] with the shortest estimated
// attention time, in units of one INT4 page of one warp, on the W = 148 SMs x 3 CTAs x 4
// warps resident warps of the persistent grid:
//   T(C) = max(C + e, work(C) / W) + (entries(C) > W ? (C + e) / 2 : 0),
// where an entry costs its pages plus e (its set-up, the ramp of its first copies, its
// record and its share of the merge), a protected-set entry kProtEntryPages, and work is
// the sum over all entries. One round of entries (entries <= W) ends with its longest
// entry; with more, the second term is the imbalance of the last round. Of the C within
// kAutoSlack of the best estimate the longest is taken (fewest partial states). The
// constants fit calls measured at forced chunk lengths: one round at the shortest C
// reaching it on 64 x 2048 and 32 x 4096 (C = 24, 21), 24- to 32-page chunks on
// 256 x 1024, 64 on the 1024-sequence rollout batch and on 128 x 16384 (32 and 48 there
// 1-5 % slower).
constexpr int kAutoMinChunk = 8;
constexpr double kAutoWarps = 148.0 * 3 * 4;
constexpr double kEntryPages = 8.0;
constexpr double kProtEntryPages = 12.0;
constexpr double kAutoSlack = 1.03;  // the longest C within 3 % of the best estimate

int chunk_of(const kv4_config *cfg, int32_t num_seqs, int32_t max_seq_len) {
  if (cfg->chunk_pages > 0) return cfg->chunk_pages;
  const int H = cfg->num_kv_heads;
  const int hpw = kv4::heads_per_warp_for(cfg->num_q_heads / H);
  const double slots = static_cast<double>(num_seqs) * ((H + hpw - 1) / hpw);
  const int S = cfg->num_sinks, R = cfg->num_recent;
  // pages of the INT4 range [S, L - R) at L = max_seq_len
  const long long int4_pages =
      max_seq_len - R > S ? (max_seq_len - R - 1) / kv4::kPage - S / kv4::kPage + 1 : 0;
  const double prot_entries = S + R > 0 ? slots : 0.0;
  double t[kv4::kMaxChunkPages + 1];
  double t_min = 0.0;
  for (int C = kAutoMinChunk; C <= kv4::kMaxChunkPages; ++C) {
    const double n_c = static_cast<double>((int4_pages + C - 1) / C);
    const double entries = slots * n_c + prot_entries;
    const double work = slots * (static_cast<double>(int4_pages) + n_c * kEntryPages) +
                        prot_entries * kProtEntryPages;
    t[C] = std::max(C + kEntryPages, work / kAutoWarps);
    if (entries > kAutoWarps) t[C] += 0.5 * (C + kEntryPages);
    if (C == kAutoMinChunk || t[C] < t_min) t_min = t[C];
  }
  int best = kAutoMinChunk;
  for (int C = kv4::kMaxChunkPages; C >= kAutoMinChunk; --C)
    if (t[C] <= kAutoSlack * t_min) {
      best = C;
      break;
    }
  return best;
}

bool misaligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

kv4_status make_view(const kv4_config *cfg, const kv4_int4_pool *pool, const kv4_int8_side *side,
                     const kv4_batch *batch, kv4::CacheView *v) {
  kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  if (pool == nullptr || side == nullptr || batch == nullptr) return KV4_ERR_INVALID_ARG;
  if (batch->num_seqs < 0 || batch->max_pages <= 0 || batch->max_seq_len < 0 ||
      pool->num_pages < 0 || batch->plan_reuse < 0 || batch->plan_reuse > 1)
    return KV4_ERR_INVALID_ARG;
  if (batch->num_seqs > 0 && (batch->page_table == nullptr || batch->seq_lens == nullptr))
    return KV4_ERR_INVALID_ARG;
  if (!pool->k_codes || !pool->v_codes || !pool->k_params || !pool->v_params)
    return KV4_ERR_INVALID_ARG;
  if (misaligned16(pool->k_codes) || misaligned16(pool->v_codes) ||
      misaligned16(pool->k_params) || misaligned16(pool->v_params))
    return KV4_ERR_INVALID_ARG;
  const int S = cfg->num_sinks, R = cfg->num_recent;
  if (S > 0) {
    if (!side->sink_k || !side->sink_v || !side->sink_ks || !side->sink_vs ||
        side->num_sink_sets <= 0 || batch->sink_idx == nullptr)
      return KV4_ERR_INVALID_ARG;
    if (misaligned16(side->sink_k) || misaligned16(side->sink_v) ||
        misaligned16(side->sink_ks) || misaligned16(side->sink_vs))
      return KV4_ERR_INVALID_ARG;
  }
  if (R > 0) {
    if (!side->ring_k || !side->ring_v || !side->ring_ks || !side->ring_vs || side->num_rings <= 0)
      return KV4_ERR_INVALID_ARG;
    if (misaligned16(side->ring_k) || misaligned16(side->ring_v) ||
        misaligned16(side->ring_ks) || misaligned16(side->ring_vs))
      return KV4_ERR_INVALID_ARG;
  }
  v->k_codes = pool->k_codes;
  v->v_codes = pool->v_codes;
  v->k_params = pool->k_params;
  v->v_params = pool->v_params;
  v->num_pages = pool->num_pages;
  v->sink_k = side->sink_k;
  v->sink_v = side->sink_v;
  v->sink_ks = side->sink_ks;
  v->sink_vs = side->sink_vs;
  v->num_sink_sets = S > 0 ? side->num_sink_sets : 0;
  v->sink_tiles = (S + kv4::kPage - 1) / kv4::kPage;
  v->ring_k = side->ring_k;
  v->ring_v = side->ring_v;
  v->ring_ks = side->ring_ks;
  v->ring_vs = side->ring_vs;
  v->num_rings = R > 0 ? side->num_rings : 0;
  v->ring_tiles = (R + kv4::kPage - 1) / kv4::kPage;
  v->page_table = batch->page_table;
  v->max_pages = batch->max_pages;
  v->seq_lens = batch->seq_lens;
  v->sink_idx = batch->sink_idx;
  v->ring_idx = batch->ring_idx;
  v->num_seqs = batch->num_seqs;
  v->num_kv_heads = cfg->num_kv_heads;
  v->gqa = cfg->num_q_heads / cfg->num_kv_heads;
  v->num_sinks = S;
  v->num_recent = R;
  v->int4_from_int8 = cfg->demotion == 1;
  return KV4_OK;
}

// The comparison baselines have no protected set and no shared-prefix read: the config
// is used with S = R = 0 and the prefix read off.
kv4_config without_protection(const kv4_config *cfg) {
  kv4_config c = *cfg;
  c.num_sinks = 0;
  c.num_recent = 0;
  c.prefix_mode = KV4_PREFIX_OFF;
  return c;
}

bool prefix_on(const kv4_config *cfg) { return cfg->prefix_mode == KV4_PREFIX_SHARED; }

// kv4_test_withhold_copy: a one-shot setting of this host thread, taken by its next
// attention call.
struct WithheldCopy {
  int32_t item = -1;
  uint32_t wait_limit = 0;
};
thread_local WithheldCopy g_withheld;

void take_test_hook(kv4::Workspace *w) {
  if (g_withheld.item < 0) return;
  w->fault_item = g_withheld.item;
  if (g_withheld.wait_limit > 0) w->wait_limit = g_withheld.wait_limit;
  g_withheld = WithheldCopy{};
}

kv4_status make_baseline_view(kv4_baseline_format fmt, const kv4_config *cfg,
                              const kv4_paged_pool *pool, const kv4_batch *batch,
                              kv4::CacheView *v) {
  if (fmt != KV4_BASELINE_BF16 && fmt != KV4_BASELINE_KV8) return KV4_ERR_INVALID_ARG;
  kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  if (pool == nullptr || batch == nullptr) return KV4_ERR_INVALID_ARG;
  if (batch->num_seqs < 0 || batch->max_pages <= 0 || batch->max_seq_len < 0 ||
      pool->num_pages < 0)
    return KV4_ERR_INVALID_ARG;
  if (batch->num_seqs > 0 && (batch->page_table == nullptr || batch->seq_lens == nullptr))
    return KV4_ERR_INVALID_ARG;
  if (!pool->k || !pool->v || misaligned16(pool->k) || misaligned16(pool->v))
    return KV4_ERR_INVALID_ARG;
  if (fmt == KV4_BASELINE_KV8 && (!pool->k_scales || !pool->v_scales ||
                                  misaligned16(pool->k_scales) || misaligned16(pool->v_scales)))
    return KV4_ERR_INVALID_ARG;
  *v = kv4::CacheView{};
  v->k_codes = static_cast<uint8_t *>(pool->k);
  v->v_codes = static_cast<uint8_t *>(pool->v);
  v->k_params = pool->k_scales;
  v->v_params = pool->v_scales;
  v->num_pages = pool->num_pages;
  v->page_table = batch->page_table;
  v->max_pages = batch->max_pages;
  v->seq_lens = batch->seq_lens;
  v->num_seqs = batch->num_seqs;
  v->num_kv_heads = cfg->num_kv_heads;
  v->gqa = cfg->num_q_heads / cfg->num_kv_heads;
  return KV4_OK;
}

// Carve the workspace for (cfg, batch): the automatic chunk choice, falling back to the
// longest chunks when the caller's workspace is too small for a finer split.
kv4_status carve_workspace(const kv4_config *cfg, const kv4::CacheView &v,
                           const kv4_batch *batch, void *workspace, size_t ws_bytes,
                           kv4::Workspace *w) {
  size_t need = kv4::workspace_bytes(batch->num_seqs, batch->max_seq_len, v.num_kv_heads, v.gqa,
                                     chunk_of(cfg, batch->num_seqs, batch->max_seq_len),
                                     prefix_on(cfg), w, workspace);
  // A workspace sized for a larger batch or longer sequences (and so for longer automatic
  // chunks) may be too small for a finer automatic split of this one: fall back to the
  // longest chunks, for which any workspace sized with this config at larger or equal
  // (num_seqs, max_seq_len) is large enough.
  if (ws_bytes < need && cfg->chunk_pages == 0)
    need = kv4::workspace_bytes(batch->num_seqs, batch->max_seq_len, v.num_kv_heads, v.gqa,
                                kv4::kMaxChunkPages, prefix_on(cfg), w, workspace);
  return ws_bytes < need ? KV4_ERR_WORKSPACE_TOO_SMALL : KV4_OK;
}

kv4_status check_attention_args(const kv4_batch *batch, const void *q, const void *out,
                                const float *out_f32, const void *workspace) {
  if (q == nullptr || out == nullptr || workspace == nullptr) return KV4_ERR_INVALID_ARG;
  if (misaligned16(q) || misaligned16(out) || misaligned16(out_f32) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return KV4_ERR_INVALID_ARG;
  return batch->num_seqs >= 0 ? KV4_OK : KV4_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

size_t kv4_workspace_size(const kv4_config *cfg, int32_t num_seqs, int32_t max_seq_len) {
  if (check_config(cfg) != KV4_OK || num_seqs < 0 || max_seq_len < 0) return 0;
  return kv4::workspace_bytes(num_seqs, max_seq_len, cfg->num_kv_heads,
                              cfg->num_q_heads / cfg->num_kv_heads,
                              chunk_of(cfg, num_seqs, max_seq_len), prefix_on(cfg), nullptr,
                              nullptr);
}

int32_t kv4_chunk_pages_for(const kv4_config *cfg, int32_t num_seqs, int32_t max_seq_len) {
  if (check_config(cfg) != KV4_OK || num_seqs < 0 || max_seq_len < 0) return -1;
  return chunk_of(cfg, num_seqs, max_seq_len);
}

kv4_status kv4_quantize_append(const kv4_config *cfg, const kv4_int4_pool *pool,
                               const kv4_int8_side *side, const kv4_batch *batch,
                               const void *k_new, const void *v_new, const int32_t *new_indptr,
                               int32_t total_new, int32_t *err_flag, kv4_stream_t stream) {
  kv4::CacheView v;
  kv4_status st = make_view(cfg, pool, side, batch, &v);
  if (st != KV4_OK) return st;
  if (total_new < 0) return KV4_ERR_INVALID_ARG;
  if (new_indptr == nullptr && total_new != batch->num_seqs) return KV4_ERR_INVALID_ARG;
  if (total_new > 0 && (k_new == nullptr || v_new == nullptr)) return KV4_ERR_INVALID_ARG;
  if (misaligned16(k_new) || misaligned16(v_new)) return KV4_ERR_INVALID_ARG;
  if (total_new == 0 || batch->num_seqs == 0) return KV4_OK;
  cudaError_t e = kv4::launch_append(v, static_cast<const uint16_t *>(k_new),
                                     static_cast<const uint16_t *>(v_new), new_indptr, total_new,
                                     err_flag, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

kv4_status kv4_decode_attention(const kv4_config *cfg, const kv4_int4_pool *pool,
                                const kv4_int8_side *side, const kv4_batch *batch, const void *q,
                                void *out, float *out_f32, float *lse, void *workspace,
                                size_t ws_bytes, int32_t *err_flag, kv4_stream_t stream) {
  kv4::CacheView v;
  kv4_status st = make_view(cfg, pool, side, batch, &v);
  if (st != KV4_OK) return st;
  if (batch->num_seqs == 0) return KV4_OK;
  st = check_attention_args(batch, q, out, out_f32, workspace);
  if (st != KV4_OK) return st;
  kv4::Workspace w;
  st = carve_workspace(cfg, v, batch, workspace, ws_bytes, &w);
  if (st != KV4_OK) return st;
  take_test_hook(&w);
  w.check_plan = batch->plan_reuse;
  const kv4::PlanSig sig = kv4::plan_signature_host(v, w);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = batch->plan_reuse ? cudaSuccess : kv4::launch_plan(v, w, err_flag, s);
  if (e == cudaSuccess) e = kv4::launch_prefix(v, w, static_cast<const uint16_t *>(q), err_flag, s);
  if (e == cudaSuccess)
    e = kv4::launch_attention(v, w, static_cast<const uint16_t *>(q), err_flag, s);
  if (e == cudaSuccess)
    e = kv4::launch_merge(w.partials, w.unit_offsets, batch->num_seqs * v.num_kv_heads, v.gqa,
                          static_cast<uint16_t *>(out), out_f32, lse, w.counter,
                          w.check_plan ? &sig : nullptr, s);
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

kv4_status kv4_decode_step(const kv4_config *cfg, const kv4_int4_pool *pool,
                           const kv4_int8_side *side, const kv4_batch *batch,
                           const void *k_new, const void *v_new, const void *q, void *out,
                           float *out_f32, float *lse, void *workspace, size_t ws_bytes,
                           int32_t *err_flag, kv4_stream_t stream) {
  kv4::CacheView v;
  kv4_status st = make_view(cfg, pool, side, batch, &v);
  if (st != KV4_OK) return st;
  if (batch->num_seqs == 0) return KV4_OK;
  if (k_new == nullptr || v_new == nullptr || misaligned16(k_new) || misaligned16(v_new))
    return KV4_ERR_INVALID_ARG;
  st = check_attention_args(batch, q, out, out_f32, workspace);
  if (st != KV4_OK) return st;
  kv4::Workspace w;
  st = carve_workspace(cfg, v, batch, workspace, ws_bytes, &w);
  if (st != KV4_OK) return st;
  take_test_hook(&w);
  w.check_plan = batch->plan_reuse;
  const kv4::PlanSig sig = kv4::plan_signature_host(v, w);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t *kn = static_cast<const uint16_t *>(k_new);
  const uint16_t *vn = static_cast<const uint16_t *>(v_new);
  // the work list and the append are independent: one launch does both
  cudaError_t e = batch->plan_reuse
                      ? kv4::launch_append(v, kn, vn, nullptr, batch->num_seqs, err_flag, s)
                      : kv4::launch_plan_append(v, w, kn, vn, err_flag, s);
  if (e == cudaSuccess) e = kv4::launch_prefix(v, w, static_cast<const uint16_t *>(q), err_flag, s);
  if (e == cudaSuccess)
    e = kv4::launch_attention(v, w, static_cast<const uint16_t *>(q), err_flag, s);
  if (e == cudaSuccess)
    e = kv4::launch_merge(w.partials, w.unit_offsets, batch->num_seqs * v.num_kv_heads, v.gqa,
                          static_cast<uint16_t *>(out), out_f32, lse, w.counter,
                          w.check_plan ? &sig : nullptr, s);
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

kv4_status kv4_regional_merge(const float *partials, const int32_t *region_offsets,
                              int32_t n_units, int32_t group, int32_t head_dim, void *out,
                              float *out_f32, float *lse, kv4_stream_t stream) {
  if (n_units < 0 || group < 1 || group > kv4::kMaxGqa) return KV4_ERR_INVALID_ARG;
  if (head_dim != kv4::kHeadDim) return KV4_ERR_UNSUPPORTED_SHAPE;
  if (n_units == 0) return KV4_OK;
  if (partials == nullptr || region_offsets == nullptr || out == nullptr)
    return KV4_ERR_INVALID_ARG;
  if (misaligned16(partials) || misaligned16(out) || misaligned16(out_f32))
    return KV4_ERR_INVALID_ARG;
  cudaError_t e = kv4::launch_merge(partials, region_offsets, n_units, group,
                                    static_cast<uint16_t *>(out), out_f32, lse, nullptr,
                                    nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

size_t kv4_baseline_workspace_size(const kv4_config *cfg, int32_t num_seqs,
                                   int32_t max_seq_len) {
  if (cfg == nullptr) return 0;
  const kv4_config c = without_protection(cfg);
  return kv4_workspace_size(&c, num_seqs, max_seq_len);
}

kv4_status kv4_baseline_append(kv4_baseline_format fmt, const kv4_config *cfg,
                               const kv4_paged_pool *pool, const kv4_batch *batch,
                               const void *k_new, const void *v_new, const int32_t *new_indptr,
                               int32_t total_new, int32_t *err_flag, kv4_stream_t stream) {
  if (cfg == nullptr) return KV4_ERR_INVALID_ARG;
  const kv4_config c = without_protection(cfg);
  kv4::CacheView v;
  kv4_status st = make_baseline_view(fmt, &c, pool, batch, &v);
  if (st != KV4_OK) return st;
  if (total_new < 0) return KV4_ERR_INVALID_ARG;
  if (new_indptr == nullptr && total_new != batch->num_seqs) return KV4_ERR_INVALID_ARG;
  if (total_new > 0 && (k_new == nullptr || v_new == nullptr)) return KV4_ERR_INVALID_ARG;
  if (misaligned16(k_new) || misaligned16(v_new)) return KV4_ERR_INVALID_ARG;
  if (total_new == 0 || batch->num_seqs == 0) return KV4_OK;
  cudaError_t e = kv4::launch_baseline_append(fmt, v, static_cast<const uint16_t *>(k_new),
                                              static_cast<const uint16_t *>(v_new), new_indptr,
                                              total_new, err_flag,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

kv4_status kv4_baseline_decode_attention(kv4_baseline_format fmt, const kv4_config *cfg,
                                         const kv4_paged_pool *pool, const kv4_batch *batch,
                                         const void *q, void *out, float *out_f32, float *lse,
                                         void *workspace, size_t ws_bytes, int32_t *err_flag,
                                         kv4_stream_t stream) {
  if (cfg == nullptr) return KV4_ERR_INVALID_ARG;
  const kv4_config c = without_protection(cfg);
  kv4::CacheView v;
  kv4_status st = make_baseline_view(fmt, &c, pool, batch, &v);
  if (st != KV4_OK) return st;
  if (batch->num_seqs == 0) return KV4_OK;
  st = check_attention_args(batch, q, out, out_f32, workspace);
  if (st != KV4_OK) return st;
  kv4::Workspace w;
  st = carve_workspace(&c, v, batch, workspace, ws_bytes, &w);
  if (st != KV4_OK) return st;
  take_test_hook(&w);
  w.heads_per_warp = 1;  // one kv head per warp and entry
  w.check_plan = batch->plan_reuse;
  const kv4::PlanSig sig = kv4::plan_signature_host(v, w);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = batch->plan_reuse ? cudaSuccess : kv4::launch_plan(v, w, err_flag, s);
  if (e == cudaSuccess)
    e = kv4::launch_baseline_attention(fmt, v, w, static_cast<const uint16_t *>(q), err_flag, s);
  if (e == cudaSuccess)
    e = kv4::launch_merge(w.partials, w.unit_offsets, batch->num_seqs * v.num_kv_heads, v.gqa,
                          static_cast<uint16_t *>(out), out_f32, lse, w.counter,
                          w.check_plan ? &sig : nullptr, s);
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

void kv4_test_withhold_copy(int32_t item, uint32_t wait_limit) {
  g_withheld.item = item < 0 ? -1 : item;
  g_withheld.wait_limit = wait_limit;
}

const char *kv4_status_string(kv4_status status) {
  switch (status) {
    case KV4_OK: return "ok";
    case KV4_ERR_INVALID_ARG: return "invalid argument";
    case KV4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case KV4_ERR_PROTECTED_TOO_LARGE: return "protected set larger than 144 positions";
    case KV4_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case KV4_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int32_t kv4_version(void) { return 500; }

}  // extern "C"
