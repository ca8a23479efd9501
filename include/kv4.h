/*
 * kv4.h -- C ABI of a B200 (sm_100a) library for batched decode-step GQA attention
 * over a paged INT4 KV cache with bounded INT8 protection of attention sinks and a
 * recent window.
 *
 * The method is KV4-RL (arXiv 2610.14448, "KV4-RL: Unlocking Faster Asynchronous
 * Rollouts for RLVR with INT4 KV Cache Quantization"):
 *   - the whole context is kept in calibration-free INT4 in a paged format, and INT8
 *     copies are kept for a fixed set of attention-sink and recent positions, at most
 *     144 of them (ai4snews summary, "Interpretation" para. 3; aimodeling article,
 *     "INT4 as the base, INT8 insurance for critical positions");
 *   - attention runs over the integer codes and combines the regions with an exact
 *     regional softmax merge (ai4snews summary, "Interpretation" para. 3);
 *   - protected positions use higher-fidelity probability-value arithmetic
 *     (aimodeling article, same section).
 * The pages give no bit-level format and no API; the format and calls below are this
 * library's own, chosen as the plainest reading of those statements.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned and allocated by the caller. The
 *     library never allocates or frees device memory at call time and never
 *     synchronises; every call is asynchronous on the given stream (NULL = the legacy
 *     default stream). (kv4_decode_step creates one stream and two events per host
 *     thread and device on first use; kv4_decode_attention_noalloc uses a fixed
 *     device array of the library's own.)
 *   - Arguments are checked on the host before anything is launched; a failed check
 *     returns a negative kv4_status and launches nothing.
 *   - Data-dependent checks run on the device: a kernel that meets a bad page id,
 *     sequence length, side-store index or workspace overflow ORs a KV4_DEVERR_* bit
 *     into *err_flag (a device int32 the caller zeroes and reads after synchronising)
 *     and skips the offending work item. Kernels never trap and never spin without a
 *     bound.
 *   - fp16 and bf16 values are passed as their 16-bit patterns.
 *
 * Storage format (all little-endian; "slot" = token position within a page or tile):
 *
 *   INT4 pool, one block per (page, kv head), pages of 16 tokens:
 *     k_codes, v_codes  uint8 [num_pages][Hkv][4 groups][16 slots][16 bytes]
 *         byte i of (group g, slot t) = code(dim 32g+2i) | code(dim 32g+2i+1) << 4
 *     k_params, v_params  fp16 [num_pages][Hkv][16 slots][4 groups][2] = (scale, min)
 *     Per token and 32-dim group:  min = fp16(group min),
 *         scale = fp16(fp32(fp32(max - min) / 15)),
 *         code  = clamp(rne(fp32(fp32(x - min) / scale)), 0, 15)   (0 if scale == 0),
 *     fp16 rounding is nearest-even saturating at +-65504. Value = code*scale + min.
 *
 *   INT8 side store, tiles of 16 slots:
 *     codes  int8 [..][Hkv][tiles][8 strips][16 slots][16 bytes]
 *         byte i of (strip c, slot t) = code(dim 16c + i)
 *     scales fp16 [..][Hkv][tiles*16]
 *     Per token: scale = fp16(fp32(max|x| / 127)),
 *         code = clamp(rne(fp32(x / scale)), -127, 127)  (0 if scale == 0).
 *     Value = code*scale.
 *     Sink sets: tiles = ceil(S/16); slot p holds position p < S.
 *     Recent rings: tiles = ceil(R/16); slot (p mod R) holds position p >= S.
 *
 *   Regions of a context of length L (S sinks, R recent, S + R <= 144):
 *     sink [0, min(S,L)) and recent [max(S, L-R), L) are read from INT8,
 *     [S, L-R) (when L-R > S) is read from the INT4 pages. Every position is also
 *     stored in INT4 ("whole context in INT4"); the INT8 copy of a position is
 *     overwritten (demoted) when position p+R is appended.
 */
#ifndef KV4_H
#define KV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *kv4_stream_t;

typedef enum {
  KV4_OK = 0,
  KV4_ERR_INVALID_ARG = -1,         /* NULL pointer, negative size, inconsistent struct */
  KV4_ERR_UNSUPPORTED_SHAPE = -2,   /* head_dim != 128, page_size != 16, group_size != 32,
                                       Hq not a multiple of Hkv, or Hq/Hkv > 8 */
  KV4_ERR_PROTECTED_TOO_LARGE = -3, /* num_sinks + num_recent > 144 */
  KV4_ERR_WORKSPACE_TOO_SMALL = -4, /* ws_bytes < kv4_workspace_size(...) */
  KV4_ERR_CUDA = -5                 /* a CUDA runtime call failed (launch error) */
} kv4_status;

/* Bits OR-ed into *err_flag by the kernels. */
#define KV4_DEVERR_PAGE_ID 1u    /* page-table entry outside [0, num_pages) */
#define KV4_DEVERR_SEQ_LEN 2u    /* seq_len < 0, > max_pages*16, or fewer tokens than appended */
#define KV4_DEVERR_SIDE_IDX 4u   /* sink_idx / ring_idx outside the side store */
#define KV4_DEVERR_Q_RANGE 8u    /* reserved: no longer raised (queries enter the dot
                                    products in per-query fixed point, any finite value) */
#define KV4_DEVERR_WORKSPACE 16u /* the batch needs more work items than the workspace holds
                                    (the call then writes zero outputs, lse = -inf) */
#define KV4_DEVERR_TIMEOUT 32u   /* a bounded wait for an async copy gave up */

#define KV4_MAX_PROTECTED 144

typedef struct {
  int32_t num_q_heads;  /* Hq */
  int32_t num_kv_heads; /* Hkv; query head j reads kv head j / (Hq/Hkv) */
  int32_t head_dim;     /* must be 128 */
  int32_t page_size;    /* must be 16 */
  int32_t group_size;   /* must be 32 */
  int32_t num_sinks;    /* S >= 0 */
  int32_t num_recent;   /* R >= 0, S + R <= 144 */
  int32_t chunk_pages;  /* split-K chunk length in pages for the INT4 region, 1..64; 0 = chosen
                           per call from num_seqs and max_seq_len: the length in 8..64 with
                           the shortest estimated attention time on the GPU's resident warps
                           (64 for large batches, shorter where long chunks would leave
                           warps idle; 64 whenever the workspace passed is too small for
                           the finer split) */
  int32_t demotion;     /* where a position's INT4 copy comes from: 0 = the bf16 input, at
                           append (reading A, the default); 1 = the position's INT8 copy,
                           dequantised (reading B: what demotion out of the recent window
                           would write). Attention is the same for both. */
  int32_t prefix_mode;  /* shared-prefix read (KV4_PREFIX_*): 0 = off (the default): every
                           sequence reads all its pages on its own; 1 = shared: consecutive
                           sequences whose page tables map their leading INT4 pages to the
                           same physical pages -- the responses of one prompt -- form a
                           group whose shared pages are read once per kv head for up to 16
                           query heads of the group (4 sequences at GQA 4) and merged as one
                           more region per sequence. Results agree within the attention
                           tolerance either way (the regions differ, so the rounding does).
                           On the 1024-sequence rollout batch the shared read removes 13 %
                           of the attention kernel's time but costs more in its own kernel
                           and in the sharing detection, so it is off by default. */
} kv4_config;

#define KV4_PREFIX_OFF 0
#define KV4_PREFIX_SHARED 1

typedef struct {
  uint8_t *k_codes;   /* see "INT4 pool" above */
  uint8_t *v_codes;
  uint16_t *k_params;
  uint16_t *v_params;
  int32_t num_pages;
} kv4_int4_pool;

typedef struct {
  int8_t *sink_k;     /* [num_sink_sets][Hkv][ceil(S/16)][8][16][16]; may be NULL if S == 0 */
  int8_t *sink_v;
  uint16_t *sink_ks;  /* [num_sink_sets][Hkv][ceil(S/16)*16] */
  uint16_t *sink_vs;
  int32_t num_sink_sets;
  int8_t *ring_k;     /* [num_rings][Hkv][ceil(R/16)][8][16][16]; may be NULL if R == 0 */
  int8_t *ring_v;
  uint16_t *ring_ks;  /* [num_rings][Hkv][ceil(R/16)*16] */
  uint16_t *ring_vs;
  int32_t num_rings;
} kv4_int8_side;

typedef struct {
  const int32_t *page_table; /* [num_seqs][max_pages]: page of positions [16i, 16i+16) */
  int32_t max_pages;
  const int32_t *seq_lens;   /* [num_seqs]: context length AFTER this step's append */
  const int32_t *sink_idx;   /* [num_seqs]: sink set of each sequence (sequences that share
                                a prompt may share one); may be NULL if S == 0 */
  const int32_t *ring_idx;   /* [num_seqs]: recent ring of each sequence; NULL = identity */
  int32_t num_seqs;
  int32_t max_seq_len;       /* host-side upper bound on seq_lens, sizes the workspace; a
                                longer sequence may overflow it (KV4_DEVERR_WORKSPACE) */
  int32_t plan_reuse;        /* 0: the attention call builds its work list in the workspace
                                (the default). 1: it uses the work list the previous
                                attention call on the same workspace left there, which must
                                have been made with this same batch (lengths, page table,
                                sink and ring indices, num_seqs, max_seq_len) and config --
                                e.g. the layers of one decode step after the first. The
                                kernels stay within their buffers if that does not hold
                                (entries of an unknown sequence or length are skipped and
                                flagged), but the results are then void. */
} kv4_batch;

/*
 * Bytes of device workspace kv4_decode_attention needs for a batch of num_seqs
 * sequences no longer than max_seq_len. Returns 0 for invalid arguments.
 * (Infrastructure of this library: no passage of the pages defines it.)
 */
size_t kv4_workspace_size(const kv4_config *cfg, int32_t num_seqs, int32_t max_seq_len);

/*
 * The split-K chunk length in pages that kv4_decode_attention and kv4_workspace_size use
 * for a batch of num_seqs sequences no longer than max_seq_len: cfg->chunk_pages when it
 * is set, else the automatic choice (see kv4_config.chunk_pages). Returns -1 for invalid
 * arguments. (Infrastructure of this library: no passage of the pages defines it.)
 */
int32_t kv4_chunk_pages_for(const kv4_config *cfg, int32_t num_seqs, int32_t max_seq_len);

/*
 * Quantise and append new tokens' K/V: the per-step write path (with n = 1 per
 * sequence), also usable for bulk prefill.
 * Defined by: the whole context kept in calibration-free INT4 in a paged format, with
 * INT8 copies of the attention-sink and recent positions (ai4snews summary,
 * "Interpretation" para. 3; kipquest abstract, "calibration-free INT4 KV
 * quantization"; aimodeling article, "INT4 as the base, INT8 insurance for critical
 * positions": paged INT4 format, INT8 side cache). The demotion of a position leaving
 * the recent window is the overwrite of its INT8 copy described below.
 *
 *   k_new, v_new: bf16 [total_new][Hkv][128], device.
 *   new_indptr:   int32 [num_seqs+1], device, CSR row ranges: rows new_indptr[b] ..
 *                 new_indptr[b+1]-1 are sequence b's new tokens, in position order,
 *                 placed at positions seq_lens[b]-n_b .. seq_lens[b]-1. NULL means
 *                 exactly one new token per sequence (row b, position seq_lens[b]-1).
 *   total_new:    number of rows (== num_seqs when new_indptr is NULL).
 *
 * Every token is written to its INT4 page slot. A token at position p < S is also
 * written to sink set sink_idx[b]; a token at p >= S whose position lies in the final
 * recent window [seq_lens[b]-R, seq_lens[b]) is written to ring slot p mod R of ring
 * ring_idx[b], overwriting -- demoting -- the INT8 copy of position p-R. (Tokens that
 * would be demoted again within the same call are not written to the ring, so a bulk
 * append leaves the same state as appending one token at a time.)
 * Sequences that share pages must not append into the same page in one call.
 */
kv4_status kv4_quantize_append(const kv4_config *cfg, const kv4_int4_pool *pool,
                               const kv4_int8_side *side, const kv4_batch *batch,
                               const void *k_new, const void *v_new,
                               const int32_t *new_indptr, int32_t total_new,
                               int32_t *err_flag, kv4_stream_t stream);

/*
 * Decode-step attention. Defined by: attention over the INT4 pages and the INT8 copies
 * of the protected positions through an integer attention path and an exact regional
 * softmax merge (ai4snews summary, "Interpretation" para. 3), with higher-fidelity
 * probability-value arithmetic on the protected positions (aimodeling article, "INT4 as
 * the base, INT8 insurance for critical positions"). For every sequence b and query
 * head j,
 *   O[b, j] = softmax(K_eff q / sqrt(128)) V_eff over positions [0, seq_lens[b]),
 * where K_eff/V_eff are the INT8 dequantised copies on protected positions and the
 * INT4 dequantised values elsewhere. Each region (the protected set, and each chunk of
 * `chunk_pages` INT4 pages) yields a partial softmax state (max, denominator, weighted
 * value sum) that an exact log-sum-exp merge combines in a fixed order, so results
 * are deterministic.
 *
 *   q:       bf16 [num_seqs][Hq][128], finite. Each query enters the dot products as
 *            15-bit fixed point with a power-of-two step set by its largest element
 *            (rounding at most 2^-14 of that element's magnitude).
 *   out:     bf16 [num_seqs][Hq][128].
 *   out_f32: optional fp32 [num_seqs][Hq][128] (NULL to skip).
 *   lse:     optional fp32 [num_seqs][Hq], natural log of the softmax denominator
 *            (including the max); -inf for empty sequences (NULL to skip).
 *   workspace, ws_bytes: device scratch of at least kv4_workspace_size(cfg, num_seqs,
 *            max_seq_len) bytes, 256-byte aligned; contents need no initialisation.
 * A sequence of length 0 yields O = 0. The probability weights p * vscale enter the PV
 * product in fp16; where the V scales are small (below 2^-6) they are lifted by an exact
 * power of two first, so that small values keep fp16's relative precision.
 */
kv4_status kv4_decode_attention(const kv4_config *cfg, const kv4_int4_pool *pool,
                                const kv4_int8_side *side, const kv4_batch *batch,
                                const void *q, void *out, float *out_f32, float *lse,
                                void *workspace, size_t ws_bytes, int32_t *err_flag,
                                kv4_stream_t stream);

/*
 * One decode step: kv4_quantize_append of one new token per sequence (new_indptr NULL,
 * total_new = num_seqs; k_new, v_new bf16 [num_seqs][Hkv][128]) followed by
 * kv4_decode_attention, with the same arguments, checks, results and error flags as
 * the two calls made in that order on `stream` (batch->seq_lens are the lengths after
 * the append). The attention's work list depends only on the lengths (and page tables),
 * which the append does not write, so one kernel launch builds it and appends the tokens;
 * with batch->plan_reuse set it only appends. Everything runs on `stream`; the call is
 * asynchronous and allocates nothing.
 */
kv4_status kv4_decode_step(const kv4_config *cfg, const kv4_int4_pool *pool,
                           const kv4_int8_side *side, const kv4_batch *batch,
                           const void *k_new, const void *v_new, const void *q, void *out,
                           float *out_f32, float *lse, void *workspace, size_t ws_bytes,
                           int32_t *err_flag, kv4_stream_t stream);

/*
 * Exact regional softmax merge (ai4snews summary, "Interpretation" para. 3) of partial
 * states. A partial record is head_dim+4 floats: acc[head_dim] (sum of e^(s-m) v),
 * m (max logit, natural-log units), l (sum of e^(s-m)), 2 unused. Record (r, j) of
 * region r and query j sits at partials + (r*group + j)*(head_dim+4).
 * Unit u merges regions region_offsets[u] .. region_offsets[u+1]-1 in that order:
 *   M = max m_r, Lambda = sum l_r e^(m_r-M), O = sum acc_r e^(m_r-M) / Lambda,
 * skipping regions with l = 0. Output (u, j): out/out_f32 at (u*group + j)*head_dim,
 * lse at u*group + j. A unit without live regions yields O = 0 and lse = -inf.
 *   partials, region_offsets: device; head_dim must be 128; group in [1, 8].
 */
kv4_status kv4_regional_merge(const float *partials, const int32_t *region_offsets,
                              int32_t n_units, int32_t group, int32_t head_dim,
                              void *out, float *out_f32, float *lse,
                              kv4_stream_t stream);

/*
 * Decode attention for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this call; it exists for callers of this library
 * that cannot call cudaMalloc (code that must not touch the allocator, e.g. inside a
 * fixed memory pool or a runtime that owns all device memory) and so cannot supply the
 * workspace kv4_decode_attention needs. Same arguments, semantics and results as
 * kv4_decode_attention, minus the workspace: the scratch space is a fixed array of
 * KV4_NOALLOC_SCRATCH_BYTES bytes in the library's device image, which every GPU that
 * loads the library holds until the process exits. Nothing is allocated or freed.
 *   - The call behaves as kv4_decode_attention given that array as a workspace of
 *     KV4_NOALLOC_SCRATCH_BYTES bytes, the fall-back to 64-page chunks included: a batch
 *     that does not fit even then is rejected with KV4_ERR_WORKSPACE_TOO_SMALL.
 *   - The first call on a device looks up the array's device address (with that device
 *     current); make that first call before capturing a stream into a CUDA graph.
 *   - The address is kept for the device's primary context: do not use the call across
 *     cudaDeviceReset (or another teardown of the primary context) in one process.
 *   - All calls share the one array per device: calls whose kernels overlap on the GPU
 *     (different streams without ordering between them) race and give wrong results.
 *     Calls ordered on one stream are safe; each call re-initialises what it reads.
 */
#define KV4_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
kv4_status kv4_decode_attention_noalloc(const kv4_config *cfg, const kv4_int4_pool *pool,
                                        const kv4_int8_side *side, const kv4_batch *batch,
                                        const void *q, void *out, float *out_f32, float *lse,
                                        int32_t *err_flag, kv4_stream_t stream);

/* Size of the fixed scratch array kv4_decode_attention_noalloc uses, in bytes. (The
 * paper has no counterpart.) */
size_t kv4_noalloc_scratch_bytes(void);

/* ---------------------------------------------------------------------------------------
 * Comparison baselines: the same paged decode attention over an unquantised BF16 cache
 * and over an all-INT8 (KV8) cache, for the throughput comparison the pages make between
 * KV4, KV8 and BF16 caches (ai4snews summary, "Interpretation" paras. 1-2: KV8 tracks
 * BF16 closely; replay throughput ratios against BF16). No protected set: cfg's num_sinks
 * and num_recent are ignored (taken as 0); the other cfg fields, the batch (sink_idx and
 * ring_idx unused), the workspace, the error bits and the output contract are those of
 * kv4_decode_attention. KV8 quantises every position with the INT8 quantiser of the
 * protected set (symmetric per token and kv head, fp16 scale = RN(amax/127), codes
 * RNE-clamped to [-127, 127]).
 * ------------------------------------------------------------------------------------- */
typedef enum {
  KV4_BASELINE_BF16 = 1,
  KV4_BASELINE_KV8 = 2
} kv4_baseline_format;

/* Paged baseline cache, per (page, kv head) block of 16 positions:
 *   BF16: k, v: bf16 [num_pages][Hkv][16 octets][16 slots][8]; element (slot t, dim d) at
 *         [d/8][t][d%8] (4 KiB per block); k_scales, v_scales unused (may be NULL).
 *   KV8:  k, v: int8 [num_pages][Hkv][8 strips][16 slots][16]; element (t, d) at
 *         [d/16][t][d%16] (2 KiB per block); k_scales, v_scales: fp16 [num_pages][Hkv][16].
 * All pointers 16-byte aligned device memory owned by the caller. */
typedef struct {
  void *k;
  void *v;
  uint16_t *k_scales;
  uint16_t *v_scales;
  int32_t num_pages;
} kv4_paged_pool;

/* Append new tokens (same CSR contract as kv4_quantize_append): BF16 copies each row into
 * its page slot; KV8 quantises it. Data-dependent errors as for kv4_quantize_append. */
kv4_status kv4_baseline_append(kv4_baseline_format fmt, const kv4_config *cfg,
                               const kv4_paged_pool *pool, const kv4_batch *batch,
                               const void *k_new, const void *v_new, const int32_t *new_indptr,
                               int32_t total_new, int32_t *err_flag, kv4_stream_t stream);

/* Workspace bytes for kv4_baseline_decode_attention (0 on invalid arguments). */
size_t kv4_baseline_workspace_size(const kv4_config *cfg, int32_t num_seqs, int32_t max_seq_len);

/* Decode attention over the baseline cache: O[b, j] = softmax(K q / sqrt(128)) V over
 * positions [0, seq_lens[b]) with K, V the stored bf16 values (BF16) or the dequantised
 * INT8 codes (KV8). Outputs, workspace and errors as for kv4_decode_attention. */
kv4_status kv4_baseline_decode_attention(kv4_baseline_format fmt, const kv4_config *cfg,
                                         const kv4_paged_pool *pool, const kv4_batch *batch,
                                         const void *q, void *out, float *out_f32, float *lse,
                                         void *workspace, size_t ws_bytes, int32_t *err_flag,
                                         kv4_stream_t stream);

/*
 * Testing hook for the error path of the bounded waits. No passage of the pages defines
 * it; it exists so that the library's tests can make a wait give up without any fault.
 * The next kv4_decode_attention, kv4_decode_step or kv4_baseline_decode_attention call
 * made by this host thread -- that one only -- withholds the first shared-memory copy of
 * work item `item` of its attention kernel (nothing is issued for it, so nothing is in
 * flight) and gives each bounded wait of its kernels `wait_limit` attempts (0 keeps the
 * normal limit). The wait on the withheld copy gives up: the call ORs KV4_DEVERR_TIMEOUT
 * into *err_flag, writes that work item's partial state as empty, lets the warp that held
 * it take no further work, and computes the rest of the batch as usual; the call returns
 * normally and the context stays usable. Work items are numbered in the order the
 * attention's work list holds them (full INT4 chunks first, in sequence order). item < 0
 * cancels a pending request.
 */
void kv4_test_withhold_copy(int32_t item, uint32_t wait_limit);

/* Human-readable name of a status code (static string). (Infrastructure of this
 * library: no passage of the pages defines it.) */
const char *kv4_status_string(kv4_status status);

/* Library version: major*10000 + minor*100 + patch. (Infrastructure: no passage.) */
int32_t kv4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KV4_H */
