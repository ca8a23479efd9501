/* Sizes and field offsets of the C ABI's structs as the C compiler lays them out;
 * the CPU test suite compares them with the Python binding's ctypes structures. Prints
 * one "name value" pair per line. */
#include <stddef.h>
#include <stdio.h>

#include "kv4.h"

#define SIZE(T) printf("sizeof %s %zu\n", #T, sizeof(T))
#define OFF(T, f) printf("offsetof %s.%s %zu\n", #T, #f, offsetof(T, f))

int main(void) {
  SIZE(kv4_config);
  OFF(kv4_config, num_q_heads); OFF(kv4_config, num_kv_heads); OFF(kv4_config, head_dim);
  OFF(kv4_config, page_size); OFF(kv4_config, group_size); OFF(kv4_config, num_sinks);
  OFF(kv4_config, num_recent); OFF(kv4_config, chunk_pages); OFF(kv4_config, demotion);
  OFF(kv4_config, prefix_mode);
  SIZE(kv4_int4_pool);
  OFF(kv4_int4_pool, k_codes); OFF(kv4_int4_pool, v_codes); OFF(kv4_int4_pool, k_params);
  OFF(kv4_int4_pool, v_params); OFF(kv4_int4_pool, num_pages);
  SIZE(kv4_int8_side);
  OFF(kv4_int8_side, sink_k); OFF(kv4_int8_side, sink_v); OFF(kv4_int8_side, sink_ks);
  OFF(kv4_int8_side, sink_vs); OFF(kv4_int8_side, num_sink_sets); OFF(kv4_int8_side, ring_k);
  OFF(kv4_int8_side, ring_v); OFF(kv4_int8_side, ring_ks); OFF(kv4_int8_side, ring_vs);
  OFF(kv4_int8_side, num_rings);
  SIZE(kv4_batch);
  OFF(kv4_batch, page_table); OFF(kv4_batch, max_pages); OFF(kv4_batch, seq_lens);
  OFF(kv4_batch, sink_idx); OFF(kv4_batch, ring_idx); OFF(kv4_batch, num_seqs);
  OFF(kv4_batch, max_seq_len); OFF(kv4_batch, plan_reuse);
  SIZE(kv4_paged_pool);
  OFF(kv4_paged_pool, k); OFF(kv4_paged_pool, v); OFF(kv4_paged_pool, k_scales);
  OFF(kv4_paged_pool, v_scales); OFF(kv4_paged_pool, num_pages);
  return 0;
}
