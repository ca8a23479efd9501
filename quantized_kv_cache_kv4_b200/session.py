"""Builds a decode batch's KV cache on the device through the library and runs steps.

Plumbing only: torch allocates and moves memory; every quantisation and attention step
runs in libkv4's kernels via :mod:`quantized_kv_cache_kv4_b200.kv4`.

Cache construction for a workload (seq_lens = lengths after step 0's append):
  1. prompt prefill: for a shared-prompt workload, the first sequence of each group
     appends the prompt positions (INT4 prompt pages, the group's sink set, its ring);
  2. fork: the other sequences of the group copy that ring (the prompt's recent window);
  3. context prefill: every sequence appends its own positions up to seq_len - 2;
  4. each decode step s appends position seq_len - 1 + s and attends over seq_len + s.
Without a shared prompt, steps 1-2 are skipped and step 3 starts at position 0.
"""
from __future__ import annotations

import numpy as np
import torch

from . import kv4
from .workload import Workload, make_paging, queries, seq_kv


class DecodeSession:
    def __init__(self, wl: Workload, layer: int = 0, steps: int = 1, device="cuda",
                 chunk_pages: int = 0, keep_streams=(), keep_bits: bool = False,
                 build: bool = True,
                 max_rows_per_call: int = 1 << 20, workspace: torch.Tensor | None = None,
                 demotion: str = "A", prefix: str = "off"):
        self.wl = wl
        self.layer = layer
        self.steps = steps
        self.device = torch.device(device)
        self.paging = make_paging(wl, extra_tokens=steps)
        self.demotion = demotion
        self.cfg = kv4.make_config(wl.num_q_heads, wl.num_kv_heads, wl.num_sinks,
                                   wl.num_recent, chunk_pages, demotion, prefix)
        self.cache = self._allocate_cache()
        B = wl.num_seqs
        self.L0 = wl.seq_lens.astype(np.int64)  # lengths after step 0's append
        dev = self.device
        self.page_table = torch.as_tensor(self.paging.page_table, device=dev)
        self.sink_idx = torch.as_tensor(self.paging.sink_idx, device=dev)
        self.ring_idx = torch.as_tensor(self.paging.ring_idx, device=dev)
        # lengths after the append of step s, for every step
        self.step_lens = torch.as_tensor(
            (self.L0[None, :] + np.arange(steps)[:, None]).astype(np.int32), device=dev)
        self.max_len = int(self.L0.max()) + steps
        self.keep = set(int(b) for b in keep_streams)
        # b -> (k, v) full bf16 streams kept on the host for the oracle: float32 values,
        # or (keep_bits) the bf16 bit patterns as uint16 (half the host memory)
        self.streams = {}
        self.keep_bits = keep_bits
        self.step_k = torch.empty((steps, B, wl.num_kv_heads, wl.head_dim), dtype=torch.bfloat16,
                                  device=dev)
        self.step_v = torch.empty_like(self.step_k)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_rows = max_rows_per_call
        # attention calls reuse the work list the previous call on the shared workspace
        # left (layers after the first of one decode step: same lengths and paging)
        self.plan_reuse = False
        ws = self._workspace_size(B, self.max_len)
        if workspace is not None and workspace.numel() >= ws:
            self.workspace = workspace  # shared with other layers (calls run in stream order)
        else:
            self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.q = torch.stack([queries(wl, s, layer, dev) for s in range(steps)])
        self.out = torch.empty((B, wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16, device=dev)
        if build:
            self.build()

    # ------------------------------------------------------------------ helpers
    def _allocate_cache(self):
        return kv4.allocate_cache(self.cfg, self.paging.num_pages, self.paging.num_sink_sets,
                                  self.paging.num_rings, device=self.device)

    def _workspace_size(self, num_seqs, max_len):
        return kv4.workspace_size(self.cfg, num_seqs, max_len)

    def append(self, batch, k, v, indptr=None, stream=None):
        """Append rows k, v (CSR by indptr, None = one per sequence) into this cache."""
        kv4.quantize_append(self.cache, batch, k, v, indptr, self.err, stream=stream)

    def attend(self, batch, q, out, out_f32=None, lse=None, stream=None):
        """Decode attention of queries q over this cache."""
        kv4.decode_attention(self.cache, batch, q, out, self.workspace, out_f32, lse,
                             self.err, stream=stream)

    def batch(self, lens: torch.Tensor) -> kv4.BatchTensors:
        return kv4.BatchTensors(self.page_table, lens, self.sink_idx, self.ring_idx,
                                self.max_len, self.plan_reuse)

    def _append_rows(self, rows_k, rows_v, counts, lens_after, page_table=None):
        """One append call: rows of all sequences, CSR by `counts`."""
        indptr = np.zeros(len(counts) + 1, dtype=np.int32)
        indptr[1:] = np.cumsum(counts)
        if indptr[-1] == 0:
            return
        dev = self.device
        k = torch.cat(rows_k, 0) if rows_k else None
        v = torch.cat(rows_v, 0) if rows_v else None
        b = kv4.BatchTensors(self.page_table if page_table is None else page_table,
                             torch.as_tensor(lens_after.astype(np.int32), device=dev),
                             self.sink_idx, self.ring_idx, self.max_len)
        self.append(b, k, v, torch.as_tensor(indptr, device=dev))

    def _gen(self, b):
        end = int(self.L0[b]) + self.steps
        k, v = seq_kv(self.wl, b, end, self.layer, self.device)
        if b in self.keep:
            if self.keep_bits:
                self.streams[b] = (k.view(torch.int16).cpu().numpy().view(np.uint16),
                                   v.view(torch.int16).cpu().numpy().view(np.uint16))
            else:
                self.streams[b] = (k.float().cpu().numpy(), v.float().cpu().numpy())
        return k, v

    # ------------------------------------------------------------------ build
    def build(self):
        wl = self.wl
        B = wl.num_seqs
        P = wl.prompt_len if wl.shared_prefix else 0
        lead = self.paging.leaders
        streams = {}
        if P:
            # 1. leaders append the shared prompt
            rows_k, rows_v, counts, lens = [], [], np.zeros(B, np.int64), np.zeros(B, np.int64)
            for b in range(B):
                if lead[b]:
                    k, v = self._gen(b)
                    streams[b] = (k, v)
                    n = min(P, int(self.L0[b]) - 1)
                    rows_k.append(k[:n]); rows_v.append(v[:n])
                    counts[b] = n
                    lens[b] = n
            self._append_rows(rows_k, rows_v, counts, lens)
            # 2. fork the leader's ring to the group's other sequences
            leader_of = {}
            rings = [] if not hasattr(self.cache, "ring_k") else [
                self.cache.ring_k, self.cache.ring_v, self.cache.ring_ks, self.cache.ring_vs]
            for b in range(B):
                g = wl.group_of(b)
                if lead[b]:
                    leader_of[g] = b
            for b in range(B):
                if not lead[b]:
                    src = leader_of[wl.group_of(b)]
                    for t in rings:
                        t[b].copy_(t[src])
        # 3. every sequence appends its own context up to position L0 - 2
        rows_k, rows_v = [], []
        counts = np.zeros(B, np.int64)
        nrows = 0
        for b in range(B):
            if b in streams:
                k, v = streams.pop(b)
            else:
                k, v = self._gen(b)
            L = int(self.L0[b])
            start = P if P else 0
            n = max(0, L - 1 - start)
            rows_k.append(k[start:start + n]); rows_v.append(v[start:start + n])
            counts[b] = n
            nrows += n
            self.step_k[:, b] = k[L - 1:L - 1 + self.steps]
            self.step_v[:, b] = v[L - 1:L - 1 + self.steps]
            if nrows >= self.max_rows or b == B - 1:
                cnt = np.zeros(B, np.int64)
                first = b - len(rows_k) + 1
                cnt[first:b + 1] = counts[first:b + 1]
                self._append_rows(rows_k, rows_v, cnt, np.maximum(self.L0 - 1, 0))
                rows_k, rows_v, nrows = [], [], 0
        torch.cuda.synchronize(self.device)

    # ------------------------------------------------------------------ steps
    def append_step(self, s: int = 0, stream=None):
        self.append(self.batch(self.step_lens[s]), self.step_k[s], self.step_v[s], None,
                    stream=stream)

    def attention_step(self, s: int = 0, out=None, out_f32=None, lse=None, stream=None):
        self.attend(self.batch(self.step_lens[s]), self.q[s], self.out if out is None else out,
                    out_f32, lse, stream=stream)

    def step(self, s: int = 0, **kw):
        self.append_step(s, stream=kw.get("stream"))
        self.attention_step(s, **kw)

    def step_call(self, batch, k, v, q, out, out_f32=None, lse=None, stream=None):
        """One decode step (one new token per sequence) as one kv4.decode_step call:
        append + attention; one launch builds the work list and appends the tokens."""
        kv4.decode_step(self.cache, batch, k, v, q, out, self.workspace, out_f32, lse,
                        self.err, stream=stream)

    def fused_step(self, s: int = 0, out=None, out_f32=None, lse=None, stream=None):
        """Step s through step_call."""
        self.step_call(self.batch(self.step_lens[s]), self.step_k[s], self.step_v[s],
                       self.q[s], self.out if out is None else out, out_f32, lse,
                       stream=stream)

    def check_err(self):
        flag = int(self.err.item())
        if flag:
            raise kv4.KV4Error(f"device error flag {flag}: {kv4.decode_err(flag)}")


class BaselineSession(DecodeSession):
    """The same decode batch over a comparison cache: BF16 (kv4.BASELINE_BF16) or all-INT8
    (kv4.BASELINE_KV8) pages, no protected set. Built and stepped like DecodeSession, with
    the library's baseline append and attention calls."""

    def __init__(self, wl: Workload, fmt: int, **kw):
        self.fmt = fmt
        super().__init__(wl, **kw)

    def _allocate_cache(self):
        return kv4.allocate_baseline_cache(self.fmt, self.cfg, self.paging.num_pages,
                                           device=self.device)

    def _workspace_size(self, num_seqs, max_len):
        return kv4.baseline_workspace_size(self.cfg, num_seqs, max_len)

    def append(self, batch, k, v, indptr=None, stream=None):
        kv4.baseline_append(self.cache, batch, k, v, indptr, self.err, stream=stream)

    def attend(self, batch, q, out, out_f32=None, lse=None, stream=None):
        kv4.baseline_decode_attention(self.cache, batch, q, out, self.workspace, out_f32, lse,
                                      self.err, stream=stream)

    def step_call(self, batch, k, v, q, out, out_f32=None, lse=None, stream=None):
        """The comparison caches have no fused entry point: the two calls in order."""
        self.append(batch, k, v, None, stream=stream)
        self.attend(batch, q, out, out_f32, lse, stream=stream)
