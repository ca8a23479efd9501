"""Seeded synthetic workloads for paged-INT4 decode attention.

This module only *generates inputs*: sequence lengths, page tables, and the bf16
key/value/query tensors of rollout-shaped decode batches.  It holds none of the
method's arithmetic (no quantisation, no attention), so the CUDA library and the
CPU oracle can both consume its output without sharing any computation.

Shapes follow the KV4-RL pages (ai4snews summary, "Interpretation": 128 groups of
eight responses per iteration, 16,384-token response cap, run-wide mean response
length about 1.45k tokens; Qwen3-4B/8B attention shapes).  The pages publish no
data, so every tensor here is a seeded stand-in with the stated distribution:

* keys/values ~ N(0, 1) (or Student-t with 3 degrees of freedom for the
  long-tail stress case), rounded to bf16 by round-to-nearest-even;
* a few key channels per KV head scaled up (outlier channels), chosen by the rng;
* queries ~ N(0, 1) in bf16.

Random tensors are drawn with ``torch.Generator`` on the requested device, one
independent stream per (workload seed, layer, token stream, tensor kind), so any
single sequence can be regenerated alone (the oracle samples sequences this way).
CUDA and CPU generators produce different numbers for the same seed; a parity
check therefore always takes both sides' inputs from one device's draw.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math

import numpy as np
import torch

PAGE_SIZE = 16
HEAD_DIM = 128


def _seed64(*parts) -> int:
    """Stable 63-bit seed from a tuple of ints/strings (independent of PYTHONHASHSEED)."""
    h = hashlib.blake2b(repr(parts).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


@dataclasses.dataclass
class Workload:
    """One decode-step batch: shapes, protected-set sizes and context lengths.

    ``seq_lens[b]`` is the context length *after* the step's append: the token at
    position ``seq_lens[b] - 1`` is the one appended this step, and attention
    covers positions ``[0, seq_lens[b])``.
    """

    name: str
    num_q_heads: int
    num_kv_heads: int
    num_sinks: int
    num_recent: int
    seq_lens: np.ndarray  # int64 [B]
    seed: int
    kv_dist: str = "normal"  # "normal" | "student_t3"
    outlier_channels: int = 0  # key channels per KV head that are scaled up
    outlier_scale: float = 1.0
    v_scale: float = 1.0  # values drawn with this standard deviation (keys stay at 1)
    v_small_tokens: int = 0  # v_scale applies to the first this many positions (0 = all)
    prompt_len: int = 0  # shared prompt prefix length (multiple of PAGE_SIZE), 0 = none
    group_seqs: int = 1  # sequences sharing one prompt
    num_layers: int = 1
    head_dim: int = HEAD_DIM
    page_size: int = PAGE_SIZE

    @property
    def num_seqs(self) -> int:
        return int(len(self.seq_lens))

    @property
    def gqa(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def shared_prefix(self) -> bool:
        return self.prompt_len > 0 and self.group_seqs > 1

    def group_of(self, b: int) -> int:
        return b // self.group_seqs if self.shared_prefix else b

    def describe(self) -> dict:
        L = self.seq_lens
        return {
            "workload": self.name,
            "num_seqs": self.num_seqs,
            "num_q_heads": self.num_q_heads,
            "num_kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim,
            "page_size": self.page_size,
            "num_sinks": self.num_sinks,
            "num_recent": self.num_recent,
            "num_layers": self.num_layers,
            "context_tokens": int(L.sum()),
            "min_len": int(L.min()),
            "max_len": int(L.max()),
            "mean_len": round(float(L.mean()), 1),
            "kv_dist": self.kv_dist,
            "shared_prompt_len": self.prompt_len if self.shared_prefix else 0,
        }


def make_workload(name: str) -> Workload:
    """The five rollout-shaped workloads (tiny correctness case first)."""
    if name in ("tiny", "1"):
        return Workload(
            name="tiny-4seq-L37-150-300-511-hkv2",
            num_q_heads=8, num_kv_heads=2, num_sinks=4, num_recent=32,
            seq_lens=np.array([37, 150, 300, 511], dtype=np.int64),
            seed=1001, outlier_channels=4, outlier_scale=8.0)
    if name in ("qwen3-8b-layer", "2"):
        return Workload(
            name="qwen3-8b-layer-64seq-L2048",
            num_q_heads=32, num_kv_heads=8, num_sinks=16, num_recent=128,
            seq_lens=np.full(64, 2048, dtype=np.int64),
            seed=1002, outlier_channels=3, outlier_scale=10.0)
    if name in ("rollout", "3"):
        rng = np.random.default_rng(1003)
        sigma = 1.0
        mu = math.log(1450.0) - sigma * sigma / 2.0  # lognormal with mean 1450
        r = np.clip(np.rint(rng.lognormal(mu, sigma, size=1024)), 1, 16384).astype(np.int64)
        return Workload(
            name="rollout-1024seq-128x8-shared256-lognormal1450",
            num_q_heads=32, num_kv_heads=8, num_sinks=16, num_recent=128,
            seq_lens=256 + r, seed=1003, outlier_channels=3, outlier_scale=10.0,
            prompt_len=256, group_seqs=8)
    if name in ("longtail", "4"):
        return Workload(
            name="longtail-128seq-L16384-student-t3",
            num_q_heads=32, num_kv_heads=8, num_sinks=16, num_recent=128,
            seq_lens=np.full(128, 16384, dtype=np.int64),
            seed=1004, kv_dist="student_t3")
    if name in ("qwen3-4b-step", "5"):
        rng = np.random.default_rng(1005)
        return Workload(
            name="qwen3-4b-36layer-512seq-U512-8192",
            num_q_heads=32, num_kv_heads=8, num_sinks=16, num_recent=128,
            seq_lens=rng.integers(512, 8193, size=512).astype(np.int64),
            seed=1005, outlier_channels=3, outlier_scale=10.0, num_layers=36)
    raise ValueError(f"unknown workload {name!r}")


def custom_workload(seq_lens, num_q_heads=8, num_kv_heads=2, num_sinks=4, num_recent=32,
                    seed=7, kv_dist="normal", outlier_channels=0, outlier_scale=1.0,
                    prompt_len=0, group_seqs=1, name="custom", v_scale=1.0,
                    v_small_tokens=0) -> Workload:
    return Workload(name=name, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                    num_sinks=num_sinks, num_recent=num_recent,
                    seq_lens=np.asarray(seq_lens, dtype=np.int64), seed=seed,
                    kv_dist=kv_dist, outlier_channels=outlier_channels,
                    outlier_scale=outlier_scale, v_scale=v_scale,
                    v_small_tokens=v_small_tokens, prompt_len=prompt_len,
                    group_seqs=group_seqs)


# ----------------------------------------------------------------------------
# token streams
# ----------------------------------------------------------------------------

def outlier_channel_ids(wl: Workload, layer: int = 0) -> np.ndarray:
    """[num_kv_heads, outlier_channels] key channel ids that get scaled up."""
    rng = np.random.default_rng(_seed64(wl.seed, layer, "outlier-channels"))
    return np.stack([rng.choice(wl.head_dim, size=wl.outlier_channels, replace=False)
                     for _ in range(wl.num_kv_heads)]) if wl.outlier_channels else \
        np.zeros((wl.num_kv_heads, 0), dtype=np.int64)


def _draw(wl: Workload, n: int, gen: torch.Generator, device) -> torch.Tensor:
    shape = (n, wl.num_kv_heads, wl.head_dim)
    if wl.kv_dist == "normal":
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if wl.kv_dist == "student_t3":
        z = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        chi = torch.randn((3,) + shape, generator=gen, device=device, dtype=torch.float32)
        return z / torch.sqrt((chi * chi).sum(0) / 3.0)
    raise ValueError(wl.kv_dist)


def _stream(wl: Workload, stream_id: int, n: int, layer: int, device):
    """bf16 K, V [n, Hkv, d] for tokens 0..n-1 of one token stream."""
    dev = torch.device(device)
    out = []
    for kind in ("k", "v"):
        gen = torch.Generator(device=dev)
        gen.manual_seed(_seed64(wl.seed, layer, "stream", stream_id, kind))
        x = _draw(wl, n, gen, dev)
        if kind == "k" and wl.outlier_channels:
            ids = torch.as_tensor(outlier_channel_ids(wl, layer), device=dev)
            scale = torch.ones(wl.num_kv_heads, wl.head_dim, device=dev)
            scale.scatter_(1, ids, wl.outlier_scale)
            x = x * scale
        if kind == "v" and wl.v_scale != 1.0:
            if wl.v_small_tokens:
                x[:wl.v_small_tokens] *= wl.v_scale
            else:
                x = x * wl.v_scale
        out.append(x.to(torch.bfloat16))
    return out[0], out[1]


def seq_kv(wl: Workload, b: int, end: int, layer: int = 0, device="cpu", start: int = 0):
    """bf16 K, V [end-start, Hkv, d] of positions [start, end) of sequence ``b``.

    With a shared prompt, positions below ``prompt_len`` come from the prompt
    stream of the sequence's group, the rest from the sequence's own stream.
    """
    if not wl.shared_prefix:
        k, v = _stream(wl, b, end, layer, device)
        return k[start:end], v[start:end]
    P = wl.prompt_len
    ngroups = (wl.num_seqs + wl.group_seqs - 1) // wl.group_seqs
    kp, vp = _stream(wl, wl.group_of(b), min(end, P), layer, device)
    if end <= P:
        return kp[start:end], vp[start:end]
    kr, vr = _stream(wl, ngroups + b, end - P, layer, device)
    k = torch.cat([kp, kr], 0)
    v = torch.cat([vp, vr], 0)
    return k[start:end], v[start:end]


def queries(wl: Workload, step: int = 0, layer: int = 0, device="cpu") -> torch.Tensor:
    """bf16 Q [B, Hq, d] for one decode step."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(_seed64(wl.seed, layer, "q", step))
    q = torch.randn((wl.num_seqs, wl.num_q_heads, wl.head_dim), generator=gen,
                    device=dev, dtype=torch.float32)
    return q.to(torch.bfloat16)


# ----------------------------------------------------------------------------
# paging
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Paging:
    """Page table, sink-set and ring assignment for a workload.

    ``page_table[b, i]`` is the physical page holding positions
    ``[16 i, 16 i + 16)`` of sequence ``b``; unused entries are -1.  With a shared
    prompt, the prompt pages of a group appear in all its sequences' rows.
    Physical pages are a seeded permutation, as after allocator churn.
    """

    page_table: np.ndarray  # int32 [B, max_pages]
    num_pages: int
    sink_idx: np.ndarray  # int32 [B]: INT8 sink set of each sequence
    num_sink_sets: int
    ring_idx: np.ndarray  # int32 [B]: INT8 recent-window ring of each sequence
    num_rings: int
    leaders: np.ndarray  # bool [B]: sequence that owns (writes) its group's prompt pages


def make_paging(wl: Workload, extra_tokens: int = 0, shuffle: bool = True) -> Paging:
    P = wl.page_size
    B = wl.num_seqs
    cap = wl.seq_lens + extra_tokens
    npages = (cap + P - 1) // P
    max_pages = int(npages.max())
    table = np.full((B, max_pages), -1, dtype=np.int64)
    nxt = 0
    leaders = np.ones(B, dtype=bool)
    if wl.shared_prefix:
        assert wl.prompt_len % P == 0, "a shared prompt must fill whole pages"
        pp = wl.prompt_len // P
        group_pages = {}
        for b in range(B):
            g = wl.group_of(b)
            if g not in group_pages:
                group_pages[g] = np.arange(nxt, nxt + pp)
                nxt += pp
            else:
                leaders[b] = False
            table[b, :pp] = group_pages[g]
            own = int(npages[b]) - pp
            table[b, pp:pp + own] = np.arange(nxt, nxt + own)
            nxt += own
        sink_idx = np.array([wl.group_of(b) for b in range(B)], dtype=np.int64)
        num_sink_sets = int(sink_idx.max()) + 1
    else:
        for b in range(B):
            table[b, :npages[b]] = np.arange(nxt, nxt + npages[b])
            nxt += int(npages[b])
        sink_idx = np.arange(B, dtype=np.int64)
        num_sink_sets = B
    num_pages = nxt
    if shuffle:
        perm = np.random.default_rng(_seed64(wl.seed, "page-perm")).permutation(num_pages)
        table = np.where(table >= 0, perm[np.maximum(table, 0)], -1)
    return Paging(page_table=table.astype(np.int32), num_pages=num_pages,
                  sink_idx=sink_idx.astype(np.int32), num_sink_sets=num_sink_sets,
                  ring_idx=np.arange(B, dtype=np.int32), num_rings=B,
                  leaders=leaders)
