"""Thin Python binding of libkv4.so (include/kv4.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
allocates device tensors with PyTorch (plumbing), fills the C structs with raw
pointers and forwards the caller's CUDA stream. There is no fallback: if the library
cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkv4.so")

KV4_OK = 0
STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape",
          -3: "protected set larger than 144 positions", -4: "workspace too small",
          -5: "CUDA error"}
DEVERR = {1: "page id", 2: "seq len", 4: "side index", 8: "q range", 16: "workspace",
          32: "timeout"}
MAX_PROTECTED = 144
HEAD_DIM = 128
PAGE = 16
GROUP = 32

EXPORTS = ("kv4_workspace_size", "kv4_chunk_pages_for", "kv4_quantize_append",
           "kv4_decode_attention", "kv4_decode_step", "kv4_regional_merge",
           "kv4_status_string", "kv4_version",
           "kv4_decode_attention_noalloc", "kv4_noalloc_scratch_bytes",
           "kv4_baseline_append", "kv4_baseline_workspace_size",
           "kv4_baseline_decode_attention", "kv4_test_withhold_copy")

BASELINE_BF16 = 1  # kv4_baseline_format
BASELINE_KV8 = 2


class Config(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("group_size", ctypes.c_int32), ("num_sinks", ctypes.c_int32),
                ("num_recent", ctypes.c_int32), ("chunk_pages", ctypes.c_int32),
                ("demotion", ctypes.c_int32), ("prefix_mode", ctypes.c_int32)]


class Int4Pool(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_params", ctypes.c_void_p), ("v_params", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32)]


class Int8Side(ctypes.Structure):
    _fields_ = [("sink_k", ctypes.c_void_p), ("sink_v", ctypes.c_void_p),
                ("sink_ks", ctypes.c_void_p), ("sink_vs", ctypes.c_void_p),
                ("num_sink_sets", ctypes.c_int32),
                ("ring_k", ctypes.c_void_p), ("ring_v", ctypes.c_void_p),
                ("ring_ks", ctypes.c_void_p), ("ring_vs", ctypes.c_void_p),
                ("num_rings", ctypes.c_int32)]


class Batch(ctypes.Structure):
    _fields_ = [("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int32),
                ("seq_lens", ctypes.c_void_p), ("sink_idx", ctypes.c_void_p),
                ("ring_idx", ctypes.c_void_p), ("num_seqs", ctypes.c_int32),
                ("max_seq_len", ctypes.c_int32), ("plan_reuse", ctypes.c_int32)]


class PagedPool(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32)]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libkv4.so not built at {path}: run "
                          "`python -m quantized_kv_cache_kv4_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.kv4_workspace_size.restype = ctypes.c_size_t
    lib.kv4_workspace_size.argtypes = [ctypes.POINTER(Config), ctypes.c_int32, ctypes.c_int32]
    lib.kv4_chunk_pages_for.restype = ctypes.c_int32
    lib.kv4_chunk_pages_for.argtypes = [ctypes.POINTER(Config), ctypes.c_int32, ctypes.c_int32]
    lib.kv4_quantize_append.restype = ctypes.c_int
    lib.kv4_quantize_append.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Int4Pool),
                                        ctypes.POINTER(Int8Side), ctypes.POINTER(Batch),
                                        P, P, P, ctypes.c_int32, P, P]
    lib.kv4_decode_attention.restype = ctypes.c_int
    lib.kv4_decode_attention.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Int4Pool),
                                         ctypes.POINTER(Int8Side), ctypes.POINTER(Batch),
                                         P, P, P, P, P, ctypes.c_size_t, P, P]
    lib.kv4_decode_step.restype = ctypes.c_int
    lib.kv4_decode_step.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Int4Pool),
                                    ctypes.POINTER(Int8Side), ctypes.POINTER(Batch),
                                    P, P, P, P, P, P, P, ctypes.c_size_t, P, P]
    lib.kv4_regional_merge.restype = ctypes.c_int
    lib.kv4_regional_merge.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       P, P, P, P]
    lib.kv4_decode_attention_noalloc.restype = ctypes.c_int
    lib.kv4_decode_attention_noalloc.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Int4Pool),
                                                 ctypes.POINTER(Int8Side), ctypes.POINTER(Batch),
                                                 P, P, P, P, P, P]
    lib.kv4_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.kv4_noalloc_scratch_bytes.argtypes = []
    lib.kv4_baseline_append.restype = ctypes.c_int
    lib.kv4_baseline_append.argtypes = [ctypes.c_int, ctypes.POINTER(Config),
                                        ctypes.POINTER(PagedPool), ctypes.POINTER(Batch),
                                        P, P, P, ctypes.c_int32, P, P]
    lib.kv4_baseline_workspace_size.restype = ctypes.c_size_t
    lib.kv4_baseline_workspace_size.argtypes = [ctypes.POINTER(Config), ctypes.c_int32,
                                                ctypes.c_int32]
    lib.kv4_baseline_decode_attention.restype = ctypes.c_int
    lib.kv4_baseline_decode_attention.argtypes = [ctypes.c_int, ctypes.POINTER(Config),
                                                  ctypes.POINTER(PagedPool),
                                                  ctypes.POINTER(Batch), P, P, P, P, P,
                                                  ctypes.c_size_t, P, P]
    lib.kv4_test_withhold_copy.restype = None
    lib.kv4_test_withhold_copy.argtypes = [ctypes.c_int32, ctypes.c_uint32]
    lib.kv4_status_string.restype = ctypes.c_char_p
    lib.kv4_status_string.argtypes = [ctypes.c_int]
    lib.kv4_version.restype = ctypes.c_int32
    lib.kv4_version.argtypes = []
    return lib


_lib = load_library()


class KV4Error(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != KV4_OK:
        raise KV4Error(f"{what}: {_lib.kv4_status_string(status).decode()} ({status})")


def _ptr(t):
    """Device pointer of a tensor argument (None -> NULL). The library reads every array
    densely from its first element, so a tensor must be a contiguous CUDA tensor."""
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("kv4 arguments must be contiguous CUDA tensors "
                         f"(got device={t.device}, contiguous={t.is_contiguous()})")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


DEMOTION = {"A": 0, "B": 1}  # kv4_config.demotion
PREFIX = {"off": 0, "shared": 1}  # kv4_config.prefix_mode


def make_config(num_q_heads, num_kv_heads, num_sinks, num_recent, chunk_pages=0,
                demotion="A", prefix="off") -> Config:
    return Config(num_q_heads, num_kv_heads, HEAD_DIM, PAGE, GROUP, num_sinks, num_recent,
                  chunk_pages, DEMOTION[demotion], PREFIX[prefix])


@dataclasses.dataclass
class Cache:
    """Device storage of one layer's cache, in the library's format (see kv4.h)."""

    cfg: Config
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    k_params: torch.Tensor
    v_params: torch.Tensor
    sink_k: torch.Tensor
    sink_v: torch.Tensor
    sink_ks: torch.Tensor
    sink_vs: torch.Tensor
    ring_k: torch.Tensor
    ring_v: torch.Tensor
    ring_ks: torch.Tensor
    ring_vs: torch.Tensor

    @property
    def num_pages(self):
        return self.k_codes.shape[0]

    def pool_struct(self) -> Int4Pool:
        return Int4Pool(self.k_codes.data_ptr(), self.v_codes.data_ptr(),
                        self.k_params.data_ptr(), self.v_params.data_ptr(), self.num_pages)

    def side_struct(self) -> Int8Side:
        return Int8Side(self.sink_k.data_ptr(), self.sink_v.data_ptr(),
                        self.sink_ks.data_ptr(), self.sink_vs.data_ptr(), self.sink_k.shape[0],
                        self.ring_k.data_ptr(), self.ring_v.data_ptr(),
                        self.ring_ks.data_ptr(), self.ring_vs.data_ptr(), self.ring_k.shape[0])


def allocate_cache(cfg: Config, num_pages: int, num_sink_sets: int, num_rings: int,
                   device="cuda") -> Cache:
    """Zero-initialised cache tensors (int8/uint8 codes, fp16 bits as int16)."""
    H = cfg.num_kv_heads
    st = max(1, (cfg.num_sinks + PAGE - 1) // PAGE)
    rt = max(1, (cfg.num_recent + PAGE - 1) // PAGE)
    z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=device)
    return Cache(
        cfg=cfg,
        k_codes=z((num_pages, H, 4, PAGE, 16), torch.uint8),
        v_codes=z((num_pages, H, 4, PAGE, 16), torch.uint8),
        k_params=z((num_pages, H, PAGE, 4, 2), torch.int16),
        v_params=z((num_pages, H, PAGE, 4, 2), torch.int16),
        sink_k=z((max(1, num_sink_sets), H, st, 8, PAGE, 16), torch.int8),
        sink_v=z((max(1, num_sink_sets), H, st, 8, PAGE, 16), torch.int8),
        sink_ks=z((max(1, num_sink_sets), H, st * PAGE), torch.int16),
        sink_vs=z((max(1, num_sink_sets), H, st * PAGE), torch.int16),
        ring_k=z((max(1, num_rings), H, rt, 8, PAGE, 16), torch.int8),
        ring_v=z((max(1, num_rings), H, rt, 8, PAGE, 16), torch.int8),
        ring_ks=z((max(1, num_rings), H, rt * PAGE), torch.int16),
        ring_vs=z((max(1, num_rings), H, rt * PAGE), torch.int16))


@dataclasses.dataclass
class BatchTensors:
    page_table: torch.Tensor  # int32 [B, max_pages]
    seq_lens: torch.Tensor    # int32 [B]
    sink_idx: torch.Tensor    # int32 [B]
    ring_idx: torch.Tensor | None
    max_seq_len: int
    plan_reuse: bool = False  # use the work list the last call on the workspace left

    def struct(self) -> Batch:
        return Batch(self.page_table.data_ptr(), self.page_table.shape[1],
                     self.seq_lens.data_ptr(), self.sink_idx.data_ptr(),
                     0 if self.ring_idx is None else self.ring_idx.data_ptr(),
                     self.seq_lens.shape[0], int(self.max_seq_len), int(self.plan_reuse))


def workspace_size(cfg: Config, num_seqs: int, max_seq_len: int) -> int:
    n = _lib.kv4_workspace_size(ctypes.byref(cfg), num_seqs, max_seq_len)
    if n == 0 and num_seqs > 0:
        raise KV4Error("kv4_workspace_size: invalid arguments")
    return n


def chunk_pages_for(cfg: Config, num_seqs: int, max_seq_len: int) -> int:
    """The INT4 chunk length (pages) the library uses for such a batch."""
    n = _lib.kv4_chunk_pages_for(ctypes.byref(cfg), num_seqs, max_seq_len)
    if n < 0:
        raise KV4Error("kv4_chunk_pages_for: invalid arguments")
    return n


def quantize_append(cache: Cache, batch: BatchTensors, k_new: torch.Tensor, v_new: torch.Tensor,
                    new_indptr: torch.Tensor | None = None, err: torch.Tensor | None = None,
                    stream=None):
    """k_new, v_new: bf16 [rows, Hkv, 128]; new_indptr int32 [B+1] or None (one row per seq)."""
    pool, side, bs = cache.pool_struct(), cache.side_struct(), batch.struct()
    st = _lib.kv4_quantize_append(ctypes.byref(cache.cfg), ctypes.byref(pool), ctypes.byref(side),
                                  ctypes.byref(bs), _ptr(k_new), _ptr(v_new), _ptr(new_indptr),
                                  int(k_new.shape[0]), _ptr(err), _stream(stream))
    _check(st, "kv4_quantize_append")


def decode_attention(cache: Cache, batch: BatchTensors, q: torch.Tensor, out: torch.Tensor,
                     workspace: torch.Tensor, out_f32: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, err: torch.Tensor | None = None,
                     stream=None):
    """q, out: bf16 [B, Hq, 128]; workspace: uint8 device tensor (256-byte aligned)."""
    pool, side, bs = cache.pool_struct(), cache.side_struct(), batch.struct()
    st = _lib.kv4_decode_attention(ctypes.byref(cache.cfg), ctypes.byref(pool),
                                   ctypes.byref(side), ctypes.byref(bs), _ptr(q), _ptr(out),
                                   _ptr(out_f32), _ptr(lse), _ptr(workspace),
                                   workspace.numel(), _ptr(err), _stream(stream))
    _check(st, "kv4_decode_attention")


def decode_step(cache: Cache, batch: BatchTensors, k_new: torch.Tensor, v_new: torch.Tensor,
                q: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                out_f32: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                err: torch.Tensor | None = None, stream=None):
    """One decode step: quantize_append of one token per sequence (k_new, v_new bf16
    [B, Hkv, 128]) then decode_attention, in one library call (one launch builds the
    attention's work list and appends the tokens). batch.lens: lengths after the
    append."""
    pool, side, bs = cache.pool_struct(), cache.side_struct(), batch.struct()
    st = _lib.kv4_decode_step(ctypes.byref(cache.cfg), ctypes.byref(pool), ctypes.byref(side),
                              ctypes.byref(bs), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(out),
                              _ptr(out_f32), _ptr(lse), _ptr(workspace), workspace.numel(),
                              _ptr(err), _stream(stream))
    _check(st, "kv4_decode_step")


def decode_attention_noalloc(cache: Cache, batch: BatchTensors, q: torch.Tensor,
                             out: torch.Tensor, out_f32: torch.Tensor | None = None,
                             lse: torch.Tensor | None = None, err: torch.Tensor | None = None,
                             stream=None):
    """decode_attention without a workspace argument, for callers that cannot allocate
    device memory: the library's fixed scratch array (kv4_noalloc_scratch_bytes()) is
    used instead. Calls that overlap on the GPU race on that array."""
    pool, side, bs = cache.pool_struct(), cache.side_struct(), batch.struct()
    st = _lib.kv4_decode_attention_noalloc(ctypes.byref(cache.cfg), ctypes.byref(pool),
                                           ctypes.byref(side), ctypes.byref(bs), _ptr(q),
                                           _ptr(out), _ptr(out_f32), _ptr(lse), _ptr(err),
                                           _stream(stream))
    _check(st, "kv4_decode_attention_noalloc")


def noalloc_scratch_bytes() -> int:
    return int(_lib.kv4_noalloc_scratch_bytes())


def regional_merge(partials: torch.Tensor, region_offsets: torch.Tensor, group: int,
                   out: torch.Tensor, out_f32: torch.Tensor | None = None,
                   lse: torch.Tensor | None = None, stream=None):
    """partials fp32 [regions, group, 132]; region_offsets int32 [units+1]."""
    n_units = region_offsets.shape[0] - 1
    st = _lib.kv4_regional_merge(_ptr(partials), _ptr(region_offsets), n_units, group, HEAD_DIM,
                                 _ptr(out), _ptr(out_f32), _ptr(lse), _stream(stream))
    _check(st, "kv4_regional_merge")


def decode_err(flag: int) -> list[str]:
    return [name for bit, name in DEVERR.items() if flag & bit]


# ----------------------------------------------------------------------------
# comparison baselines (BF16 and all-INT8 paged caches)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class BaselineCache:
    """Device storage of one layer's BF16 or KV8 paged cache (layouts in kv4.h)."""

    fmt: int
    cfg: Config
    k: torch.Tensor
    v: torch.Tensor
    k_scales: torch.Tensor | None
    v_scales: torch.Tensor | None

    @property
    def num_pages(self):
        return self.k.shape[0]

    def pool_struct(self) -> PagedPool:
        ks = 0 if self.k_scales is None else self.k_scales.data_ptr()
        vs = 0 if self.v_scales is None else self.v_scales.data_ptr()
        return PagedPool(self.k.data_ptr(), self.v.data_ptr(), ks, vs, self.num_pages)


def allocate_baseline_cache(fmt: int, cfg: Config, num_pages: int, device="cuda") -> BaselineCache:
    """Zero-initialised BF16 ([pages, Hkv, 16 octets, 16 slots, 8]) or KV8 ([pages, Hkv,
    8 strips, 16 slots, 16] int8 + fp16 scales [pages, Hkv, 16]) page pool."""
    H = cfg.num_kv_heads
    z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=device)
    if fmt == BASELINE_BF16:
        return BaselineCache(fmt, cfg, z((num_pages, H, 16, PAGE, 8), torch.bfloat16),
                             z((num_pages, H, 16, PAGE, 8), torch.bfloat16), None, None)
    if fmt == BASELINE_KV8:
        return BaselineCache(fmt, cfg, z((num_pages, H, 8, PAGE, 16), torch.int8),
                             z((num_pages, H, 8, PAGE, 16), torch.int8),
                             z((num_pages, H, PAGE), torch.int16),
                             z((num_pages, H, PAGE), torch.int16))
    raise ValueError(f"unknown baseline format {fmt}")


def baseline_workspace_size(cfg: Config, num_seqs: int, max_seq_len: int) -> int:
    n = _lib.kv4_baseline_workspace_size(ctypes.byref(cfg), num_seqs, max_seq_len)
    if n == 0 and num_seqs > 0:
        raise KV4Error("kv4_baseline_workspace_size: invalid arguments")
    return n


def baseline_append(cache: BaselineCache, batch: BatchTensors, k_new: torch.Tensor,
                    v_new: torch.Tensor, new_indptr: torch.Tensor | None = None,
                    err: torch.Tensor | None = None, stream=None):
    pool, bs = cache.pool_struct(), batch.struct()
    st = _lib.kv4_baseline_append(cache.fmt, ctypes.byref(cache.cfg), ctypes.byref(pool),
                                  ctypes.byref(bs), _ptr(k_new), _ptr(v_new), _ptr(new_indptr),
                                  int(k_new.shape[0]), _ptr(err), _stream(stream))
    _check(st, "kv4_baseline_append")


def baseline_decode_attention(cache: BaselineCache, batch: BatchTensors, q: torch.Tensor,
                              out: torch.Tensor, workspace: torch.Tensor,
                              out_f32: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                              err: torch.Tensor | None = None, stream=None):
    pool, bs = cache.pool_struct(), batch.struct()
    st = _lib.kv4_baseline_decode_attention(cache.fmt, ctypes.byref(cache.cfg),
                                            ctypes.byref(pool), ctypes.byref(bs), _ptr(q),
                                            _ptr(out), _ptr(out_f32), _ptr(lse), _ptr(workspace),
                                            workspace.numel(), _ptr(err), _stream(stream))
    _check(st, "kv4_baseline_decode_attention")
