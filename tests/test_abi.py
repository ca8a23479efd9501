"""The C-ABI library loads, exports every symbol include/kv4.h declares, and validates
arguments on the host (these calls return before touching CUDA, so they run without a
GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kv4.h")


@pytest.fixture(scope="module")
def kv4():
    from quantized_kv_cache_kv4_b200 import build
    build.build()
    from quantized_kv_cache_kv4_b200 import kv4 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kv4_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for want in ("kv4_quantize_append", "kv4_decode_attention", "kv4_decode_step",
                 "kv4_regional_merge", "kv4_workspace_size", "kv4_status_string",
                 "kv4_version"):
        assert want in names


def test_library_exports_every_declared_symbol(kv4):
    lib = ctypes.CDLL(kv4.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", kv4.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (kv4_\w+)", out))
    assert set(declared_functions()) <= exported


def test_status_strings_and_version(kv4):
    lib = kv4._lib
    assert lib.kv4_version() == 500
    assert lib.kv4_status_string(0) == b"ok"
    assert b"144" in lib.kv4_status_string(-3)
    assert lib.kv4_status_string(-99) == b"unknown status"


def _cfg(kv4, **kw):
    d = dict(num_q_heads=32, num_kv_heads=8, num_sinks=16, num_recent=128, chunk_pages=0)
    raw_demotion = kw.pop("demotion", None)  # ints: written to the struct as they are
    raw_prefix = kw.pop("prefix_mode", None)
    d.update(kw)
    c = kv4.make_config(**d)
    if raw_demotion is not None:
        c.demotion = raw_demotion
    if raw_prefix is not None:
        c.prefix_mode = raw_prefix
    return c


def test_workspace_size_host_only(kv4):
    c = _cfg(kv4, chunk_pages=32)
    n1 = kv4.workspace_size(c, 64, 2048)
    n2 = kv4.workspace_size(c, 128, 2048)
    assert 0 < n1 < n2
    assert n1 % 256 == 0
    # partial records dominate: >= 64 seqs * 8 heads * 4 q heads * 132 floats * (1 + chunks)
    assert n1 >= 64 * 8 * 4 * 132 * 4 * (1 + 5)
    bad = _cfg(kv4, num_sinks=100, num_recent=45)
    assert kv4._lib.kv4_workspace_size(ctypes.byref(bad), 4, 100) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(num_sinks=16, num_recent=129), -3),
    (dict(num_sinks=145, num_recent=0), -3),
    (dict(num_q_heads=30), -2),
    (dict(num_q_heads=128, num_kv_heads=8), -2),
    (dict(chunk_pages=65), -2),
    (dict(demotion=2), -1),
    (dict(demotion=-1), -1),
    (dict(prefix_mode=2), -1),
    (dict(prefix_mode=-1), -1),
    (dict(num_sinks=-1), -1),
])
def test_config_rejected_before_launch(kv4, kw, status):
    c = _cfg(kv4, **kw)
    pool, side, batch = kv4.Int4Pool(), kv4.Int8Side(), kv4.Batch()
    st = kv4._lib.kv4_decode_attention(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                       ctypes.byref(batch), None, None, None, None, None, 0,
                                       None, None)
    assert st == status
    st = kv4._lib.kv4_quantize_append(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                      ctypes.byref(batch), None, None, None, 0, None, None)
    assert st == status


def test_bad_shapes_and_pointers_rejected(kv4):
    c = _cfg(kv4)
    c.head_dim = 64
    pool, side, batch = kv4.Int4Pool(), kv4.Int8Side(), kv4.Batch()
    st = kv4._lib.kv4_decode_attention(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                       ctypes.byref(batch), None, None, None, None, None, 0,
                                       None, None)
    assert st == -2
    c = _cfg(kv4)
    st = kv4._lib.kv4_decode_attention(ctypes.byref(c), None, None, None, None, None, None, None,
                                       None, 0, None, None)
    assert st == -1
    # null pool pointers
    batch = kv4.Batch(0, 4, 0, 0, 0, 2, 100)
    st = kv4._lib.kv4_decode_attention(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                       ctypes.byref(batch), None, None, None, None, None, 0,
                                       None, None)
    assert st == -1
    # misaligned codes pointer
    pool = kv4.Int4Pool(1 << 20 | 8, 1 << 20, 1 << 20, 1 << 20, 10)
    batch = kv4.Batch(1 << 20, 4, 1 << 20, 1 << 20, 0, 2, 100)
    side = kv4.Int8Side(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1, 1 << 20, 1 << 20, 1 << 20,
                        1 << 20, 1)
    st = kv4._lib.kv4_decode_attention(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                       ctypes.byref(batch), None, None, None, None, None, 0,
                                       None, None)
    assert st == -1


def test_merge_argument_checks(kv4):
    lib = kv4._lib
    assert lib.kv4_regional_merge(None, None, 4, 4, 64, None, None, None, None) == -2
    assert lib.kv4_regional_merge(None, None, 4, 0, 128, None, None, None, None) == -1
    assert lib.kv4_regional_merge(None, None, 4, 9, 128, None, None, None, None) == -1
    assert lib.kv4_regional_merge(None, None, 0, 4, 128, None, None, None, None) == 0
    assert lib.kv4_regional_merge(None, None, 2, 4, 128, None, None, None, None) == -1


def test_automatic_chunk_splits_small_batches_finer(kv4):
    auto, c64 = _cfg(kv4), _cfg(kv4, chunk_pages=64)
    # a small batch gets a finer split (more partial states) than 64-page chunks ...
    assert kv4.workspace_size(auto, 2, 1000) > kv4.workspace_size(c64, 2, 1000)
    # ... a large one gets 64-page chunks
    assert kv4.workspace_size(auto, 1024, 14348) == kv4.workspace_size(c64, 1024, 14348)


def test_automatic_chunk_length(kv4):
    """The automatic chunk length (kv4_chunk_pages_for): within 8..64; the configured length
    when one is set; 64 pages for large batches; for batches whose entries fit one round of
    the 1776 resident warps of the persistent grid, the shortest length that keeps them in
    one round (64 x 2048: 120 INT4 pages per kv-head pair -> 5 chunks of 24; 32 x 4096:
    248 pages -> 12 chunks of 21); the shortest length for a handful of sequences."""
    c = _cfg(kv4)
    assert kv4.chunk_pages_for(_cfg(kv4, chunk_pages=32), 2, 1000) == 32
    assert kv4.chunk_pages_for(c, 64, 2049) == 24
    assert kv4.chunk_pages_for(c, 32, 4097) == 21
    assert kv4.chunk_pages_for(c, 1024, 14349) == 64
    assert kv4.chunk_pages_for(c, 128, 16385) == 64
    assert kv4.chunk_pages_for(c, 2, 1000) == 8
    for B in (1, 7, 100, 600, 3000):
        for L in (0, 150, 5000, 100000):
            assert 8 <= kv4.chunk_pages_for(c, B, L) <= 64, (B, L)
    # one round: the entries (two kv heads per warp: 4 slots per sequence, one protected
    # entry per slot) at the chosen length fit the resident warps, one page shorter not
    for B, L in ((64, 2049), (32, 4097), (16, 8193)):
        pages = (L - 128 - 1) // 16 - 16 // 16 + 1
        C = kv4.chunk_pages_for(c, B, L)
        entries = lambda C: B * 4 * (-(-pages // C)) + B * 4
        assert entries(C) <= 1776 < entries(C - 1), (B, L, C)
    bad = _cfg(kv4, num_sinks=100, num_recent=100)
    assert kv4._lib.kv4_chunk_pages_for(ctypes.byref(bad), 4, 100) == -1


def test_workspace_too_small_is_reported(kv4):
    c = _cfg(kv4)
    # too small even for 64-page chunks, the fallback of the automatic choice
    need = kv4.workspace_size(_cfg(kv4, chunk_pages=64), 2, 1000)
    pool = kv4.Int4Pool(1 << 20, 1 << 20, 1 << 20, 1 << 20, 10)
    side = kv4.Int8Side(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1, 1 << 20, 1 << 20, 1 << 20,
                        1 << 20, 2)
    batch = kv4.Batch(1 << 20, 64, 1 << 20, 1 << 20, 0, 2, 1000)
    st = kv4._lib.kv4_decode_attention(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                       ctypes.byref(batch), ctypes.c_void_p(1 << 20),
                                       ctypes.c_void_p(1 << 20), None, None,
                                       ctypes.c_void_p(1 << 20), need - 256, None, None)
    assert st == -4


def test_decode_step_argument_checks(kv4):
    """kv4_decode_step checks the append's and the attention's arguments before it
    creates or launches anything (no device needed for these)."""
    lib = kv4._lib
    P = ctypes.c_void_p
    good = P(1 << 20)

    def call(c, pool, side, batch, k, v, ws_bytes):
        return lib.kv4_decode_step(ctypes.byref(c), ctypes.byref(pool), ctypes.byref(side),
                                   ctypes.byref(batch), k, v, good, good, None, None, good,
                                   ws_bytes, None, None)
    pool = kv4.Int4Pool(1 << 20, 1 << 20, 1 << 20, 1 << 20, 10)
    side = kv4.Int8Side(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1, 1 << 20, 1 << 20, 1 << 20,
                        1 << 20, 2)
    batch = kv4.Batch(1 << 20, 64, 1 << 20, 1 << 20, 0, 2, 1000)
    need = kv4.workspace_size(_cfg(kv4, chunk_pages=64), 2, 1000)
    c = _cfg(kv4)
    c.head_dim = 64
    assert call(c, pool, side, batch, good, good, need) == -2
    c = _cfg(kv4, num_sinks=100, num_recent=100)
    assert call(c, pool, side, batch, good, good, need) == -3
    c = _cfg(kv4)
    assert call(c, pool, side, batch, None, good, need) == -1        # no new K
    assert call(c, pool, side, batch, P((1 << 20) + 8), good, need) == -1  # misaligned K rows
    assert call(c, pool, side, batch, good, good, need - 256) == -4  # workspace too small
    empty = kv4.Batch(1 << 20, 64, 1 << 20, 1 << 20, 0, 0, 1000)
    assert call(c, pool, side, empty, None, None, 0) == 0             # nothing to do


def test_baseline_argument_checks(kv4):
    lib = kv4._lib
    c = _cfg(kv4)
    none_prot = _cfg(kv4, num_sinks=0, num_recent=0)
    # the baselines ignore the protected set and read no shared prefix: same workspace as
    # KV4-RL without either
    assert kv4.baseline_workspace_size(c, 64, 2048) == kv4.workspace_size(none_prot, 64, 2048)
    pool = kv4.PagedPool(1 << 20, 1 << 20, 1 << 20, 1 << 20, 10)
    batch = kv4.Batch(1 << 20, 64, 1 << 20, 0, 0, 2, 1000)
    call = lambda fmt, p=pool: lib.kv4_baseline_decode_attention(
        fmt, ctypes.byref(c), ctypes.byref(p), ctypes.byref(batch), ctypes.c_void_p(1 << 20),
        ctypes.c_void_p(1 << 20), None, None, ctypes.c_void_p(1 << 20), 1 << 30, None, None)
    assert call(3) == -1 and call(0) == -1                # unknown format
    no_scales = kv4.PagedPool(1 << 20, 1 << 20, 0, 0, 10)
    assert call(kv4.BASELINE_KV8, no_scales) == -1        # KV8 needs its scales
    misaligned = kv4.PagedPool((1 << 20) + 8, 1 << 20, 0, 0, 10)
    assert call(kv4.BASELINE_BF16, misaligned) == -1
    # too small a workspace is reported before anything is launched
    st = lib.kv4_baseline_decode_attention(
        kv4.BASELINE_BF16, ctypes.byref(c), ctypes.byref(pool), ctypes.byref(batch),
        ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 20), None, None,
        ctypes.c_void_p(1 << 20), 256, None, None)
    assert st == -4


def test_plain_c_program_uses_the_abi(kv4, tmp_path):
    """tests/c_abi_check.c, compiled with gcc against the header alone and linked to the
    library, runs the host-answered calls from C."""
    exe = tmp_path / "c_abi_check"
    lib_dir = os.path.dirname(kv4.LIB_PATH)
    build = subprocess.run(
        ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
         os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", lib_dir, "-lkv4",
         "-Wl,-rpath," + lib_dir, "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr


def test_binding_structs_match_the_c_layout(kv4, tmp_path):
    """The ctypes structures of the Python binding against the C compiler's layout of
    the header's structs (sizes and every field offset)."""
    exe = tmp_path / "c_abi_layout"
    build = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I",
                            os.path.join(ROOT, "include"),
                            os.path.join(ROOT, "tests", "c_abi_layout.c"), "-o", str(exe)],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60).stdout
    c_layout = dict((k, int(v)) for k, v in (line.rsplit(" ", 1) for line in out.splitlines()))
    py = {"kv4_config": kv4.Config, "kv4_int4_pool": kv4.Int4Pool,
          "kv4_int8_side": kv4.Int8Side, "kv4_batch": kv4.Batch,
          "kv4_paged_pool": kv4.PagedPool}
    checked = 0
    for key, val in c_layout.items():
        kind, name = key.split(" ", 1)
        if kind == "sizeof":
            assert ctypes.sizeof(py[name]) == val, name
        else:
            struct, field = name.split(".")
            assert getattr(py[struct], field).offset == val, name
        checked += 1
    assert checked == 5 + 10 + 5 + 10 + 8 + 5


def test_binding_refuses_host_or_strided_tensors(kv4):
    """The binding passes bare pointers, so it refuses tensors the library would misread."""
    import torch
    assert kv4._ptr(None) is None
    with pytest.raises(ValueError):
        kv4._ptr(torch.zeros(4, 4))  # host memory



def _prototypes():
    """{name: (return type, [parameter declarations])} of the header's functions."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    out = {}
    for m in re.finditer(r"([A-Za-z_][\w \t\*]*?)\b(kv4_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text):
        params = [" ".join(p.split()) for p in m.group(3).split(",")]
        out[m.group(2)] = (" ".join(m.group(1).split()), [] if params == ["void"] else params)
    return out


def test_binding_signatures_match_the_header(kv4):
    """Every function the binding declares takes as many parameters as the header's
    prototype, each of the same kind and width: pointers (and the stream handle) as
    pointers, int32_t as 32-bit, size_t as size_t, enums as int; and returns the
    prototype's type."""
    protos = _prototypes()
    assert set(protos) == set(kv4.EXPORTS)
    ptr_types = (ctypes.c_void_p, ctypes._Pointer)

    def kind(ct):
        if ct is None:
            return "void"
        if ct in (ctypes.c_void_p, ctypes.c_char_p) or issubclass(ct, ptr_types):
            return "pointer"
        return {ctypes.c_int32: "int32", ctypes.c_int: "int32", ctypes.c_uint32: "uint32",
                ctypes.c_size_t: "size_t"}[ct]

    def c_kind(decl):
        if "*" in decl or decl.startswith("kv4_stream_t"):
            return "pointer"
        if decl.startswith("size_t"):
            return "size_t"
        if decl == "void":
            return "void"
        if decl.split()[0] in ("int32_t", "kv4_status", "kv4_baseline_format"):
            return "int32"
        if decl.split()[0] == "uint32_t":
            return "uint32"
        raise AssertionError(f"unclassified parameter {decl!r}")

    for name, (ret, params) in protos.items():
        fn = getattr(kv4._lib, name)
        assert len(fn.argtypes) == len(params), name
        for decl, ct in zip(params, fn.argtypes):
            assert kind(ct) == c_kind(decl), (name, decl, ct)
        assert kind(fn.restype) == c_kind(ret), (name, ret, fn.restype)


def test_workspace_fallback_to_longest_chunks_always_fits(kv4):
    """A workspace sized for (num_seqs, max_seq_len) with the automatic chunk choice also
    holds any smaller or equal batch split into 64-page chunks, the fallback the call
    takes when that batch's own automatic split would need more room (automatic sizes
    themselves are not monotone: longer sequences get longer chunks); and 64-page sizes
    grow with the batch. Checked on random shapes for four head configurations."""
    import numpy as np
    rng = np.random.default_rng(3)
    for hq, hkv, s, r in ((32, 8, 16, 128), (8, 2, 4, 32), (16, 2, 0, 0), (12, 3, 7, 13)):
        auto = _cfg(kv4, num_q_heads=hq, num_kv_heads=hkv, num_sinks=s, num_recent=r)
        c64 = _cfg(kv4, num_q_heads=hq, num_kv_heads=hkv, num_sinks=s, num_recent=r,
                   chunk_pages=64)
        for _ in range(200):
            B1, L1 = int(rng.integers(1, 3000)), int(rng.integers(0, 20000))
            B2, L2 = int(rng.integers(1, B1 + 1)), int(rng.integers(0, L1 + 1))
            big = kv4.workspace_size(auto, B1, L1)
            assert big >= kv4.workspace_size(c64, B2, L2), (hq, hkv, B1, L1, B2, L2)
            assert kv4.workspace_size(c64, B1, L1) >= kv4.workspace_size(c64, B2, L2)
