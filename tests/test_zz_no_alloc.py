"""kv4_decode_attention_noalloc: decode attention for callers that cannot allocate.

Some callers cannot call cudaMalloc (code that must not touch the device allocator, for
instance inside a fixed memory pool or a runtime that owns all device memory), so they
cannot hand kv4_decode_attention a workspace. This entry point uses a fixed scratch
array in the library's device image instead. The test checks, through the C ABI, that
two calls in a row give the same output as kv4_decode_attention with a caller-supplied
workspace (bit for bit, which is within the attention tolerance used by the parity
tests), after a larger batch has left other data in the array, and that a batch too
large for the array is refused before anything runs.

This file is collected last on purpose: if it fails, every other test has already run.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def mods():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_kv_cache_kv4_b200 import build
    build.build()
    from quantized_kv_cache_kv4_b200 import kv4, session, workload
    return kv4, session, workload


def _noalloc(kv4, sess, batch, out, o32, lse):
    pool, side, bs = sess.cache.pool_struct(), sess.cache.side_struct(), batch.struct()
    return kv4._lib.kv4_decode_attention_noalloc(
        ctypes.byref(sess.cfg), ctypes.byref(pool), ctypes.byref(side), ctypes.byref(bs),
        ctypes.c_void_p(sess.q[0].data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(o32.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(sess.err.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_call_twice(mods):
    """A larger batch first (the 64 x 2048 layer), so that the array holds another call's
    work list and partial states; then the tiny batch twice in a row. The no-allocation
    call runs the same kernels with the same chunk choice as kv4_decode_attention, so its
    outputs must equal the workspace call's bit for bit (bf16 output, fp32 output, LSE),
    on the first call and on the second."""
    kv4, session, W = mods
    for name in ("qwen3-8b-layer", "tiny"):
        wl = W.make_workload(name)
        sess = session.DecodeSession(wl)
        sess.append_step(0)
        B, Hq = wl.num_seqs, wl.num_q_heads
        batch = sess.batch(sess.step_lens[0])
        assert kv4.workspace_size(sess.cfg, B, sess.max_len) <= kv4.noalloc_scratch_bytes()
        ref32 = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
        ref_lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        kv4.decode_attention(sess.cache, batch, sess.q[0], sess.out, sess.workspace, ref32,
                             ref_lse, sess.err)
        torch.cuda.synchronize()
        ref16 = sess.out.clone()
        for call in range(2 if name == "tiny" else 1):
            out = torch.full((B, Hq, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
            o32 = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
            lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
            st = _noalloc(kv4, sess, batch, out, o32, lse)
            assert st == 0, kv4._lib.kv4_status_string(st)
            torch.cuda.synchronize()
            assert torch.equal(out, ref16), (name, call)
            assert torch.equal(o32, ref32), (name, call)
            assert torch.equal(lse, ref_lse), (name, call)
            # and within the tolerance of the parity tests, the same comparison stated loosely
            scale = float(ref32.abs().max())
            assert float((o32 - ref32).abs().max()) <= TOL * scale
        sess.check_err()


def test_noalloc_refuses_a_batch_beyond_the_array(mods):
    kv4, session, W = mods
    wl = W.make_workload("tiny")
    sess = session.DecodeSession(wl)
    cfg = sess.cfg
    # a batch whose workspace would exceed the fixed array: refused on the host
    big = kv4.Batch(sess.page_table.data_ptr(), sess.page_table.shape[1],
                    sess.step_lens[0].data_ptr(), sess.sink_idx.data_ptr(), 0, 200000, 16384)
    assert kv4._lib.kv4_workspace_size(ctypes.byref(cfg), 200000, 16384) > \
        kv4.noalloc_scratch_bytes()
    pool, side = sess.cache.pool_struct(), sess.cache.side_struct()
    st = kv4._lib.kv4_decode_attention_noalloc(
        ctypes.byref(cfg), ctypes.byref(pool), ctypes.byref(side), ctypes.byref(big),
        ctypes.c_void_p(sess.q[0].data_ptr()), ctypes.c_void_p(sess.out.data_ptr()), None, None,
        ctypes.c_void_p(sess.err.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == -4  # KV4_ERR_WORKSPACE_TOO_SMALL
    assert kv4.noalloc_scratch_bytes() == 32 * 1024 * 1024
