"""GPU parity of the comparison baselines (BF16 and all-INT8 paged caches) against the
oracle, through the C ABI.

* KV8 pages: every code and scale bit-exact (the INT8 quantiser of the protected set,
  applied to every position); BF16 pages: the input bits, in the documented layout.
* Attention: the tolerance of the KV4-RL parity tests (2e-3 x max|O_ref| for fp32
  output; plus half a bf16 ulp for bf16 output; LSE within 2e-3 x max(1, |lse|)).
"""
import numpy as np
import pytest
import torch

from oracle import kv4_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_kv_cache_kv4_b200 import build
    build.build()


def _mods():
    from quantized_kv_cache_kv4_b200 import kv4, session, workload
    return kv4, session, workload


def bf16_half_ulp(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    return np.where(a > 0, 2.0 ** (e - 8), 2.0 ** -133)


def reference(fmt, sess, b, step=0):
    kv4 = _mods()[0]
    k, v = sess.streams[b]
    L = int(sess.L0[b]) + step
    q = sess.q[step, b].float().cpu().numpy()
    if fmt == kv4.BASELINE_BF16:
        return O.decode_reference_bf16(q, k[:L], v[:L])
    return O.decode_reference_kv8(q, k[:L], v[:L])


def check(fmt, sess, seqs, step=0):
    B, Hq = sess.wl.num_seqs, sess.wl.num_q_heads
    o32 = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    sess.attention_step(step, out_f32=o32, lse=lse)
    torch.cuda.synchronize()
    o16, o32, lse = sess.out.float().cpu().numpy(), o32.cpu().numpy(), lse.cpu().numpy()
    refs = {b: reference(fmt, sess, b, step) for b in seqs}
    scale = max(max(np.abs(r[0]).max() for r in refs.values()), 1e-30)
    for b, (oref, lref) in refs.items():
        e32 = np.abs(o32[b] - oref).max()
        assert e32 <= TOL * scale, (b, e32, scale)
        assert np.all(np.abs(o16[b] - oref) <= TOL * scale + bf16_half_ulp(oref)), b
        assert np.all(np.abs(lse[b] - lref) <= TOL * np.maximum(1, np.abs(lref))), b
    sess.check_err()


def check_pages(fmt, sess, seqs):
    """Every stored page of the given sequences against the oracle / the input bits."""
    kv4 = _mods()[0]
    c = sess.cache
    pt = sess.page_table.cpu().numpy()
    K, V = c.k.cpu(), c.v.cpu()
    if fmt == kv4.BASELINE_KV8:
        K, V = K.numpy(), V.numpy()
        KS, VS = c.k_scales.cpu().numpy().view(np.uint16), c.v_scales.cpu().numpy().view(np.uint16)
    else:
        K, V = K.view(torch.int16).numpy(), V.view(torch.int16).numpy()
    for b in seqs:
        k, v = sess.streams[b]
        L = int(sess.L0[b])
        for which, (x, store) in enumerate(((k[:L], K), (v[:L], V))):
            for p in range((L + 15) // 16):
                page = pt[b, p]
                rows = x[16 * p:16 * p + 16]  # [n, Hkv, 128]
                n = rows.shape[0]
                if fmt == kv4.BASELINE_KV8:
                    codes, sc = O.quantize_int8(rows)  # [n, Hkv, 128], [n, Hkv]
                    got = store[page][:, :, :n, :]     # [Hkv, 8 strips, n, 16]
                    want = codes.reshape(n, -1, 8, 16).transpose(1, 2, 0, 3)
                    assert np.array_equal(got, want.astype(np.int8)), (b, p, which)
                    gsc = (KS if which == 0 else VS)[page][:, :n]
                    assert np.array_equal(gsc, O.f16_bits(sc).T), (b, p, which)
                else:
                    bits = torch.from_numpy(rows.astype(np.float32)).to(torch.bfloat16)
                    bits = bits.view(torch.int16).numpy()     # [n, Hkv, 128]
                    got = store[page][:, :, :n, :]            # [Hkv, 16 octets, n, 8]
                    want = bits.reshape(n, -1, 16, 8).transpose(1, 2, 0, 3)
                    assert np.array_equal(got, want), (b, p, which)


def make(fmt, wl, keep=None, **kw):
    _, session, _ = _mods()
    keep = range(wl.num_seqs) if keep is None else keep
    s = session.BaselineSession(wl, fmt, keep_streams=keep, **kw)
    s.append_step(0)
    torch.cuda.synchronize()
    return s


FORMATS = [1, 2]  # kv4.BASELINE_BF16, kv4.BASELINE_KV8
IDS = ["bf16", "kv8"]

CASES = [
    # (name, lens, Hq, Hkv, chunk_pages)
    ("short", [1, 2, 15, 16, 17, 33, 100], 8, 2, 0),
    ("gqa1", [40, 333], 4, 4, 0),
    ("gqa8", [40, 333], 16, 2, 0),
    ("chunk3", [700, 40, 260], 8, 2, 3),
    ("chunk64", [2100, 1030, 40], 8, 2, 64),
]


@pytest.mark.parametrize("fmt", FORMATS, ids=IDS)
@pytest.mark.parametrize("name,lens,Hq,Hkv,C", CASES, ids=[c[0] for c in CASES])
def test_baseline_small_cases(fmt, name, lens, Hq, Hkv, C):
    W = _mods()[2]
    wl = W.custom_workload(lens, num_q_heads=Hq, num_kv_heads=Hkv, seed=41)
    sess = make(fmt, wl, chunk_pages=C)
    check_pages(fmt, sess, range(wl.num_seqs))
    check(fmt, sess, range(wl.num_seqs))


@pytest.mark.parametrize("fmt", FORMATS, ids=IDS)
def test_baseline_tiny_steps_and_shared_prompt(fmt):
    W = _mods()[2]
    wl = W.make_workload("tiny")
    sess = make(fmt, wl, steps=3)
    check(fmt, sess, range(wl.num_seqs), 0)
    for s in (1, 2):
        sess.append_step(s)
        torch.cuda.synchronize()
        check(fmt, sess, range(wl.num_seqs), s)
    wl2 = W.custom_workload([300, 420, 150, 600], seed=9, prompt_len=64, group_seqs=2)
    sess2 = make(fmt, wl2)
    check_pages(fmt, sess2, range(4))
    check(fmt, sess2, range(4))


@pytest.mark.parametrize("fmt", FORMATS, ids=IDS)
def test_baseline_full_size_sampled(fmt):
    """The rollout batch in the benchmark's configuration, sampled sequences."""
    W = _mods()[2]
    wl = W.make_workload("rollout")
    rng = np.random.default_rng(5)
    keep = sorted(set(rng.choice(wl.num_seqs, 6, replace=False).tolist()) | {int(np.argmax(wl.seq_lens))})
    sess = make(fmt, wl, keep=keep)
    check(fmt, sess, keep)
