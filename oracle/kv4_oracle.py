"""CPU oracle for KV4-RL decode attention over a paged INT4 + bounded INT8 KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module; only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference arm
of ``bench.py`` use it.  It shares no code with the CUDA library.

What it computes, and which passage each step follows (pages on arXiv 2610.14448,
"KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4 KV Cache
Quantization"):

* Whole context stored in calibration-free INT4, with INT8 copies of a bounded
  protected set (attention sinks + recent window, at most 144 positions), read by
  an exact regional softmax merge -- ai4snews summary, "Interpretation" para. 3;
  aimodeling article, section "INT4 as the base, INT8 insurance for critical
  positions" (paged INT4 format, INT8 side cache).
* Calibration-free INT4 quantisation: kipquest abstract ("calibration-free INT4 KV
  quantization"); ai4snews "Synopsis".  The pages give no bit-level formula; the
  scheme used (per-token asymmetric uint4 in groups of 32 along head_dim, fp16
  scale and min, round-half-even; symmetric per-token INT8 with an fp16 scale) is
  the plainest reading consistent with "calibration-free": every token is
  quantised from its own values only.

Numeric conventions (readings where the pages are silent):

* Inputs are bf16 values carried in float32 arrays (exact).
* Every floating-point step that *decides an integer code or a stored fp16
  parameter* is taken in IEEE binary32 with round-to-nearest-even, in exactly the
  order written below; fp16 conversion is round-to-nearest-even with saturation to
  +-65504.  The CUDA kernels take the same decisions in the same precision, so the
  codes are unique and must match bit for bit.
* Dequantisation, logits, softmax and the merge are evaluated in float64.
* Softmax scale is 1/sqrt(head_dim); query head j reads KV head j // G.

Parity pins for every function live in ``tests/test_oracle_pins.py`` and the
hand-worked fixtures under ``tests/golden/``.
"""
from __future__ import annotations

import math

import numpy as np

F16_MAX = np.float32(65504.0)
GROUP = 32          # INT4 group size along head_dim
PAGE = 16           # tokens per page / per INT8 tile
MAX_PROTECTED = 144  # bound on |sinks + recent| (ai4snews "Interpretation" para. 3)


# ----------------------------------------------------------------------------
# quantisers
# ----------------------------------------------------------------------------

def to_f16(x) -> np.ndarray:
    """Round float32 values to fp16 (nearest-even), saturating at +-65504."""
    x = np.asarray(x, dtype=np.float32)
    return np.clip(x, -F16_MAX, F16_MAX).astype(np.float16)


def quantize_int4(x: np.ndarray):
    """Per-token asymmetric uint4 quantisation in groups of 32 along the last axis.

    For each group of 32 values: mn, mx = min, max;
      min_h   = fp16(mn)
      scale_h = fp16(fp32(fp32(mx - mn) / 15))
      code    = clamp(rne(fp32(fp32(x - min_h) / scale_h)), 0, 15), or 0 if scale_h == 0.
    Returns codes uint8 [..., D], scale fp16 [..., D/32], min fp16 [..., D/32].
    """
    x = np.asarray(x, dtype=np.float32)
    D = x.shape[-1]
    assert D % GROUP == 0
    g = x.reshape(x.shape[:-1] + (D // GROUP, GROUP))
    mn = g.min(axis=-1)
    mx = g.max(axis=-1)
    min_h = to_f16(mn)
    with np.errstate(over="ignore"):
        rng = mx - mn  # fp32, may overflow to inf for huge inputs -> scale saturates
    scale_h = to_f16(rng / np.float32(15.0))
    num = g - min_h.astype(np.float32)[..., None]
    s32 = scale_h.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = num / s32
        codes = np.clip(np.rint(q), 0, 15)
    codes = np.where(s32 == 0, 0, codes)
    return codes.reshape(x.shape).astype(np.uint8), scale_h, min_h


def quantize_int8(x: np.ndarray):
    """Symmetric per-token INT8 over the last axis.

      scale_h = fp16(fp32(amax / 127)),  code = clamp(rne(fp32(x / scale_h)), -127, 127).
    Returns codes int8 [..., D], scale fp16 [...].
    """
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale_h = to_f16(amax / np.float32(127.0))
    s32 = scale_h.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        codes = np.clip(np.rint(x / s32), -127, 127)
    codes = np.where(s32 == 0, 0, codes)
    return codes.astype(np.int8), scale_h


def dequant_int4(codes, scale_h, min_h) -> np.ndarray:
    """code * scale + min per group, in float64."""
    codes = np.asarray(codes)
    D = codes.shape[-1]
    c = codes.reshape(codes.shape[:-1] + (D // GROUP, GROUP)).astype(np.float64)
    out = c * scale_h.astype(np.float64)[..., None] + min_h.astype(np.float64)[..., None]
    return out.reshape(codes.shape)


def dequant_int8(codes, scale_h) -> np.ndarray:
    return np.asarray(codes).astype(np.float64) * scale_h.astype(np.float64)[..., None]


# ----------------------------------------------------------------------------
# the protected set and the region partition
# ----------------------------------------------------------------------------

def check_protection(S: int, R: int) -> None:
    if S < 0 or R < 0:
        raise ValueError("sink and recent counts must be non-negative")
    if S + R > MAX_PROTECTED:
        raise ValueError(f"protected set S+R={S + R} exceeds {MAX_PROTECTED} positions")


def regions(L: int, S: int, R: int):
    """Half-open position ranges (sink, int4, recent) of a context of length L.

    sink = [0, min(S, L)), recent = [max(S, L - R), L), int4 = [S, L - R) when
    L - R > S.  The three are disjoint and cover [0, L).
    """
    check_protection(S, R)
    sink = (0, min(S, L))
    lo = max(S, L - R)
    recent = (lo, L) if lo < L else (L, L)
    int4 = (S, L - R) if L - R > S else (sink[1], sink[1])
    return sink, int4, recent


def protected_mask(L: int, S: int, R: int) -> np.ndarray:
    (s0, s1), _, (r0, r1) = regions(L, S, R)
    m = np.zeros(L, dtype=bool)
    m[s0:s1] = True
    m[r0:r1] = True
    return m


def ring_slot(pos: int, R: int) -> int:
    """Slot of the recent-window ring that holds position ``pos``."""
    return pos % R


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def int4_source(x: np.ndarray, reading: str = "A") -> np.ndarray:
    """The values a position's INT4 copy is quantised from.

    Reading A (the one built by default): the bf16 input itself -- "keeps the whole
    context in paged INT4" (ai4snews summary, "Interpretation" para. 3), so every position
    is written to INT4 when it is appended.  Reading B: the position's INT8 copy,
    dequantised -- the INT4 copy is made when the position is demoted out of the recent
    window, from what the INT8 side cache holds (aimodeling article, "INT4 as the base,
    INT8 insurance for critical positions").  code * scale of an INT8 copy has at most 18
    significant bits, so the float32 value below is exact."""
    if reading == "A":
        return x
    if reading != "B":
        raise ValueError(f"unknown demotion reading {reading!r}")
    c8, s8 = quantize_int8(x)
    return (c8.astype(np.float32) * s8.astype(np.float32)[..., None]).astype(np.float32)


def effective_kv(k: np.ndarray, v: np.ndarray, S: int, R: int, reading: str = "A"):
    """Values the cache yields for each position: INT8 dequant where protected,
    INT4 dequant elsewhere.  k, v: float32 (bf16 values) [L, Hkv, D] -> float64.
    reading: where the INT4 copies come from (see int4_source)."""
    L = k.shape[0]
    prot = protected_mask(L, S, R)
    out = []
    for x in (k, v):
        c4, s4, m4 = quantize_int4(int4_source(x, reading))
        y = dequant_int4(c4, s4, m4)
        if prot.any():
            c8, s8 = quantize_int8(x[prot])
            y[prot] = dequant_int8(c8, s8)
        out.append(y)
    return out[0], out[1]


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """Monolithic softmax attention of one decode query against L keys.

    q: [Hq, D]; K, V: [L, Hkv, D] (float64); query head j uses KV head j // G.
    Returns O [Hq, D] float64 and lse [Hq] (natural log of the softmax denominator
    including the running max), O = 0 and lse = -inf when L == 0.
    """
    Hq, D = q.shape
    L, Hkv, _ = K.shape
    G = Hq // Hkv
    O = np.zeros((Hq, D))
    lse = np.full(Hq, -np.inf)
    if L == 0:
        return O, lse
    qq = q.astype(np.float64)
    for j in range(Hq):
        h = j // G
        s = K[:, h, :] @ qq[j] / math.sqrt(D)
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        O[j] = (e @ V[:, h, :]) / l
        lse[j] = m + math.log(l)
    return O, lse


def decode_reference(q, k, v, S: int, R: int, reading: str = "A"):
    """KV4-RL decode output for one sequence: quantise -> dequantise -> softmax.

    q float32 [Hq, D]; k, v float32 [L, Hkv, D] (the whole token stream of the
    sequence including the token appended this step)."""
    K, V = effective_kv(k, v, S, R, reading)
    return attention(q, K, V)


# ----------------------------------------------------------------------------
# comparison baselines: the same decode attention over a BF16 cache and over an
# all-INT8 (KV8) cache.  The pages compare KV4 against both: KV8 "tracks BF16
# closely" (ai4snews summary, "Interpretation" para. 2) and the replay throughput
# ratios are quoted against BF16 (ai4snews summary, "Interpretation" paras. 1-2).
# ----------------------------------------------------------------------------

def decode_reference_bf16(q, k, v):
    """Decode output over an unquantised BF16 cache: plain softmax attention on the
    bf16 values themselves.  q float32 [Hq, D]; k, v float32 (bf16 values) [L, Hkv, D]."""
    return attention(q, k.astype(np.float64), v.astype(np.float64))


def decode_reference_kv8(q, k, v):
    """Decode output over an all-INT8 cache: every position quantised with the INT8
    quantiser of the protected set (symmetric, per token and kv head, fp16 scale),
    dequantised, then softmax attention."""
    out = []
    for x in (k, v):
        c8, s8 = quantize_int8(x)
        out.append(dequant_int8(c8, s8))
    return attention(q, out[0], out[1])


def partial_state(q_row: np.ndarray, K: np.ndarray, V: np.ndarray):
    """Unnormalised softmax state of one query over one region of keys.

    K, V: [n, D] float64.  Returns (m, l, acc): m = max logit, l = sum exp(s - m),
    acc = sum exp(s - m) v.  An empty region is (-inf, 0, 0)."""
    D = K.shape[-1]
    if K.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(D)
    s = K @ q_row.astype(np.float64) / math.sqrt(D)
    m = s.max()
    e = np.exp(s - m)
    return m, e.sum(), e @ V


def merge_partials(parts):
    """Exact log-sum-exp merge of regional softmax states (ai4snews "Interpretation"
    para. 3, "exact regional softmax merge").

    M = max_r m_r; Lambda = sum_r l_r e^(m_r - M); O = sum_r acc_r e^(m_r - M) / Lambda.
    Empty regions (m = -inf) are skipped.  Returns (O, lse = M + ln Lambda)."""
    live = [(m, l, a) for (m, l, a) in parts if m != -np.inf and l > 0]
    if not live:
        D = len(parts[0][2]) if parts else 0
        return np.zeros(D), -np.inf
    M = max(m for m, _, _ in live)
    lam = sum(l * math.exp(m - M) for m, l, _ in live)
    acc = sum(a * math.exp(m - M) for m, _, a in live)
    return acc / lam, M + math.log(lam)


# ----------------------------------------------------------------------------
# storage format (byte layout shared with the CUDA library by specification)
# ----------------------------------------------------------------------------
#
# INT4 pool, per (page, kv head):
#   codes  [4 groups][16 slots][16 bytes]   byte i of (group g, slot t) holds the codes
#          of dims 32g+2i (low nibble) and 32g+2i+1 (high nibble) of the token in slot t
#   params [16 slots][4 groups][2] fp16     (scale, min)
# INT8 side store, per (set, kv head, tile of 16 slots):
#   codes  [8 strips][16 slots][16 bytes]   byte i of (strip c, slot t) = code of dim 16c+i
#   scales [16 slots] fp16

def pack_int4_token(codes: np.ndarray) -> np.ndarray:
    """codes uint8 [..., 128] -> strip bytes uint8 [..., 4, 16]."""
    c = codes.reshape(codes.shape[:-1] + (4, 16, 2)).astype(np.uint8)
    return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8)


def pack_int8_token(codes: np.ndarray) -> np.ndarray:
    """codes int8 [..., 128] -> strip bytes int8 [..., 8, 16]."""
    return codes.reshape(codes.shape[:-1] + (8, 16))


def f16_bits(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float16).view(np.uint16)


def token_records(k: np.ndarray, v: np.ndarray, reading: str = "A"):
    """Per-position stored records of a token stream (INT4 copies per `reading`).

    Returns a dict of arrays indexed by position:
      k4, v4   uint8  [L, Hkv, 4, 16]   INT4 strips
      kp, vp   uint16 [L, Hkv, 4, 2]    (scale, min) fp16 bits
      k8, v8   int8   [L, Hkv, 8, 16]   INT8 strips
      ks, vs   uint16 [L, Hkv]          INT8 scale fp16 bits
    """
    out = {}
    for name, x in (("k", k), ("v", v)):
        c4, s4, m4 = quantize_int4(int4_source(x, reading))
        out[name + "4"] = pack_int4_token(c4)
        out[name + "p"] = np.stack([f16_bits(s4), f16_bits(m4)], axis=-1)
        c8, s8 = quantize_int8(x)
        out[name + "8"] = pack_int8_token(c8)
        out[name + "s"] = f16_bits(s8)
    return out


def expected_pages(rec, L: int, page_row: np.ndarray):
    """INT4 pool contents of one sequence's pages after positions [0, L) were appended.

    Returns {page id: (kc [Hkv,4,16,16], kp [Hkv,16,4,2], vc, vp)}; slots past L are 0."""
    H = rec["k4"].shape[1]
    pages = {}
    for i in range((L + PAGE - 1) // PAGE):
        pid = int(page_row[i])
        kc = np.zeros((H, 4, PAGE, 16), np.uint8)
        vc = np.zeros((H, 4, PAGE, 16), np.uint8)
        kp = np.zeros((H, PAGE, 4, 2), np.uint16)
        vp = np.zeros((H, PAGE, 4, 2), np.uint16)
        for t in range(PAGE):
            pos = i * PAGE + t
            if pos >= L:
                break
            kc[:, :, t, :] = rec["k4"][pos]
            vc[:, :, t, :] = rec["v4"][pos]
            kp[:, t] = rec["kp"][pos]
            vp[:, t] = rec["vp"][pos]
        pages[pid] = (kc, kp, vc, vp)
    return pages


def expected_side(rec, L: int, S: int, R: int):
    """INT8 sink store and recent ring of one sequence after positions [0, L).

    Sinks hold positions [0, min(S, L)) in slots 0..; ring slot pos % R holds the
    latest position written there, i.e. the window [max(S, L-R), L); slots never
    written are 0.  Returns (sink_codes_k, sink_scales_k, sink_codes_v, ...,
    ring_codes_k, ring_scales_k, ring_codes_v, ring_scales_v) with tile-padded
    slot axes: codes [Hkv, tiles, 8, 16 slots, 16], scales [Hkv, tiles*16]."""
    H = rec["k8"].shape[1]
    st = max(1, (S + PAGE - 1) // PAGE)
    rt = max(1, (R + PAGE - 1) // PAGE)
    out = []
    for tiles, positions, slot_of in (
            (st, range(0, min(S, L)), lambda p: p),
            (rt, range(max(S, L - R), L), lambda p: ring_slot(p, R))):
        for name in ("k", "v"):
            codes = np.zeros((H, tiles, 8, PAGE, 16), np.int8)
            scales = np.zeros((H, tiles * PAGE), np.uint16)
            for pos in positions:
                s = slot_of(pos)
                codes[:, s // PAGE, :, s % PAGE, :] = rec[name + "8"][pos]
                scales[:, s] = rec[name + "s"][pos]
            out += [codes, scales]
    return tuple(out)
