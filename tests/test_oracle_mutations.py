"""The oracle's pins catch plausible mistakes.

Each of the 35 cases below plants one mistake in the CPU oracle (on the CPU, by replacing one of
its functions for the duration of the case: a dropped term, a wrong sign, index or
operand, another rounding rule, an off-by-one region edge) and checks that the pins of
``test_oracle_pins.py`` named beside it fail. A pin set that let such a mistake through
would let the same mistake in the CUDA path through the parity tests, whose expected
values come from the oracle.

Mistakes that cannot change any result on the inputs the method sees are not listed:
for example rounding the group minimum to fp16 or not (bf16 values in the fp16 normal
range are fp16 values already), or clamping INT8 codes to -128 instead of -127
(|x| / RN(amax / 127) stays below 127.5).
"""
import math

import numpy as np
import pytest

from oracle import kv4_oracle as O
import test_oracle_pins as P

_orig = {name: getattr(O, name) for name in dir(O) if callable(getattr(O, name))}


# --------------------------------------------------------------------------
# the planted mistakes (each a full replacement of one oracle function)
# --------------------------------------------------------------------------

def _to_f16_truncating(x):
    """fp16 conversion rounding toward zero instead of to nearest-even."""
    x = np.clip(np.asarray(x, dtype=np.float32), -O.F16_MAX, O.F16_MAX).astype(np.float64)
    h = x.astype(np.float16)
    over = np.abs(h.astype(np.float64)) > np.abs(x)
    step = np.nextafter(h, np.float16(0))
    return np.where(over, step, h).astype(np.float16)


def _to_f16_unsaturated(x):
    """fp16 conversion that overflows to infinity instead of saturating."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float32).astype(np.float16)


def _int4_with(round_fn=np.rint, levels=15.0, top=15, reciprocal=False, range_f16=False):
    """quantize_int4 with one step changed: the integer rounding, the number of
    levels the range is divided into, the top code of the clamp, the quotient taken as
    a product with the rounded reciprocal of the scale, or the range rounded to fp16
    before the division (the scale rounded twice)."""
    def quantize_int4(x):
        x = np.asarray(x, dtype=np.float32)
        g = x.reshape(x.shape[:-1] + (x.shape[-1] // O.GROUP, O.GROUP))
        mn, mx = g.min(axis=-1), g.max(axis=-1)
        min_h = O.to_f16(mn)
        rng = O.to_f16(mx - mn).astype(np.float32) if range_f16 else mx - mn
        scale_h = O.to_f16(rng / np.float32(levels))
        s32 = scale_h.astype(np.float32)[..., None]
        with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
            num = g - min_h.astype(np.float32)[..., None]
            q = num * (np.float32(1.0) / s32) if reciprocal else num / s32
            codes = np.clip(round_fn(q), 0, top)
        codes = np.where(s32 == 0, 0, codes)
        return codes.reshape(x.shape).astype(np.uint8), scale_h, min_h
    return quantize_int4


def _int8_with(round_fn=np.rint, div=127.0):
    """quantize_int8 with the rounding rule or the divisor of amax changed."""
    def quantize_int8(x):
        x = np.asarray(x, dtype=np.float32)
        scale_h = O.to_f16(np.abs(x).max(axis=-1) / np.float32(div))
        s32 = scale_h.astype(np.float32)[..., None]
        with np.errstate(divide="ignore", invalid="ignore"):
            codes = np.clip(round_fn(x / s32), -127, 127)
        codes = np.where(s32 == 0, 0, codes)
        return codes.astype(np.int8), scale_h
    return quantize_int8


def _near_ties_up(q):
    """Nearest integer, except that a quotient within 2^-9 of a half-integer (but not
    exactly on it) goes to the upper neighbour: a tie rule applied with a tolerance."""
    a = np.abs(q)
    fr = a - np.floor(a)
    near = (np.abs(fr - np.float32(0.5)) <= np.float32(2.0 ** -9)) & (fr != np.float32(0.5))
    return np.where(near, np.sign(q) * np.ceil(a), np.rint(q))


def _half_up(q):
    return np.floor(q + np.float32(0.5))


def _half_away(q):
    return np.sign(q) * np.floor(np.abs(q) + np.float32(0.5))


def _dequant_int4_no_min(codes, scale_h, min_h):
    """code * scale, the group minimum dropped."""
    return _orig["dequant_int4"](codes, scale_h, np.zeros_like(min_h))


def _dequant_int4_one_scale(codes, scale_h, min_h):
    """every group dequantised with group 0's scale and min (wrong group index)."""
    s0 = np.repeat(scale_h[..., :1], scale_h.shape[-1], axis=-1)
    m0 = np.repeat(min_h[..., :1], min_h.shape[-1], axis=-1)
    return _orig["dequant_int4"](codes, s0, m0)


def _regions_recent_short(L, S, R):
    """recent window starting one position late (R - 1 positions)."""
    sink, int4, recent = _orig["regions"](L, S, R)
    if recent[0] < recent[1] and recent[0] > sink[1]:
        recent = (recent[0] + 1, recent[1])
    return sink, int4, recent


def _regions_int4_inclusive(L, S, R):
    """INT4 range closed at L - R, overlapping the recent window."""
    sink, int4, recent = _orig["regions"](L, S, R)
    if int4[0] < int4[1]:
        int4 = (int4[0], min(L, int4[1] + 1))
    return sink, int4, recent


def _attention_with(scale_of_d=lambda d: 1.0 / math.sqrt(d), kv_of=lambda j, G, H: j // G,
                    lse_max=True):
    """Monolithic attention with the softmax scale, the GQA map, or the LSE changed."""
    def attention(q, K, V):
        Hq, D = q.shape
        L, Hkv, _ = K.shape
        G = Hq // Hkv
        out = np.zeros((Hq, D))
        lse = np.full(Hq, -np.inf)
        if L == 0:
            return out, lse
        for j in range(Hq):
            h = kv_of(j, G, Hkv)
            s = K[:, h, :] @ q[j].astype(np.float64) * scale_of_d(D)
            m = s.max()
            e = np.exp(s - m)
            out[j] = (e @ V[:, h, :]) / e.sum()
            lse[j] = (m if lse_max else 0.0) + math.log(e.sum())
        return out, lse
    return attention


def _merge_with(sign=1.0, rescale_acc=True):
    """Regional merge with the rescaling exponent's sign flipped, or the accumulators
    summed without rescaling."""
    def merge_partials(parts):
        live = [(m, l, a) for (m, l, a) in parts if m != -np.inf and l > 0]
        if not live:
            return np.zeros(len(parts[0][2]) if parts else 0), -np.inf
        M = max(m for m, _, _ in live)
        lam = sum(l * math.exp(sign * (m - M)) for m, l, _ in live)
        acc = sum(a * (math.exp(sign * (m - M)) if rescale_acc else 1.0) for m, _, a in live)
        return acc / lam, M + math.log(lam)
    return merge_partials


def _partial_state_unscaled(q_row, K, V):
    """Regional partial state without the 1/sqrt(d) softmax scale."""
    return _orig["partial_state"](q_row * math.sqrt(K.shape[-1]), K, V)


def _pack_int4_swapped(codes):
    """dim 2i in the high nibble instead of the low one."""
    c = codes.reshape(codes.shape[:-1] + (4, 16, 2)).astype(np.uint8)
    return (c[..., 1] | (c[..., 0] << 4)).astype(np.uint8)


def _ring_slot_shifted(pos, R):
    return (pos + 1) % R


def _int4_source_always_a(x, reading="A"):
    """Reading B treated as reading A (the INT4 copy always from the bf16 input)."""
    return x


def _effective_kv_unprotected(k, v, S, R, reading="A"):
    """Every position read from INT4: the protected set ignored."""
    return _orig["effective_kv"](k, v, 0, 0, reading)


def _kv8_from_int4(q, k, v):
    """The all-INT8 reference computed on INT4 copies instead."""
    return _orig["decode_reference"](q, k, v, 0, 0)


def _expected_pages_slot_shifted(rec, L, page_row):
    """Page contents one slot late (position p in slot p % 16 + 1)."""
    pages = _orig["expected_pages"](rec, L, page_row)
    return {pid: tuple(np.roll(a, 1, axis=2 if a.ndim == 4 and a.shape[-1] == 16 else 1)
                       for a in arrs) for pid, arrs in pages.items()}


def _records_v_from_k(k, v, reading="A"):
    """V records quantised from the K stream."""
    return _orig["token_records"](k, k, reading)


def _side_short_context_in_ring(rec, L, S, R):
    """While the context is shorter than the sink count, tokens go to the ring instead
    of the sink store (sink membership decided by the length, not the position)."""
    return _orig["expected_side"](rec, L, S if L >= S else 0, R)


def _side_ring_one_short(rec, L, S, R):
    """A ring that keeps one position fewer than the recent window."""
    return _orig["expected_side"](rec, L, S, R - 1 if R > 1 else R)


def _int8_tensor_amax(x):
    """INT8 scale from the largest magnitude of the whole tensor, not of each row."""
    x = np.asarray(x, dtype=np.float32)
    scale_h = O.to_f16(np.full(x.shape[:-1], np.abs(x).max(), np.float32) / np.float32(127.0))
    s32 = scale_h.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        codes = np.clip(np.rint(x / s32), -127, 127)
    return np.where(s32 == 0, 0, codes).astype(np.int8), scale_h


def _int4_interleaved_groups(x):
    """INT4 groups of every fourth dim instead of 32 consecutive dims."""
    x = np.asarray(x, dtype=np.float32)
    D = x.shape[-1]
    perm = np.arange(D).reshape(D // O.GROUP, O.GROUP).T.reshape(-1)
    codes, scale_h, min_h = _orig["quantize_int4"](x[..., perm])
    return codes[..., np.argsort(perm)], scale_h, min_h


def _pack_int8_transposed(codes):
    """INT8 strips holding every eighth dim instead of 16 consecutive dims."""
    return codes.reshape(codes.shape[:-1] + (16, 8)).swapaxes(-1, -2)


MUTATIONS = {
    # name: (oracle function, replacement, pins that must fail)
    "to_f16 truncates": ("to_f16", _to_f16_truncating,
                         ["test_to_f16_is_round_nearest_even_with_saturation"]),
    "to_f16 overflows to inf": ("to_f16", _to_f16_unsaturated,
                                ["test_to_f16_is_round_nearest_even_with_saturation"]),
    "INT4 rounds half up": ("quantize_int4", _int4_with(round_fn=_half_up),
                            ["test_int4_golden_group_a", "test_exact_ties_round_to_even"]),
    "INT4 rounds half away from zero": ("quantize_int4", _int4_with(round_fn=_half_away),
                                        ["test_int4_golden_group_a",
                                         "test_exact_ties_round_to_even"]),
    "INT4 range over 16 levels": ("quantize_int4", _int4_with(levels=16.0),
                                  ["test_int4_golden_group_a",
                                   "test_int4_codes_are_the_exact_nearest_level"]),
    "INT4 top code 14": ("quantize_int4", _int4_with(top=14),
                         ["test_int4_golden_group_a",
                          "test_int4_reconstruction_bound_and_special_groups"]),
    "INT4 near-ties rounded up": ("quantize_int4", _int4_with(round_fn=_near_ties_up),
                                  ["test_int4_codes_are_the_exact_nearest_level"]),
    "INT4 quotient by reciprocal product": ("quantize_int4", _int4_with(reciprocal=True),
                                            ["test_exact_ties_at_scales_without_an_exact_reciprocal"]),
    "INT4 scale rounded twice": ("quantize_int4", _int4_with(range_f16=True),
                                 ["test_int4_codes_are_the_exact_nearest_level"]),
    "INT8 near-ties rounded up": ("quantize_int8", _int8_with(round_fn=_near_ties_up),
                                  ["test_int8_exact_nearest_and_symmetry"]),
    "INT8 rounds half away from zero": ("quantize_int8", _int8_with(round_fn=_half_away),
                                        ["test_int8_golden_rows", "test_exact_ties_round_to_even"]),
    "INT8 rounds half up": ("quantize_int8", _int8_with(round_fn=_half_up),
                            ["test_exact_ties_round_to_even"]),
    "INT8 scale amax/128": ("quantize_int8", _int8_with(div=128.0),
                            ["test_int8_golden_rows", "test_int8_exact_nearest_and_symmetry"]),
    "INT4 dequant drops the min": ("dequant_int4", _dequant_int4_no_min,
                                   ["test_int4_golden_group_a",
                                    "test_int4_reconstruction_bound_and_special_groups"]),
    "INT4 dequant wrong group": ("dequant_int4", _dequant_int4_one_scale,
                                 ["test_int4_reconstruction_bound_and_special_groups"]),
    "recent window one short": ("regions", _regions_recent_short,
                                ["test_regions_partition_and_protected_bound"]),
    "INT4 region overlaps recent": ("regions", _regions_int4_inclusive,
                                    ["test_regions_partition_and_protected_bound"]),
    "softmax scale 1/d": ("attention", _attention_with(scale_of_d=lambda d: 1.0 / d),
                          ["test_attention_brute_force_tiny",
                           "test_regional_merge_equals_monolithic_softmax"]),
    "GQA map j mod Hkv": ("attention", _attention_with(kv_of=lambda j, G, H: j % H),
                          ["test_attention_brute_force_tiny", "test_attention_gqa_mapping"]),
    "LSE without the max": ("attention", _attention_with(lse_max=False),
                            ["test_attention_closed_forms"]),
    "merge exponent sign flipped": ("merge_partials", _merge_with(sign=-1.0),
                                    ["test_regional_merge_equals_monolithic_softmax"]),
    "merge accumulators not rescaled": ("merge_partials", _merge_with(rescale_acc=False),
                                        ["test_regional_merge_equals_monolithic_softmax"]),
    "partial state unscaled": ("partial_state", _partial_state_unscaled,
                               ["test_regional_merge_equals_monolithic_softmax"]),
    "nibbles swapped": ("pack_int4_token", _pack_int4_swapped,
                        ["test_int4_golden_group_a", "test_expected_pages_layout"]),
    "ring slot shifted": ("ring_slot", _ring_slot_shifted,
                          ["test_ring_window_matches_sequential_appends"]),
    "reading B is reading A": ("int4_source", _int4_source_always_a,
                               ["test_demotion_reading_b"]),
    "protected set ignored": ("effective_kv", _effective_kv_unprotected,
                              ["test_decode_reference_partition_special_cases",
                               "test_all_int8_tracks_bf16_within_derived_bound"]),
    "KV8 reference on INT4": ("decode_reference_kv8", _kv8_from_int4,
                              ["test_baseline_references_reduce_to_pinned_cases"]),
    "page slots shifted": ("expected_pages", _expected_pages_slot_shifted,
                           ["test_expected_pages_layout"]),
    "V records from K": ("token_records", _records_v_from_k,
                         ["test_expected_pages_layout", "test_token_record_layouts_by_hand"]),
    "short context in the ring": ("expected_side", _side_short_context_in_ring,
                                  ["test_ring_window_matches_sequential_appends"]),
    "ring one short": ("expected_side", _side_ring_one_short,
                       ["test_ring_window_matches_sequential_appends"]),
    "INT8 scale per tensor": ("quantize_int8", _int8_tensor_amax,
                              ["test_int8_exact_nearest_and_symmetry"]),
    "INT4 groups interleaved": ("quantize_int4", _int4_interleaved_groups,
                                ["test_int4_golden_group_a", "test_token_record_layouts_by_hand",
                                 "test_int4_codes_are_the_exact_nearest_level"]),
    "INT8 strips transposed": ("pack_int8_token", _pack_int8_transposed,
                               ["test_token_record_layouts_by_hand"]),
}


def _run_pin(name):
    """Run one pin (parametrised pins over all their parameter sets); True if it failed."""
    fn = getattr(P, name)
    marks = getattr(fn, "pytestmark", [])
    params = [m for m in marks if m.name == "parametrize"]
    cases = [()]
    if params:
        cases = [tuple(c) if isinstance(c, (tuple, list)) else (c,) for c in params[0].args[1]]
    for args in cases:
        try:
            fn(*args)
        except (AssertionError, ArithmeticError, ValueError, IndexError, KeyError, TypeError):
            return True
    return False


def test_every_pin_passes_unmutated():
    for _, _, pins in MUTATIONS.values():
        for pin in pins:
            assert not _run_pin(pin), pin


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    target, replacement, pins = MUTATIONS[name]
    monkeypatch.setattr(O, target, replacement)
    missed = [pin for pin in pins if not _run_pin(pin)]
    assert not missed, f"mistake '{name}' in {target} not caught by {missed}"
