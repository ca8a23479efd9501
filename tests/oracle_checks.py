"""Oracle side of the full-size GPU parity tests, run in worker processes.

Test infrastructure: each task carries one sequence's token stream (bf16 bits), its
query, what the device wrote (the sequence's INT4 pages, its INT8 sink set and ring)
and what it computed (fp32 and bf16 outputs, LSE); the worker rebuilds the records,
pages and decode output with the CPU oracle and reports the comparison. Imports only
numpy and the oracle (no torch, no CUDA), so spawned workers start light.
"""
import numpy as np

from oracle import kv4_oracle as O


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    return np.where(a > 0, 2.0 ** (e - 8), 2.0 ** -133)


def check_sequence(task: dict) -> dict:
    """Pages and side copies byte for byte; with task["attention"], also the attention
    errors for the caller to bound (the tolerance is relative to the largest reference
    output over the sequences checked)."""
    b, L = task["b"], task["L"]
    k = bf16_bits_to_f32(task["k"])[:L]
    v = bf16_bits_to_f32(task["v"])[:L]
    reading = task["reading"]
    S, R = task["S"], task["R"]
    res = {"b": b, "bad": []}
    rec = O.token_records(k, v, reading)
    pages = O.expected_pages(rec, L, task["page_row"])
    dev = task["pages"]  # page id -> (kc, kp, vc, vp) as the device holds them
    for pid, want in pages.items():
        got = dev[pid]
        for name, g, w in zip(("k codes", "k params", "v codes", "v params"), got, want):
            if not np.array_equal(g, w):
                res["bad"].append(f"page {pid} {name}")
    exp = O.expected_side(rec, L, S, R)
    for i, name in enumerate(("sink k", "sink ks", "sink v", "sink vs",
                              "ring k", "ring ks", "ring v", "ring vs")):
        got = task["side"][i]
        if got is not None and not np.array_equal(got, exp[i]):
            res["bad"].append(name)
    if not task["attention"]:
        return res
    oref, lref = O.decode_reference(task["q"], k, v, S, R, reading)
    res["ref_max"] = float(np.abs(oref).max())
    res["e32"] = float(np.abs(task["out32"] - oref).max())
    res["e16_excess"] = float((np.abs(task["out16"] - oref) - bf16_half_ulp(oref)).max())
    res["lse_rel"] = float((np.abs(task["lse"] - lref) / np.maximum(1.0, np.abs(lref))).max())
    return res
