"""The oracle-side checker the full-size GPU tests run in worker processes
(`oracle_checks.check_sequence`), exercised on the CPU with "device" values built by the
oracle itself: it must pass them, and must report a planted wrong byte or output."""
import numpy as np

import oracle_checks
from oracle import kv4_oracle as O


def _task(L=77, S=4, R=32, H=2, G=4, seed=5):
    rng = np.random.default_rng(seed)
    # bf16 values as bits (round-to-nearest-even of float32 draws)
    def bf16_bits(a):
        u = a.astype(np.float32).view(np.uint32)
        u = u + 0x7FFF + ((u >> 16) & 1)
        return (u >> 16).astype(np.uint16)
    k = bf16_bits(rng.standard_normal((L, H, 128)))
    v = bf16_bits(rng.standard_normal((L, H, 128)))
    q = oracle_checks.bf16_bits_to_f32(bf16_bits(rng.standard_normal((H * G, 128))))
    kf, vf = oracle_checks.bf16_bits_to_f32(k), oracle_checks.bf16_bits_to_f32(v)
    rec = O.token_records(kf, vf)
    row = rng.permutation(50)[:(L + 15) // 16].astype(np.int32)
    pages = {pid: tuple(a.copy() for a in arrs)
             for pid, arrs in O.expected_pages(rec, L, row).items()}
    side = [a.copy() for a in O.expected_side(rec, L, S, R)]
    o, lse = O.decode_reference(q, kf, vf, S, R)
    return {"b": 0, "L": L, "k": k, "v": v, "reading": "A", "S": S, "R": R, "q": q,
            "page_row": row, "pages": pages, "side": side, "out32": o.astype(np.float32),
            "out16": o.astype(np.float32), "lse": lse.astype(np.float32), "attention": True}


def test_checker_passes_the_oracles_own_values():
    r = oracle_checks.check_sequence(_task())
    assert r["bad"] == []
    assert r["e32"] < 1e-6 * r["ref_max"] and r["lse_rel"] < 1e-6
    assert r["e16_excess"] <= 0


def test_checker_reports_planted_differences():
    t = _task()
    pid = int(t["page_row"][2])
    t["pages"][pid][0][1, 2, 3, 4] ^= 0x10  # one nibble of a K code
    t["side"][6][0, 1, 2, 3, 4] += 1         # one INT8 V code of the ring
    r = oracle_checks.check_sequence(t)
    assert f"page {pid} k codes" in r["bad"] and "ring v" in r["bad"]
    t = _task()
    t["out32"] = t["out32"] + 1e-2
    r = oracle_checks.check_sequence(t)
    assert r["bad"] == [] and r["e32"] > 5e-3
