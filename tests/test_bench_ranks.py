"""The multi-rank logic of bench.py on CPU: two gloo ranks, as torchrun would start them.

Each rank runs its own replica batch (same shape, its own seed) and reports its timed
region; rank 0's line carries the max time over ranks and the sum of the units, which is
what `value` divides. Nothing here needs a GPU.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, units = bench.combine_ranks(10.0 + 5.0 * rank, 1000 * (rank + 1), world, "cpu")
        e2e, zero = bench.combine_ranks(20.0 - rank, 0, world, "cpu")
        wl = bench.rank_workload("tiny", rank)
        out.put((rank, ms, units, e2e, zero, wl.seed, tuple(wl.seq_lens)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_summed_units():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        r = out.get(timeout=120)
        got[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        _, ms, units, e2e, zero, _, _ = got[r]
        assert ms == 15.0 and units == 3000.0  # max of 10 and 15 ms; 1000 + 2000 units
        assert e2e == 20.0 and zero == 0.0
    # same shape on every rank, different data
    assert got[0][6] == got[1][6]
    assert got[0][5] != got[1][5]


def test_single_rank_passes_values_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_ranks(12.5, 77, 1, "cpu") == (12.5, 77.0)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line
    with the contract's keys; on the tiny workload it finishes in seconds, no GPU."""
    import json
    import subprocess
    run = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [l for l in run.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["config"]["workload"].startswith("tiny")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def _brute_force_bytes(wl, lens, cache):
    """Position by position: which stored copy every read touches, and its bytes."""
    H, S, R = wl.num_kv_heads, wl.num_sinks, wl.num_recent
    P = wl.prompt_len if wl.shared_prefix else 0
    logical, seen = 0, set()
    for b, L in enumerate(lens):
        g = wl.group_of(b)
        for p in range(int(L)):
            if cache != "kv4":
                nbytes = 512 if cache == "bf16" else 260
                where = ("page", g, p) if p < P else ("page", b, p)
            elif p < S:
                nbytes = 260
                where = ("sink", g if P else b, p)
            elif p >= L - R:
                nbytes = 260
                where = ("ring", b, p)
            else:
                nbytes = 160
                where = ("page", g, p) if p < P else ("page", b, p)
            logical += nbytes * H
            seen.add((where, nbytes))
    unique = sum(nb for _, nb in seen) * H
    io = len(lens) * wl.num_q_heads * wl.head_dim * 4
    return unique + io, logical + io


@pytest.mark.parametrize("cache", ["kv4", "bf16", "kv8"])
def test_algorithmic_bytes_match_a_position_count(cache):
    """The roofline numerator (bench.attention_bytes) against a count of every read,
    with and without shared prompts, sequences shorter than the protected set and
    recent windows reaching into the prompt."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from quantized_kv_cache_kv4_b200 import workload as W
    rng = np.random.default_rng(3)
    cases = [W.custom_workload(rng.integers(1, 700, 12), num_sinks=4, num_recent=32),
             W.custom_workload(rng.integers(65, 500, 12), num_sinks=16, num_recent=128,
                               prompt_len=64, group_seqs=4),
             W.custom_workload([65, 70, 400, 900, 66, 1000, 129, 130], num_sinks=4,
                               num_recent=96, prompt_len=64, group_seqs=4)]
    for wl in cases:
        got = bench.attention_bytes(wl, wl.seq_lens, cache)
        assert got == _brute_force_bytes(wl, wl.seq_lens, cache), (wl.seq_lens, cache)
