"""Benchmark: batched decode steps of paged INT4 + INT8-protected attention on B200.

One step = the whole hot path for one batch: kv4_decode_step, i.e. the quantise-append
of one new token per sequence (INT4 page write, INT8 copy, demotion out of the recent
window) followed by the decode attention (INT8 protected partials, split-K INT4
partials, exact regional merge), in one call per layer. The attention is also timed as
the separate kv4_decode_attention call, for the roofline. The workload defaults to the 1024-sequence async-rollout batch (128 groups x 8
responses sharing a 256-token prompt, lognormal response lengths with mean 1450).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl kv4|reference]
                  [--launch graph|eager]

The timed steps are replayed from CUDA graphs captured once per step (the same kernels
on the same per-step inputs, without host launch gaps between them); the eager numbers
are reported beside them.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own full batch (data-parallel
rollout replicas, no collective in the data path: weak scaling); the timed region is the
max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attention tokens*KV-heads/s"
UNIT = "tokens*kv_heads/s"


# ----------------------------------------------------------------------------
# workload accounting (host arithmetic on lengths only)
# ----------------------------------------------------------------------------

DTYPE = {"kv4": "f16-mma/f32-acc, int4/int8 codes",
         "kv8": "f16-mma/f32-acc, int8 codes (comparison cache)",
         "bf16": "bf16-mma/f32-acc, bf16 cache (comparison cache)"}
CALL = {"kv4": "kv4_decode_attention", "kv8": "kv4_baseline_decode_attention(KV8)",
        "bf16": "kv4_baseline_decode_attention(BF16)"}


def units_per_step(wl, lens) -> int:
    """Context tokens x KV heads attended in one step."""
    return int(np.asarray(lens, dtype=np.int64).sum()) * wl.num_kv_heads


def attention_bytes(wl, lens, cache="kv4"):
    """Algorithmic HBM bytes of one attention call: (unique, logical).

    Per token and KV head: 160 B when read from INT4 (64 B K codes + 16 B K params +
    the same for V), 260 B when read from INT8 (128 B codes + 2 B scale, K and V).
    Plus the query read and the output write (bf16). `logical` counts every sequence's
    reads; `unique` counts each stored byte read once: with a shared prompt, a group's
    sink set and the prompt positions of its shared INT4 pages once for the group (a
    prompt position inside a member's recent window is read from that member's own
    ring). Comparison caches: 512 B per token and head for BF16, 260 B for KV8, at every
    position; a group's shared prompt positions counted once in `unique`."""
    lens = np.asarray(lens, dtype=np.int64)
    H = wl.num_kv_heads
    io = lens.size * wl.num_q_heads * wl.head_dim * 2 * 2
    G = wl.group_seqs if wl.shared_prefix else 1
    P = wl.prompt_len if wl.shared_prefix else 0
    groups = [lens[g:g + G] for g in range(0, lens.size, G)]
    if cache in ("bf16", "kv8"):
        per = 512 if cache == "bf16" else 260
        logical = int(lens.sum()) * per * H
        unique = sum(int(min(P, gl.max())) + int(np.maximum(0, gl - P).sum())
                     for gl in groups) * per * H
        return int(unique + io), int(logical + io)
    S, R = wl.num_sinks, wl.num_recent
    prot = np.minimum(lens, S + R)
    int4 = np.maximum(0, lens - S - R)
    logical = int((int4 * 160 + prot * 260).sum()) * H
    unique = 0
    for gl in groups:
        ring = np.maximum(0, gl - np.maximum(S, gl - R))  # recent window: per sequence
        if P:  # sink set per group; INT4 prompt pages shared, the rest per sequence
            sink = int(min(S, gl.max()))
            shared4 = max(0, int(min(P, (gl - R).max())) - S)
            own4 = np.maximum(0, gl - R - max(P, S))
            unique += sink * 260 + shared4 * 160 + int((ring * 260 + own4 * 160).sum())
        else:
            sink = np.minimum(S, gl)
            own4 = np.maximum(0, gl - R - S)
            unique += int(((sink + ring) * 260 + own4 * 160).sum())
    return int(unique * H + io), int(logical + io)


def time_prefill(sess, wl, dev, max_rows=1 << 20, reps=5):
    """Bulk prefill through the append call: the context rows [0, L-1) of the first
    sequences (up to max_rows rows) re-appended in one CSR call (the cache ends as it
    was). Returns a dict with rows, mean ms per call and algorithmic GB/s (read bf16 K/V,
    write the INT4 records and the INT8 copies of protected positions)."""
    import torch
    from quantized_kv_cache_kv4_b200.workload import seq_kv
    B, H = wl.num_seqs, wl.num_kv_heads
    L0 = wl.seq_lens.astype(np.int64)
    ks, vs, counts, n = [], [], np.zeros(B, np.int64), 0
    for b in range(B):
        if n >= max_rows:
            break
        m = int(L0[b]) - 1
        k, v = seq_kv(wl, b, m, sess.layer, dev)
        ks.append(k); vs.append(v)
        counts[b] = m
        n += m
    k, v = torch.cat(ks), torch.cat(vs)
    del ks, vs
    indptr = np.zeros(B + 1, dtype=np.int32)
    indptr[1:] = np.cumsum(counts)
    lens = torch.as_tensor(np.where(counts > 0, L0 - 1, 0).astype(np.int32), device=dev)
    batch = sess.batch(lens)
    ip = torch.as_tensor(indptr, device=dev)
    S, R = wl.num_sinks, wl.num_recent
    prot = sum(min(int(c), S + R) for c in counts if c > 0)
    nbytes = n * H * (2 * 2 * wl.head_dim + 160) + prot * H * 260
    if getattr(sess, "fmt", None) is not None:  # comparison cache: bf16 or int8 copy
        per = 512 if sess.fmt == 1 else 260
        nbytes = n * H * (2 * 2 * wl.head_dim + per)
    sess.append(batch, k, v, ip)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        sess.append(batch, k, v, ip)
    e1.record()
    torch.cuda.synchronize(dev)
    sess.check_err()
    ms = e0.elapsed_time(e1) / reps
    return {"rows": int(n), "ms": ms, "gbs": nbytes / (ms / 1000.0) / 1e9,
            "bytes_per_call": int(nbytes)}


def append_bytes(wl) -> int:
    """Per step: read bf16 K/V of the new token, write INT4 record (+ INT8 copy)."""
    return wl.num_seqs * wl.num_kv_heads * (2 * 2 * wl.head_dim + 160 + 260)


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------

def oracle_sample(wl, budget_s: float, start_seq: int = 0, cache: str = "kv4",
                  demotion: str = "A"):
    """Time the oracle's decode output (quantise -> dequantise -> softmax attention; for a
    comparison cache its BF16 / KV8 reference) on consecutive sequences of the workload
    until `budget_s` of CPU time is used. For the KV4-RL cache the oracle's quantiser
    alone (the stored records of every position: what the append writes) is timed on the
    same sequences too. Returns (units, seconds, description, threads, quantise seconds
    or None)."""
    import torch
    from oracle import kv4_oracle as O
    from quantized_kv_cache_kv4_b200.workload import queries, seq_kv
    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    q_all = queries(wl, 0, 0, "cpu").float().numpy()
    units, spent, seqs = 0, 0.0, []
    quant = 0.0 if cache == "kv4" else None
    b = start_seq
    while spent < budget_s and len(seqs) < wl.num_seqs:
        bb = b % wl.num_seqs
        L = int(wl.seq_lens[bb])
        k, v = seq_kv(wl, bb, L, 0, "cpu")
        k, v = k.float().numpy(), v.float().numpy()
        t0 = time.perf_counter()
        if cache == "bf16":
            O.decode_reference_bf16(q_all[bb], k, v)
        elif cache == "kv8":
            O.decode_reference_kv8(q_all[bb], k, v)
        else:
            O.decode_reference(q_all[bb], k, v, wl.num_sinks, wl.num_recent, demotion)
        spent += time.perf_counter() - t0
        if quant is not None:
            t0 = time.perf_counter()
            O.token_records(k, v, demotion)
            quant += time.perf_counter() - t0
        units += L * wl.num_kv_heads
        seqs.append(bb)
        b += 1
    fn = {"bf16": "decode_reference_bf16", "kv8": "decode_reference_kv8"}.get(
        cache, "decode_reference")
    desc = (f"oracle {fn} (fp64 numpy: quantise every position, dequantise, "
            f"softmax attention) on {len(seqs)} sequence(s) of the workload "
            f"({units // wl.num_kv_heads} context tokens)")
    return units, spent, desc, threads, quant


def bench_config(wl, cache, world):
    """The `config` both arms print: the workload, the cache, how L2 is kept from serving
    the timed reads, and the data parallelism (so the two arms' lines compare key for key)."""
    ub, _ = attention_bytes(wl, wl.seq_lens, cache)
    return {"workload": wl.name, **wl.describe(), "cache": cache,
            "l2": "inputs larger than L2: the cache read per step is "
                  f"{ub / 1e9:.2f} GB (L2 is 126 MB)",
            "parallelism": f"dp{world} (independent replica batches)"}


def output_check(sess, step, nseq=8, seed=5):
    """The attention output of one decode step (in sess.out) against the oracle on a
    seeded sample of sequences: the worst error of the bf16 output beyond half a bf16 ulp
    of the reference, relative to the sample's max |O_ref|, and whether it is within the
    2e-3 tolerance."""
    from oracle import kv4_oracle as O
    from quantized_kv_cache_kv4_b200.workload import seq_kv
    wl = sess.wl
    rng = np.random.default_rng(seed)
    seqs = sorted(rng.choice(wl.num_seqs, size=min(nseq, wl.num_seqs), replace=False).tolist())
    out = sess.out.float().cpu().numpy()
    refs = {}
    for b in seqs:
        L = int(sess.L0[b]) + step
        # drawn as the session drew it (the whole stream, then the positions in use): a
        # stream's values can depend on its drawn length (the Student-t draws)
        k, v = seq_kv(wl, b, int(sess.L0[b]) + sess.steps, sess.layer, sess.device)
        k, v = k[:L], v[:L]
        q = sess.q[step, b].float().cpu().numpy()
        refs[b] = O.decode_reference(q, k.float().cpu().numpy(), v.float().cpu().numpy(),
                                     wl.num_sinks, wl.num_recent, sess.demotion)[0]
    scale = max(float(np.abs(r).max()) for r in refs.values())
    worst = 0.0
    for b, ref in refs.items():
        a = np.abs(ref)
        half_ulp = np.where(a > 0, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-38))) - 8), 0.0)
        worst = max(worst, float((np.abs(out[b] - ref) - half_ulp).max()) / scale)
    return {"step": int(step), "sequences": len(seqs), "max_err_over_scale": worst,
            "tol": 2e-3, "passed": bool(worst <= 2e-3),
            "what": "bf16 output of the last timed step (layer 0) against the oracle, beyond "
                    "half a bf16 ulp, relative to max |O_ref| of the sample"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = rank_workload(args.workload, 0, args.sinks, args.recent)
    total_units, total_s, descs, threads = 0, 0.0, [], 1
    per_step_budget = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for s in range(args.warmup + args.steps):
        u, t, d, threads, _ = oracle_sample(wl, per_step_budget, start_seq=s * 3,
                                            cache=args.cache, demotion=args.demotion)
        if s >= args.warmup:
            total_units += u
            total_s += t
            descs.append(d)
    value = total_units / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total_s / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args.cache, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": descs[0] if descs else ""},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def rank_workload(name, rank, sinks=None, recent=None):
    """The workload of one rank: the named shape with its own data seed, so that N ranks
    run N independent replica batches (weak scaling, no exchange). sinks / recent
    override the protected-set widths (the name then says so)."""
    from quantized_kv_cache_kv4_b200.workload import make_workload
    wl = make_workload(name)
    wl.seed = wl.seed + 7919 * rank
    if sinks is not None or recent is not None:
        wl.num_sinks = wl.num_sinks if sinks is None else int(sinks)
        wl.num_recent = wl.num_recent if recent is None else int(recent)
        wl.name = f"{wl.name}-S{wl.num_sinks}-R{wl.num_recent}"
    return wl


def combine_ranks(ms, units, world, device):
    """(max over ranks of a timed region in ms, sum over ranks of the units processed).
    Every rank calls this the same number of times, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms), float(units)], dtype=torch.float64, device=device)
    if world > 1:
        tmax = t[:1].clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        usum = t[1:].clone()
        dist.all_reduce(usum, op=dist.ReduceOp.SUM)
        return float(tmax.item()), float(usum.item())
    return float(t[0].item()), float(t[1].item())


def recorded_traffic(workload):
    """DRAM bytes (read + write) of one attention-kernel launch on `workload`, from the ncu
    capture recorded under profiles/, or None when the kernel sources have changed since
    that capture (or none was recorded for this workload)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "attn_kernel_rollout1024.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    if rec.get("workload") != workload:
        return None
    for rel, digest in rec["sources_sha256"].items():
        with open(os.path.join(ROOT, rel), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    return rec["dram_bytes_read_per_launch"] + rec["dram_bytes_write_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from quantized_kv_cache_kv4_b200 import build
    build.build()
    from quantized_kv_cache_kv4_b200 import kv4
    from quantized_kv_cache_kv4_b200.session import BaselineSession, DecodeSession
    from quantized_kv_cache_kv4_b200.host_io import HostStepPipeline

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    wl = rank_workload(args.workload, rank, args.sinks, args.recent)
    if args.demotion == "B":
        wl.name += "-demotionB"
    if args.prefix == "shared" and args.cache == "kv4":
        wl.name += "-prefix-shared"
    W, K = args.warmup, args.steps
    # one session per layer (same lengths and paging, own data); they share a workspace
    if args.cache == "kv4":
        make_session = lambda *a, **kw: DecodeSession(*a, demotion=args.demotion,
                                                      prefix=args.prefix, **kw)
    else:
        fmt = kv4.BASELINE_BF16 if args.cache == "bf16" else kv4.BASELINE_KV8
        make_session = lambda *a, **kw: BaselineSession(*a, fmt=fmt, **kw)
    sess = make_session(wl, steps=W + K, device=dev)
    layers = [sess] + [make_session(wl, layer=li, steps=W + K, device=dev,
                                    workspace=sess.workspace)
                       for li in range(1, wl.num_layers)]
    # the layers after the first of a step reuse its work list (same lengths and paging;
    # the layers' calls run in order on one stream and share the workspace)
    for ls in layers[1:]:
        ls.plan_reuse = args.plan_reuse == "on"
    nl = len(layers)
    stream = torch.cuda.current_stream(dev)
    H = wl.num_kv_heads
    L0 = wl.seq_lens.astype(np.int64)

    def barrier():
        if world > 1:
            dist.barrier()

    # warm-up
    for s in range(W):
        for ls in layers:
            ls.step(s)
    torch.cuda.synchronize(dev)
    for ls in layers:
        ls.check_err()

    # ---- timed region: K full steps (append + attention of every layer), device events ----
    steps = list(range(W, W + K))

    def timed(run_append, run_attention):
        """run_append(i, s, l) / run_attention(i, s, l) launch step s's calls of layer l;
        every attention call is bracketed by events."""
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        att = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(len(steps) * nl)]
        barrier()
        torch.cuda.synchronize(dev)
        ev[0].record(stream)
        for i, s in enumerate(steps):
            for li in range(nl):
                run_append(i, s, li)
                att[i * nl + li][0].record(stream)
                run_attention(i, s, li)
                att[i * nl + li][1].record(stream)
        ev[1].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        for ls in layers:
            ls.check_err()
        return ev[0].elapsed_time(ev[1]), [a.elapsed_time(b) for a, b in att]

    # A timed step is one kv4_decode_step call per layer (append + attention in one call,
    # the work list and the append in one launch); the attention calls are also
    # timed on their own, as the separate kv4_decode_attention call, for the roofline.
    # eager: every call launches its kernels from the host
    with ClockSampler(local_rank) as clocks_eager:
        ms_eager_calls, att_eager = timed(lambda i, s, li: layers[li].append_step(s),
                                          lambda i, s, li: layers[li].attention_step(s))
        ms_eager, _ = timed(lambda i, s, li: layers[li].fused_step(s), lambda i, s, li: None)
    if args.launch == "graph":
        # graphs: every call captured once per step and layer (outside the timed region)
        # and replayed; the same kernels on the same per-step inputs
        g_app, g_att, g_step = [], [], []
        for s in steps:
            for ls in layers:
                for gl, fn in ((g_app, ls.append_step), (g_att, ls.attention_step),
                               (g_step, ls.fused_step)):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        fn(s)
                    gl.append(g)
        ms_calls, att_ms = timed(lambda i, s, li: g_app[i * nl + li].replay(),
                                 lambda i, s, li: g_att[i * nl + li].replay())
        with ClockSampler(local_rank) as clocks:
            ms, _ = timed(lambda i, s, li: g_step[i * nl + li].replay(), lambda i, s, li: None)
    else:
        clocks, ms, att_ms, ms_calls = clocks_eager, ms_eager, att_eager, ms_eager_calls
    units_local = nl * sum(units_per_step(wl, L0 + s) for s in range(W, W + K))
    ms_max, units_all = combine_ranks(ms, units_local, world, dev)
    value = units_all / (ms_max / 1000.0)
    ms_eager_max, _ = combine_ranks(ms_eager, 0, world, dev)
    ms_calls_max, _ = combine_ranks(ms_calls, 0, world, dev)

    # ---- the last timed step's output against the oracle (rank 0, KV4-RL cache): the
    # timed passes replay steps that already ran, but after the last pass layer 0's
    # output holds step W+K-1, whose recent window no later token has overwritten ----
    check = output_check(layers[0], W + K - 1) if rank == 0 and args.cache == "kv4" else None

    # ---- roofline of the attention call (plan + split-K attention + merge) ----
    uniq = [attention_bytes(wl, L0 + s, args.cache) for s in range(W, W + K)]
    mean_att_s = statistics.mean(att_ms) / 1000.0
    achieved = statistics.mean(u for u, _ in uniq) / mean_att_s / 1e9
    peak, peak_kind = load_peaks()

    # ---- e2e through the public API with host buffers (H2D inputs, D2H output) ----
    B, Hq, D = wl.num_seqs, wl.num_q_heads, wl.head_dim
    host_inputs = [(ls.step_k.cpu().pin_memory(), ls.step_v.cpu().pin_memory(),
                    ls.q.cpu().pin_memory(), ls.step_lens.cpu().pin_memory()) for ls in layers]
    hout = [torch.empty((K, B, Hq, D), dtype=torch.bfloat16).pin_memory() for _ in layers]
    pipe = HostStepPipeline(layers)
    h2d, d2h = pipe.bytes_per_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    t_host = time.perf_counter()
    pipe.run(host_inputs, hout, range(W, W + K), start_event=e0)
    e1.record(stream)
    host_ms = (time.perf_counter() - t_host) * 1000.0  # host time to issue the K steps
    torch.cuda.synchronize(dev)
    barrier()
    for ls in layers:
        ls.check_err()
    e2e_ms, _ = combine_ranks(e0.elapsed_time(e1), 0, world, dev)
    e2e_value = units_all / (e2e_ms / 1000.0)

    prefill = time_prefill(sess, wl, dev) if args.prefill else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        u, secs, desc, threads, qsecs = oracle_sample(wl, args.cpu_budget, cache=args.cache,
                                                      demotion=args.demotion)
        cpu = {"value": u / secs, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc}
        if qsecs:
            cpu["quantise"] = {"value": u / qsecs, "unit": "tokens*kv_heads/s",
                               "what": "oracle token_records (INT4 records and INT8 copies "
                                       "of every position) on the same sample"}

    if rank == 0:
        ub = statistics.mean(u for u, _ in uniq)
        lb = statistics.mean(l for _, l in uniq)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE[args.cache],
            "data": "synthetic",
            "config": bench_config(wl, args.cache, world),
            "method": {"step": "one kv4_decode_step call per layer (append + attention; "
                               "the work list and the append in one launch"
                               + ("; layers after the first reuse the first layer's work list"
                                  if nl > 1 and args.plan_reuse == "on" else "") + ")",
                       "launch": {"graph": "cuda graph per call, replayed (each layer's "
                                           "call of every step)",
                                  "eager": "eager"}[args.launch]},
            "attention_ms": statistics.mean(att_ms),
            "two_calls": {"ms_per_step": ms_calls_max / K,
                          "note": "kv4_quantize_append and kv4_decode_attention as separate "
                                  "calls; attention_ms and the roofline time the latter"},
            "eager": {"value": units_all / (ms_eager_max / 1000.0),
                      "ms_per_step": ms_eager_max / K,
                      "attention_ms": statistics.mean(att_eager)},
            "attention_gbs_unique": ub / mean_att_s / 1e9,
            "attention_gbs_logical": lb / mean_att_s / 1e9,
            "roofline": {"kernel": CALL[args.cache] + " (plan + attention + merge launches)",
                         "bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": recorded_traffic(wl.name) if args.cache == "kv4" else None},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                    "host_issue_ms_per_step": host_ms / K},
            "output_check": check,
            # per step and layer for KV4-RL: the work list and the append in one launch (the
            # append alone with a reused list), attention, lift, merge (+ the prefix kernel
            # with the shared-prefix read); for a comparison cache: append, plan (none
            # with a reused list), attention, merge
            "gpu_launches": ((4 + (1 if args.prefix == "shared" else 0)) * nl
                             if args.cache == "kv4" else
                             4 * nl - (nl - 1 if nl > 1 and args.plan_reuse == "on" else 0)) * K,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        if prefill is not None:
            line["prefill"] = {**prefill, "peak_gbs": peak, "frac": prefill["gbs"] / peak}
        print(json.dumps(line), flush=True)
    del layers
    if world > 1:
        dist.destroy_process_group()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kv4", choices=["kv4", "reference"])
    ap.add_argument("--workload", default="rollout")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cache", default="kv4", choices=["kv4", "kv8", "bf16"],
                    help="KV4-RL cache (default) or a comparison cache: all-INT8 or BF16")
    ap.add_argument("--demotion", default="A", choices=["A", "B"],
                    help="INT4 copies from the bf16 input (A) or from the INT8 copy (B)")
    ap.add_argument("--prefix", default="off", choices=["off", "shared"],
                    help="shared-prefix read: pages shared by a group's sequences read by "
                         "every sequence (off, the default) or once per group (shared)")
    ap.add_argument("--plan-reuse", default="on", choices=["on", "off"],
                    help="multi-layer workloads: layers after the first of a step reuse its "
                         "work list (on, the default) or build their own (off)")
    ap.add_argument("--sinks", type=int, default=None, help="override S (protection sweep)")
    ap.add_argument("--recent", type=int, default=None, help="override R (protection sweep)")
    ap.add_argument("--prefill", action="store_true",
                    help="also time a bulk prefill (one CSR append call of ~1M rows)")
    ap.add_argument("--launch", default="graph", choices=["graph", "eager"],
                    help="timed calls replayed from CUDA graphs (default) or launched eagerly")
    args = ap.parse_args(argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
