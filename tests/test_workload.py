"""The seeded synthetic inputs and the paging (plumbing shared by the tests and the
benchmark; no method arithmetic): the shapes the workloads are stated with, determinism,
the shared-prompt structure, and page tables that never give two sequences the same
page except a group's prompt pages. CPU only."""
import numpy as np
import pytest
import torch

from quantized_kv_cache_kv4_b200 import workload as W

NAMES = ("tiny", "qwen3-8b-layer", "rollout", "longtail", "qwen3-4b-step")


def test_workload_shapes():
    t = W.make_workload("tiny")
    assert list(t.seq_lens) == [37, 150, 300, 511]
    assert (t.num_q_heads, t.num_kv_heads, t.num_sinks, t.num_recent) == (8, 2, 4, 32)
    q = W.make_workload("qwen3-8b-layer")
    assert q.num_seqs == 64 and set(q.seq_lens) == {2048}
    assert (q.num_q_heads, q.num_kv_heads, q.num_sinks, q.num_recent) == (32, 8, 16, 128)
    r = W.make_workload("rollout")
    assert r.num_seqs == 1024 and r.group_seqs == 8 and r.prompt_len == 256
    resp = r.seq_lens - 256
    assert resp.min() >= 1 and resp.max() <= 16384
    assert abs(resp.mean() - 1450) < 0.15 * 1450  # lognormal with mean 1450 (sampled)
    lt = W.make_workload("longtail")
    assert lt.num_seqs == 128 and set(lt.seq_lens) == {16384} and lt.kv_dist == "student_t3"
    s5 = W.make_workload("qwen3-4b-step")
    assert s5.num_seqs == 512 and s5.num_layers == 36
    assert s5.seq_lens.min() >= 512 and s5.seq_lens.max() <= 8192
    with pytest.raises(ValueError):
        W.make_workload("nope")


@pytest.mark.parametrize("name", NAMES)
def test_workloads_and_paging_are_deterministic(name):
    a, b = W.make_workload(name), W.make_workload(name)
    assert np.array_equal(a.seq_lens, b.seq_lens)
    pa, pb = W.make_paging(a, extra_tokens=3), W.make_paging(b, extra_tokens=3)
    assert np.array_equal(pa.page_table, pb.page_table)
    assert np.array_equal(pa.sink_idx, pb.sink_idx) and np.array_equal(pa.ring_idx, pb.ring_idx)


@pytest.mark.parametrize("name", NAMES)
def test_pages_are_private_except_shared_prompts(name):
    wl = W.make_workload(name)
    pg = W.make_paging(wl, extra_tokens=5)
    P = wl.page_size
    owners = {}
    for b in range(wl.num_seqs):
        n = (int(wl.seq_lens[b]) + 5 + P - 1) // P
        row = pg.page_table[b]
        assert np.all(row[:n] >= 0) and np.all(row[:n] < pg.num_pages)
        assert np.all(row[n:] == -1)
        shared = wl.prompt_len // P if wl.shared_prefix else 0
        for i, pid in enumerate(row[:n]):
            key = (wl.group_of(b), i) if i < shared else (None, b, i)
            owners.setdefault(int(pid), set()).add(key)
    # every physical page belongs to exactly one (group prompt page) or (sequence page)
    assert all(len(v) == 1 for v in owners.values())
    assert len(owners) == pg.num_pages
    # one leader per group writes the prompt; sink sets per group, rings per sequence
    if wl.shared_prefix:
        groups = [wl.group_of(b) for b in range(wl.num_seqs)]
        assert pg.leaders.sum() == len(set(groups))
        assert np.array_equal(pg.sink_idx, np.array(groups))
    else:
        assert pg.leaders.all() and np.array_equal(pg.sink_idx, np.arange(wl.num_seqs))
    assert np.array_equal(pg.ring_idx, np.arange(wl.num_seqs))


def test_shared_prompt_rows_are_the_groups():
    wl = W.custom_workload([300, 290, 280, 270], num_kv_heads=2, prompt_len=256, group_seqs=2,
                           seed=9)
    k0, v0 = W.seq_kv(wl, 0, 300)
    k1, v1 = W.seq_kv(wl, 1, 290)
    k2, _ = W.seq_kv(wl, 2, 280)
    assert torch.equal(k0[:256], k1[:256]) and torch.equal(v0[:256], v1[:256])  # group 0
    assert not torch.equal(k0[256:290], k1[256:290])                            # own responses
    assert not torch.equal(k0[:256], k2[:256])                                  # group 1
    # a slice is the same rows as the whole stream's
    ks, _ = W.seq_kv(wl, 0, 280, start=250)
    assert torch.equal(ks, k0[250:280])
    assert k0.dtype == torch.bfloat16 and k0.shape == (300, 2, 128)


def test_queries_are_seeded_per_step_and_layer():
    wl = W.make_workload("tiny")
    q0, q0b = W.queries(wl, 0, 0), W.queries(wl, 0, 0)
    assert torch.equal(q0, q0b) and q0.shape == (4, 8, 128) and q0.dtype == torch.bfloat16
    assert not torch.equal(q0, W.queries(wl, 1, 0))
    assert not torch.equal(q0, W.queries(wl, 0, 1))


def test_outlier_channels_are_scaled_keys():
    wl = W.make_workload("tiny")  # 4 K channels per kv head x8
    ids = W.outlier_channel_ids(wl)
    assert ids.shape == (2, 4) and all(len(set(r)) == 4 for r in ids)
    k, v = W.seq_kv(wl, 3, 511)
    kf, vf = k.float(), v.float()
    for h in range(2):
        others = [c for c in range(128) if c not in ids[h]]
        ratio = kf[:, h, ids[h]].std() / kf[:, h, others].std()
        assert 6.0 < float(ratio) < 10.0                       # ~8x on the chosen channels
        assert 0.8 < float(vf[:, h].std()) < 1.2               # values unscaled
