"""GPU parity for batches of more than 1024 sequences: the work-list kernel then scans
the lengths in several block-wide passes (offsets, class bases and the length ranks of
the short-chunk class carried from one block of 1024 sequences to the next) instead of
keeping the offsets of a single pass. The attention of every sequence is compared within
tolerance; the pages and side stores (written by the append kernel, which the work list
does not touch) bit for bit for a seeded sample of sequences on both sides of the block
boundary."""
import numpy as np
import pytest
import torch

from test_gpu_parity import check_attention, check_cache, make_session

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_kv_cache_kv4_b200 import build
    build.build()


@pytest.mark.parametrize("num_seqs,chunk_pages", [(1300, 8), (2100, 0)])
def test_batches_beyond_one_plan_block(num_seqs, chunk_pages):
    """Lengths from 1 to 700 (empty INT4 regions, full chunks, long and short last
    chunks of every length, so every length class spans both sides of the 1024-sequence
    block boundary); 8-page chunks, then the automatic choice."""
    from quantized_kv_cache_kv4_b200 import workload as W
    rng = np.random.default_rng(num_seqs)
    lens = rng.integers(1, 701, num_seqs)
    lens[:8] = [1, 36, 37, 53, 164, 165, 700, 2]
    wl = W.custom_workload(lens, num_sinks=4, num_recent=32, seed=num_seqs & 0xFFFF,
                           outlier_channels=2, outlier_scale=8.0)
    sess = make_session(wl, chunk_pages=chunk_pages)
    sample = np.unique(np.concatenate([np.arange(8), rng.choice(num_seqs, 120, replace=False)]))
    check_cache(sess, sample.tolist())
    check_attention(sess, range(num_seqs))
    sess.check_err()
