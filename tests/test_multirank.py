"""Multi-rank host logic of the benchmark, run as two gloo ranks on the CPU.

The layer forward shards by sequence: every rank runs its own batch with the
same weights and no collective on the data path; the only collectives are the
reductions of the timed milliseconds (max over ranks) and of the token counts
(sum over ranks) after the timed region.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle.hstu_oracle as O  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # rank r reports a different time and token count; every rank must see
        # the slowest time and the total of the tokens
        ms, tokens = bench.reduce_over_ranks(10.0 + 5.0 * rank, 1000 + rank, world, "cpu")
        results[rank] = (ms, tokens)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                           join=True, start_method="spawn")
        got = dict(results)
    assert got == {0: (15.0, 2001), 1: (15.0, 2001)}


def test_reduce_over_ranks_single_rank_is_identity():
    assert bench.reduce_over_ranks(3.5, 77, 1) == (3.5, 77)


def test_rank_workloads_share_weights_not_data():
    w0 = bench.rank_workload(0)
    w1 = bench.rank_workload(1)
    # one model
    for a, b in zip(w0.layers, w1.layers):
        for name in ("w1", "w2", "pos_bias", "time_bias"):
            assert np.array_equal(getattr(a, name), getattr(b, name))
    # independent sequences from the same recipe: same batch size and length range
    assert len(w0.seq_offsets) == len(w1.seq_offsets)
    assert not np.array_equal(w0.seq_offsets, w1.seq_offsets) or not np.array_equal(w0.x, w1.x)
    for w in (w0, w1):
        lens = np.diff(w.seq_offsets)
        assert lens.min() >= 4096 and lens.max() <= 8192
        assert np.all(np.diff(w.timestamps[w.seq_offsets[0]:w.seq_offsets[1]]) >= 0)


def test_unmasked_pairs_matches_oracle_count():
    offs = np.array([0, 1, 5, 5, 133, 300], dtype=np.int64)
    nt = np.array([0, 2, 0, 64, 167], dtype=np.int64)
    assert bench.unmasked_pairs(offs) == O.attention_pairs(offs)
    assert bench.unmasked_pairs(offs, nt) == O.attention_pairs(offs, nt)
    # and against the mask itself, built by the oracle, on one small sequence
    mask = O.attention_mask(12, 5)
    assert bench.unmasked_pairs([0, 12], [5]) == int(np.count_nonzero(mask))


def test_traffic_is_null_once_the_kernel_changed(tmp_path):
    """The roofline's DRAM traffic comes from a committed ncu capture only while
    the kernel's sources still match the digest recorded with it."""
    digest = bench.kernel_digest("attn_fwd_tc")
    good = tmp_path / "good.txt"
    good.write_text(f"# comment attn_fwd_tc 1 2\nattn_fwd_tc 12345 {digest}\n")
    stale = tmp_path / "stale.txt"
    stale.write_text("attn_fwd_tc 12345 0000000000000000\n")
    assert bench.read_traffic("attn_fwd_tc", str(good)) == 12345.0
    assert bench.read_traffic("attn_fwd_tc", str(stale)) is None
    assert bench.read_traffic("attn_fwd_tc", str(tmp_path / "missing.txt")) is None


def test_mfalcon_pairs_match_one_pass_over_all_candidates():
    """The ranking row's FLOP count: with the history cached, a call attends the
    pairs of one M-FALCON pass over [history ; all candidates] per user."""
    hist = np.array([2048, 0, 37, 130], dtype=np.int64)
    cands = np.array([4096, 9, 0, 12], dtype=np.int64)
    offs = np.concatenate([[0], np.cumsum(hist + cands)])
    assert bench.mfalcon_pairs(hist, cands) == O.attention_pairs(offs, cands)
