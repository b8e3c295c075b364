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


def _dp_rank_main(rank, world, port, results):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from hstu_sequential_transducer_02_b200.data_parallel import GradAllReduce, PARAM_GRADS
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        shapes = {"w1": (16, 4), "b1": (16,), "ln1_gamma": (4,), "ln1_beta": (4,), "ln2_gamma": (8,),
                  "ln2_beta": (8,), "w2": (4, 8), "b2": (4,), "pos_bias": (128,), "time_bias": (128,)}
        layers = []
        for l in range(3):
            g = {n: torch.full(shapes[n], float((rank + 1) * (l + 1))) + torch.arange(
                int(np.prod(shapes[n])), dtype=torch.float32).reshape(shapes[n]) for n in PARAM_GRADS}
            g["uvqk"] = torch.full((5, 2), float(rank))      # per-token gradient: not reduced
            layers.append(g)
        red = GradAllReduce()
        for g in reversed(layers):                             # the backward finishes the last layer first
            red.layer_done(g)
        red.wait()
        results[rank] = {(l, n): layers[l][n].clone().numpy() for l in range(3) for n in list(PARAM_GRADS) + ["uvqk"]}
    finally:
        dist.destroy_process_group()


def test_data_parallel_gradient_sum_gloo_world2():
    """Every rank ends with the sum over ranks of each parameter gradient, in
    its own tensors and shapes; the per-token activation gradient is left alone."""
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_dp_rank_main, args=(world, _free_port(), results), nprocs=world, join=True,
                           start_method="spawn")
        got = dict(results)
    for rank in range(world):
        for (l, n), v in got[rank].items():
            if n == "uvqk":
                assert np.all(v == rank)
                continue
            ar = np.arange(v.size, dtype=np.float32).reshape(v.shape)
            want = sum(float((r + 1) * (l + 1)) + ar for r in range(world))
            assert np.array_equal(v, want), (rank, l, n)


def test_data_parallel_single_rank_is_a_no_op():
    import torch
    from hstu_sequential_transducer_02_b200.data_parallel import GradAllReduce, PARAM_GRADS
    g = {n: torch.ones(3) for n in PARAM_GRADS}
    red = GradAllReduce()
    red.layer_done(g)
    red.wait()
    assert all(torch.equal(g[n], torch.ones(3)) for n in PARAM_GRADS)
