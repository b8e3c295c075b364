"""GPU parity of the attention entry points (hstu_attn_fwd / hstu_attn_bwd)
and of the bucket and mask rule, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.hstu_oracle as O
from hstu_sequential_transducer_02_b200 import workload as W
from tests.helpers import assert_close, dev, torch_dtype

pytestmark = pytest.mark.gpu


def _b():
    from hstu_sequential_transducer_02_b200 import binding
    return binding


def _run_attn(d, H, dh, dtype_name, force_simt=False):
    b = _b()
    td = torch_dtype(dtype_name)
    T = d["q"].shape[0]
    q = dev(d["q"].reshape(T, H * dh), td)
    k = dev(d["k"].reshape(T, H * dh), td)
    v = dev(d["v"].reshape(T, H * dh), td)
    nt = None if d["num_targets"] is None else dev(d["num_targets"])
    out, ws = b.attn_fwd(q, k, v, dev(d["seq_offsets"]), dev(d["timestamps"]), dev(d["pos_bias"]),
                         dev(d["time_bias"]), H, num_targets=nt, force_simt=force_simt, return_workspace=True)
    torch.cuda.synchronize()
    assert b.workspace_status(ws) == 0
    return out.float().cpu().numpy().reshape(T, H, dh)


def _ref(d):
    return O.attention_forward(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], d["pos_bias"],
                               d["time_bias"], d["num_targets"])


def test_attn_fwd_fp32_tiny_config():
    """configuration 0 shapes: B=4, n in [8, 64], H=2, dh=32, fp32 (CUDA-core path)."""
    lens = W.sample_lengths(np.random.default_rng(20240), 4, "uniform", 8, 64)
    d = W.random_attention_inputs(20240, lens, 2, 32, "f32")
    assert_close(_run_attn(d, 2, 32, "f32"), _ref(d), "f32", "attn fp32")


@pytest.mark.parametrize("dh", [64, 128])
@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("mfalcon", [False, True])
def test_attn_fwd_bf16_tensor_cores(dh, per_head, mfalcon):
    """tcgen05 path: several tiles, ragged tails, empty and one-token sequences."""
    lens = [1, 127, 128, 129, 0, 300, 513]
    nt = [0, 5, 0, 64, 0, 129, 200] if mfalcon else None
    d = W.random_attention_inputs(7 + dh, lens, 2, dh, "bf16", num_targets=nt, per_head_rab=per_head)
    assert_close(_run_attn(d, 2, dh, "bf16"), _ref(d), "bf16", f"attn bf16 dh={dh}")


@pytest.mark.parametrize("dh", [32, 64, 128])
def test_attn_fwd_bf16_cuda_core_path(dh):
    d = W.random_attention_inputs(11, [65, 1, 190], 2, dh, "bf16", num_targets=[0, 0, 17])
    assert_close(_run_attn(d, 2, dh, "bf16", force_simt=True), _ref(d), "bf16", "attn simt bf16")


@pytest.mark.parametrize("gap", [1.0, 600.0, 5e6])
def test_attn_fwd_time_bias_regimes(gap):
    """Timestamp gaps from 1 s to ~2 months: constant, few-bucket and general
    bias paths of the tensor-core epilogue all occur."""
    d = W.random_attention_inputs(5, [700, 260], 4, 64, "bf16", gap_mean=gap)
    d["time_bias"] = (np.random.default_rng(1).normal(0, 1.0, 128)).astype(np.float32)
    assert_close(_run_attn(d, 4, 64, "bf16"), _ref(d), "bf16", f"attn gap={gap}")


def test_attn_fwd_unsorted_and_huge_timestamps():
    d = W.random_attention_inputs(6, [400, 131], 2, 128, "bf16")
    rng = np.random.default_rng(3)
    ts = d["timestamps"].copy()
    ts[:400] = rng.permutation(ts[:400])                 # non-monotone inside a sequence
    ts[400:] = rng.integers(0, 2 ** 45, 131)             # spans beyond the 32-bit fast path
    d["timestamps"] = ts
    d["time_bias"] = np.linspace(-1, 1, 128).astype(np.float32)
    assert_close(_run_attn(d, 2, 128, "bf16"), _ref(d), "bf16", "attn odd timestamps")


def test_rab_bucket_and_mask_dump_bit_exact():
    b = _b()
    rng = np.random.default_rng(9)
    lens = [50, 300, 9]
    offs = W.offsets_from_lengths(lens)
    thr = np.array(b.build_time_thresholds(0.301), dtype=np.int64)
    # timestamps whose differences hit thresholds exactly and one off
    ts = []
    for n in lens:
        base = 1_700_000_000
        deltas = rng.choice(thr[1:60], size=n) + rng.integers(-1, 2, size=n)
        ts.append(base + np.cumsum(np.maximum(deltas, 0)))
    ts = np.concatenate(ts).astype(np.int64)
    nt = np.array([0, 40, 9], dtype=np.int32)
    pairs = []
    for s, n in enumerate(lens):
        for _ in range(400):
            pairs.append((s, int(rng.integers(0, n)), int(rng.integers(0, n))))
    pairs += [(1, 299, 0), (1, 299, 299), (1, 280, 270), (0, 49, 49), (2, 3, 3)]
    pairs = np.array(pairs, dtype=np.int32)
    got = b.debug_rab_buckets(dev(offs), dev(ts), dev(pairs.reshape(-1)).reshape(-1, 3), num_targets=dev(nt))
    got = got.cpu().numpy()
    want = []
    for s, i, j in pairs:
        a = offs[s]
        n = offs[s + 1] - a
        p = O.positions(n, nt[s])
        want.append((int(O.pos_bucket(p[i] - p[j])), int(O.time_bucket(ts[a + i] - ts[a + j])),
                     int(O.attention_mask(n, nt[s])[i, j])))
    assert np.array_equal(got, np.array(want, dtype=np.int32))


@pytest.mark.parametrize("mfalcon", [False, True])
def test_attn_bwd_tensor_core_several_tiles(mfalcon):
    """bf16, head dim 64 (the tensor-core backward): sequences spanning several
    128-row tiles, a ragged last tile and a one-token sequence, so that kv tiles
    meet several q tiles and the dQ atomics of different kv tiles add up."""
    b = _b()
    lens = [257, 600, 1, 130]
    nt = [0, 75, 0, 129] if mfalcon else None
    d = W.random_attention_inputs(47, lens, 2, 64, "bf16", num_targets=nt, qk_std=0.5)
    T = sum(lens)
    q, k, v, do = (dev(d[n].reshape(T, 2 * 64), torch.bfloat16) for n in ("q", "k", "v", "dout"))
    ntd = None if nt is None else dev(d["num_targets"])
    dq, dk, dv, dpb, dtb = b.attn_bwd(q, k, v, do, dev(d["seq_offsets"]), dev(d["timestamps"]), dev(d["pos_bias"]),
                                      dev(d["time_bias"]), 2, num_targets=ntd)
    torch.cuda.synchronize()
    rq, rk, rv, rpb, rtb = O.attention_backward(d["q"], d["k"], d["v"], d["dout"], d["seq_offsets"],
                                                d["timestamps"], d["pos_bias"], d["time_bias"], d["num_targets"])
    for got, ref, name in [(dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")]:
        assert_close(got.float().cpu().numpy().reshape(ref.shape), ref, "bf16", name, grad=True)
    for got, ref, name in [(dpb, rpb, "dpos"), (dtb, rtb, "dtime")]:
        g = got.cpu().numpy()
        assert np.linalg.norm(g - ref) <= 1e-2 * max(np.linalg.norm(ref), 1e-6), name


def _oracle_thresholds():
    """Smallest |dt| of every time bucket, by bisection over the oracle's rule."""
    thr = []
    for b in range(128):
        lo, hi = 0, 2 ** 62
        while lo < hi:
            mid = (lo + hi) // 2
            if int(O.time_bucket(np.int64(mid))) >= b:
                hi = mid
            else:
                lo = mid + 1
        thr.append(lo)
    return thr


def test_time_bucket_at_every_threshold():
    """The tensor-core kernel's 32-bit bucket rule (log estimate, exact compare
    near a boundary) and the 64-bit search, bit-exact against the oracle at
    every bucket threshold and three steps either side."""
    b = _b()
    ds = [0, 1, 2, 3, 2 ** 23 - 1, 2 ** 23, 2 ** 23 + 1, 2 ** 31 - 2, 2 ** 31 - 1, 2 ** 31, 2 ** 40 + 7]
    for t in _oracle_thresholds():
        ds += [d for d in range(t - 3, t + 4) if 0 <= d < 2 ** 45]
    ds = np.array(sorted(set(ds)), dtype=np.int64)
    base = 1_700_000_000
    ts = np.concatenate([[base], base + ds]).astype(np.int64)   # row k > 0 is dt = ds[k-1] from row 0
    n = len(ts)
    offs = np.array([0, n], dtype=np.int32)
    pairs = np.array([(0, k, 0) for k in range(1, n)] + [(0, 0, k) for k in range(1, n)], dtype=np.int32)
    got = b.debug_rab_buckets(dev(offs), dev(ts), dev(pairs.reshape(-1)).reshape(-1, 3)).cpu().numpy()
    want = O.time_bucket(np.concatenate([ds, ds]))
    assert np.array_equal(got[:, 1], want.astype(np.int32))


def _gpu_buckets_of(ds):
    """Time buckets of the differences `ds` from the GPU's rule (row k + 1 sits
    ds[k] seconds after row 0 of one sequence)."""
    b = _b()
    base = 1_700_000_000
    ts = np.concatenate([[base], base + ds]).astype(np.int64)
    n = len(ts)
    offs = np.array([0, n], dtype=np.int32)
    pairs = np.zeros((n - 1, 3), dtype=np.int32)
    pairs[:, 1] = np.arange(1, n, dtype=np.int32)
    got = b.debug_rab_buckets(dev(offs), dev(ts), dev(pairs.reshape(-1)).reshape(-1, 3))
    return got[:, 1].cpu().numpy()


def test_time_bucket_every_difference_below_2_24_and_a_stride_beyond():
    """The 32-bit bucket rule trusts its log estimate (error below 2e-4) unless
    the estimate lies within 2^-9 of an integer: every |dt| in [0, 2^24] and a
    prime stride from 2^24 to 2^31 give the oracle's fp64 bucket bit for bit,
    which pins that error bound itself, not only the thresholds."""
    for lo in range(0, 1 << 24, 1 << 22):
        ds = np.arange(lo, lo + (1 << 22) + 1, dtype=np.int64)
        got = _gpu_buckets_of(ds)
        want = O.time_bucket(ds).astype(np.int32)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, f"dt {ds[bad[:5]]}: GPU {got[bad[:5]]} oracle {want[bad[:5]]}"
    ds = np.arange(1 << 24, (1 << 31) - 1, 1021, dtype=np.int64)
    got = _gpu_buckets_of(ds)
    want = O.time_bucket(ds).astype(np.int32)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"dt {ds[bad[:5]]}: GPU {got[bad[:5]]} oracle {want[bad[:5]]}"


@pytest.mark.parametrize("mfalcon", [False, True])
def test_attn_bwd_long_sequences(mfalcon):
    """The tensor-core backward on sequences longer than 1,024 tokens (kv tiles
    that meet up to 20 q tiles), with and without M-FALCON targets."""
    b = _b()
    lens = [2433, 1090, 64]
    nt = [300, 0, 17] if mfalcon else None
    d = W.random_attention_inputs(53, lens, 2, 64, "bf16", num_targets=nt, qk_std=0.5)
    T = sum(lens)
    q, k, v, do = (dev(d[n].reshape(T, 2 * 64), torch.bfloat16) for n in ("q", "k", "v", "dout"))
    ntd = None if nt is None else dev(d["num_targets"])
    dq, dk, dv, dpb, dtb = b.attn_bwd(q, k, v, do, dev(d["seq_offsets"]), dev(d["timestamps"]), dev(d["pos_bias"]),
                                      dev(d["time_bias"]), 2, num_targets=ntd)
    torch.cuda.synchronize()
    rq, rk, rv, rpb, rtb = O.attention_backward(d["q"], d["k"], d["v"], d["dout"], d["seq_offsets"],
                                                d["timestamps"], d["pos_bias"], d["time_bias"], d["num_targets"])
    for got, ref, name in [(dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")]:
        assert_close(got.float().cpu().numpy().reshape(ref.shape), ref, "bf16", name, grad=True)
    for got, ref, name in [(dpb, rpb, "dpos"), (dtb, rtb, "dtime")]:
        assert_close(got.cpu().numpy(), ref, "bf16", name, grad=True)


def test_bounded_wait_times_out_and_reports():
    b = _b()
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    b.debug_timeout_probe(2_000_000, st)  # 2 ms
    torch.cuda.synchronize()
    assert int(st.item()) == b.ERR_TIMEOUT
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum().item()) == 4.0


def test_bad_offsets_reported_not_crashing():
    b = _b()
    d = W.random_attention_inputs(2, [10, 20], 2, 64, "bf16")
    T = 30
    q = dev(d["q"].reshape(T, 128), torch.bfloat16)
    bad = dev(np.array([0, 25, 20], dtype=np.int32))
    out, ws = b.attn_fwd(q, q, q, bad, dev(d["timestamps"]), dev(d["pos_bias"]), dev(d["time_bias"]), 2,
                         return_workspace=True)
    torch.cuda.synchronize()
    assert b.workspace_status(ws) == b.ERR_BAD_OFFSETS
    too_long = dev(np.array([0, 10, 31], dtype=np.int32))
    out, ws = b.attn_fwd(q, q, q, too_long, dev(d["timestamps"]), dev(d["pos_bias"]), dev(d["time_bias"]), 2,
                         return_workspace=True)
    torch.cuda.synchronize()
    assert b.workspace_status(ws) == b.ERR_BAD_OFFSETS


@pytest.mark.parametrize("dtype_name,dh", [("f32", 32), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("mfalcon", [False, True])
def test_attn_bwd_matches_oracle(dtype_name, dh, mfalcon):
    b = _b()
    lens = [70, 1, 130]
    nt = [10, 0, 33] if mfalcon else None
    d = W.random_attention_inputs(31, lens, 2, dh, dtype_name, num_targets=nt, qk_std=0.5)
    td = torch_dtype(dtype_name)
    T = sum(lens)
    q, k, v, do = (dev(d[n].reshape(T, 2 * dh), td) for n in ("q", "k", "v", "dout"))
    ntd = None if nt is None else dev(d["num_targets"])
    dq, dk, dv, dpb, dtb = b.attn_bwd(q, k, v, do, dev(d["seq_offsets"]), dev(d["timestamps"]), dev(d["pos_bias"]),
                                      dev(d["time_bias"]), 2, num_targets=ntd)
    torch.cuda.synchronize()
    rq, rk, rv, rpb, rtb = O.attention_backward(d["q"], d["k"], d["v"], d["dout"], d["seq_offsets"],
                                                d["timestamps"], d["pos_bias"], d["time_bias"], d["num_targets"])
    for got, ref, name in [(dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv")]:
        assert_close(got.float().cpu().numpy().reshape(ref.shape), ref, dtype_name, name, grad=True)
    # rab gradients are fp32 sums over many pairs: relative Frobenius bound
    for got, ref, name in [(dpb, rpb, "dpos"), (dtb, rtb, "dtime")]:
        g = got.cpu().numpy()
        assert np.linalg.norm(g - ref) <= 1e-2 * max(np.linalg.norm(ref), 1e-6), name
