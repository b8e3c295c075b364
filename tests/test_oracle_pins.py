"""Pins for the fp64 oracle: each test checks it against something other than
itself (hand-computed values, closed forms, library routines, invariants the
pages state, brute force, finite differences).  CPU only."""
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle.hstu_oracle as O
from hstu_sequential_transducer_02_b200 import workload as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _silu(x):
    return x / (1.0 + math.exp(-x))


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ----------------------------------------------------------------------------
# buckets
# ----------------------------------------------------------------------------

def test_time_bucket_hand_values():
    rows = _read_golden("time_buckets.txt")
    dts = np.array([int(r[0]) for r in rows], dtype=np.int64)
    want = np.array([int(r[-1]) for r in rows])
    assert np.array_equal(O.time_bucket(dts), want)


def test_time_bucket_thresholds_exact_arithmetic():
    """Around every bucket threshold exp(0.301 b) up to b = 100 (dt ~ 1.2e13 s,
    about 380,000 years), the fp64 evaluation agrees with 60-digit decimal
    arithmetic (an independent evaluation of the same rule).  Beyond that the
    fp64 rounding of ln(dt)/0.301 can flip the floor right at a threshold; there
    the fp64 evaluation is the definition both sides follow."""
    getcontext().prec = 60
    div = Decimal("0.301")
    probes = []
    for b in range(1, 101):
        thr = int((div * b).exp().to_integral_value(rounding="ROUND_CEILING"))
        probes += [thr - 2, thr - 1, thr, thr + 1, thr + 2]
    probes = np.array(sorted(set(p for p in probes if p >= 0)), dtype=np.int64)
    exact = []
    for p in probes:
        v = Decimal(int(max(p, 1)))
        e = int((v.ln() / div).to_integral_value(rounding="ROUND_FLOOR"))
        exact.append(min(max(e, 0), 127))
    assert np.array_equal(O.time_bucket(probes), np.array(exact))


def test_pos_bucket_hand_values():
    rows = _read_golden("pos_buckets.txt")
    d = np.array([int(r[0]) for r in rows])
    assert np.array_equal(O.pos_bucket(d), np.array([int(r[1]) for r in rows]))


def test_positions_and_mask_mfalcon_by_hand():
    # n = 5 with 2 candidates: history 0,1,2; candidates at position 3
    assert list(O.positions(5, 2)) == [0, 1, 2, 3, 3]
    m = O.attention_mask(5, 2).astype(int)
    want = np.array([[1, 0, 0, 0, 0],
                     [1, 1, 0, 0, 0],
                     [1, 1, 1, 0, 0],
                     [1, 1, 1, 1, 0],
                     [1, 1, 1, 0, 1]])
    assert np.array_equal(m, want)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def test_single_token_closed_form():
    rng = np.random.default_rng(1)
    q = rng.normal(size=(1, 1, 8))
    k = rng.normal(size=(1, 1, 8))
    v = rng.normal(size=(1, 1, 8))
    pb = rng.normal(size=128)
    tb = rng.normal(size=128)
    out = O.attention_forward(q, k, v, [0, 1], np.array([123], np.int64), pb, tb)
    s = float(q[0, 0] @ k[0, 0]) + pb[0] + tb[0]
    assert np.allclose(out[0, 0], _silu(s) * v[0, 0], rtol=1e-14, atol=0)


def test_two_token_hand_example():
    # dh = 1: q = [1, 2], k = [3, -1], v = [1, 10], no rab, equal timestamps
    q = np.array([1.0, 2.0]).reshape(2, 1, 1)
    k = np.array([3.0, -1.0]).reshape(2, 1, 1)
    v = np.array([1.0, 10.0]).reshape(2, 1, 1)
    z = np.zeros(128)
    out = O.attention_forward(q, k, v, [0, 2], np.array([5, 5], np.int64), z, z)
    o0 = _silu(3.0) * 1.0 / 2
    o1 = (_silu(6.0) * 1.0 + _silu(-2.0) * 10.0) / 2
    assert np.allclose(out[:, 0, 0], [o0, o1], rtol=1e-14)


def test_bias_direction_and_buckets():
    """q = k = 0 and V = identity expose SiLU(rab_ij)/N for every pair."""
    n = 6
    q = np.zeros((n, 1, 2))
    k = np.zeros((n, 1, 2))
    v = np.eye(n).reshape(n, 1, n)
    ts = (np.arange(n) * 600).astype(np.int64)   # dt = 600 (i - j)
    pos = np.zeros(128)
    pos[1] = 1.0                                 # only i - j == 1
    tim = np.zeros(128)
    tim[23] = 2.0                                # dt = 1200 -> bucket 23, only i - j == 2
    out = O.attention_forward(q, k, v.astype(float), [0, n], ts, pos, tim)[:, 0, :]
    want = np.zeros((n, n))
    for i in range(n):
        if i >= 1:
            want[i, i - 1] = _silu(1.0) / n
        if i >= 2:
            want[i, i - 2] = _silu(2.0) / n
    assert np.allclose(out, want, atol=1e-15)


@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("targets", [None, [0, 3, 1]])
def test_pairwise_loop_matches_dense(per_head, targets):
    d = W.random_attention_inputs(7, [5, 9, 4], 2, 4, "f32", num_targets=targets, per_head_rab=per_head)
    a = O.attention_forward(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"],
                            d["pos_bias"], d["time_bias"], d["num_targets"])
    b = O.attention_forward_pairwise(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"],
                                     d["pos_bias"], d["time_bias"], d["num_targets"])
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)


def test_causality_perturbation():
    d = W.random_attention_inputs(3, [12], 2, 8, "f32")
    base = O.attention_forward(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"],
                               d["pos_bias"], d["time_bias"])
    for j in [4, 7, 11]:
        q, k, v = d["q"].copy(), d["k"].copy(), d["v"].copy()
        q[j] += 3.0
        k[j] -= 2.0
        v[j] *= -5.0
        ts = d["timestamps"].copy()
        ts[j:] += 100_000
        pert = O.attention_forward(q, k, v, d["seq_offsets"], ts, d["pos_bias"], d["time_bias"])
        assert np.array_equal(pert[:j], base[:j])
        assert not np.allclose(pert[j], base[j])


def test_no_softmax_row_sums():
    """With zero rab and V = 1 every output component is sum_j SiLU(q_i.k_j)/N;
    the weights do not sum to one (no softmax)."""
    d = W.random_attention_inputs(5, [10], 1, 4, "f32", qk_std=1.0)
    v = np.ones_like(d["v"])
    z = np.zeros(128)
    out = O.attention_forward(d["q"], d["k"], v, d["seq_offsets"], d["timestamps"], z, z)
    q, k = d["q"][:, 0].astype(float), d["k"][:, 0].astype(float)
    for i in range(10):
        s = sum(_silu(float(q[i] @ k[j])) for j in range(i + 1)) / 10
        assert np.allclose(out[i, 0], s, rtol=1e-13)
    assert not np.allclose(out[:, 0, 0] * 10, np.arange(1, 11))


def test_mfalcon_invariants():
    """A candidate's output is the same scored alone, in any microbatch, in any
    order; history rows equal a causal pass over the history alone."""
    rng = np.random.default_rng(11)
    n, m, H, dh = 9, 5, 2, 4
    q = rng.normal(0, .5, (n + m, H, dh))
    k = rng.normal(0, .5, (n + m, H, dh))
    v = rng.normal(0, 1, (n + m, H, dh))
    ts = np.concatenate([np.cumsum(rng.integers(1, 2000, n)), np.full(m, 30_000)]).astype(np.int64)
    pb = rng.normal(0, .3, 128)
    tb = rng.normal(0, .3, 128)
    full = O.attention_forward(q, k, v, [0, n + m], ts, pb, tb, num_targets=[m])
    hist = O.attention_forward(q[:n], k[:n], v[:n], [0, n], ts[:n], pb, tb)
    assert np.allclose(full[:n], hist, rtol=1e-13, atol=1e-15)
    for c in range(m):
        idx = np.r_[np.arange(n), n + c]
        alone = O.attention_forward(q[idx], k[idx], v[idx], [0, n + 1], ts[idx], pb, tb, num_targets=[1])
        assert np.allclose(alone[n], full[n + c], rtol=1e-13, atol=1e-15)
    perm = rng.permutation(m)
    idx = np.r_[np.arange(n), n + perm]
    permuted = O.attention_forward(q[idx], k[idx], v[idx], [0, n + m], ts[idx], pb, tb, num_targets=[m])
    assert np.allclose(permuted[n:], full[n + perm], rtol=1e-13, atol=1e-15)


def test_mfalcon_rank_microbatch_invariance():
    wl = W.make_workload(3, scale=1 / 128, batch=2)
    nh, hd = wl.spec.num_heads, wl.spec.head_dim
    e = wl.extras
    args = (wl.layers, wl.seq_offsets, wl.x, wl.timestamps, e["cand_offsets"], e["cand_x"], e["cand_ts"])
    r1 = O.mfalcon_rank(*args, 1, nh, hd)
    r3 = O.mfalcon_rank(*args, 3, nh, hd)
    rall = O.mfalcon_rank(*args, 10 ** 6, nh, hd)
    assert np.allclose(r1, r3, rtol=1e-12, atol=1e-12)
    assert np.allclose(r1, rall, rtol=1e-12, atol=1e-12)


def test_attention_pairs_counts_mask():
    offs = [0, 5, 5, 12]
    nt = [2, 0, 3]
    want = sum(int(O.attention_mask(n, t).sum()) for n, t in [(5, 2), (0, 0), (7, 3)])
    assert O.attention_pairs(offs, nt) == want


# ----------------------------------------------------------------------------
# LayerNorm, layer
# ----------------------------------------------------------------------------

def test_layer_norm_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.normal(3, 2, (7, 16))
    g = rng.normal(1, .2, 16)
    b = rng.normal(0, .2, 16)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (16,), torch.tensor(g), torch.tensor(b), 1e-5).numpy()
    assert np.allclose(O.layer_norm(x, g, b), ref, rtol=1e-13, atol=1e-13)
    const = np.full((2, 16), 4.0)
    assert np.allclose(O.layer_norm(const, g, b), np.broadcast_to(b, (2, 16)))


def _tiny_layer(seed, d=8, H=2, dh=4, random_affine=True):
    rng = np.random.default_rng(seed)
    hv = H * dh
    return W.LayerParams(
        w1=rng.normal(0, .4, (4 * hv, d)), b1=rng.normal(0, .2, 4 * hv),
        ln1_g=rng.normal(1, .2, d) if random_affine else np.ones(d),
        ln1_b=rng.normal(0, .2, d) if random_affine else np.zeros(d),
        ln2_g=rng.normal(1, .2, hv) if random_affine else np.ones(hv),
        ln2_b=rng.normal(0, .2, hv) if random_affine else np.zeros(hv),
        w2=rng.normal(0, .4, (d, hv)), b2=rng.normal(0, .2, d),
        pos_bias=rng.normal(0, .3, 128), time_bias=rng.normal(0, .3, 128))


def test_layer_closed_form_constant_projection():
    """W1 = 0: U, V, Q, K are SiLU of the bias blocks, the same for every token.
    Then O_i = ((i+1)/n) SiLU(q.k + 0) v per head, and
    Y_i = X_i + (LN2(O_i) * U) W2^T + b2 — which fixes the split order
    (U first, V second) and the 1/N scale."""
    d, H, dh, n = 8, 2, 4, 6
    hv = H * dh
    p = _tiny_layer(4, d, H, dh)
    p.w1 = np.zeros_like(p.w1)
    p.pos_bias = np.zeros(128)
    p.time_bias = np.zeros(128)
    rng = np.random.default_rng(5)
    x = rng.normal(size=(n, d))
    ts = np.arange(n, dtype=np.int64)
    y = O.layer_forward(x, p, [0, n], ts, H, dh)
    sil = lambda a: np.array([_silu(float(t)) for t in a])
    Ub, Vb, Qb, Kb = (sil(p.b1[i * hv:(i + 1) * hv]) for i in range(4))
    want = np.zeros((n, d))
    for i in range(n):
        o = np.zeros(hv)
        for h in range(H):
            s = float(Qb[h * dh:(h + 1) * dh] @ Kb[h * dh:(h + 1) * dh])
            o[h * dh:(h + 1) * dh] = (i + 1) / n * _silu(s) * Vb[h * dh:(h + 1) * dh]
        on = torch.nn.functional.layer_norm(torch.tensor(o), (hv,), torch.tensor(p.ln2_g),
                                            torch.tensor(p.ln2_b), 1e-5).numpy()
        want[i] = x[i] + (on * Ub) @ p.w2.T + p.b2
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)


def test_layer_query_key_orientation():
    """Only the K block of W1 is non-zero, so K varies per token while Q is the
    constant SiLU(b_Q): O_i = (1/n) sum_{j<=i} SiLU(q.k_j) v."""
    d, H, dh, n = 8, 1, 4, 5
    hv = H * dh
    p = _tiny_layer(6, d, H, dh, random_affine=False)
    w1 = np.zeros_like(p.w1)
    w1[3 * hv:4 * hv] = p.w1[3 * hv:4 * hv]
    p.w1 = w1
    p.pos_bias = np.zeros(128)
    p.time_bias = np.zeros(128)
    x = np.random.default_rng(7).normal(size=(n, d))
    ts = np.zeros(n, dtype=np.int64)
    _, it = O.layer_forward(x, p, [0, n], ts, H, dh, return_intermediates=True)
    sil = lambda a: a / (1 + np.exp(-a))
    xh = torch.nn.functional.layer_norm(torch.tensor(x), (d,), eps=1e-5).numpy()
    kt = sil(xh @ w1[3 * hv:].T + p.b1[3 * hv:])
    qb = sil(p.b1[2 * hv:3 * hv])
    vb = sil(p.b1[hv:2 * hv])
    for i in range(n):
        want = sum(_silu(float(qb @ kt[j])) for j in range(i + 1)) / n * vb
        assert np.allclose(it["O"][i, 0], want, rtol=1e-12)


# ----------------------------------------------------------------------------
# backward: central finite differences
# ----------------------------------------------------------------------------

def _fd(f, arr, idx, h=1e-6):
    old = arr[idx]
    arr[idx] = old + h
    fp = f()
    arr[idx] = old - h
    fm = f()
    arr[idx] = old
    return (fp - fm) / (2 * h)


@pytest.mark.parametrize("targets", [None, [2, 0]])
def test_attention_backward_finite_differences(targets):
    d = W.random_attention_inputs(9, [6, 5], 2, 3, "f32", num_targets=targets, qk_std=0.7)
    q, k, v = (d[n].astype(np.float64) for n in ("q", "k", "v"))
    pb, tb = d["pos_bias"].astype(np.float64), d["time_bias"].astype(np.float64)
    g = np.random.default_rng(3).normal(size=v.shape)
    loss = lambda: float((O.attention_forward(q, k, v, d["seq_offsets"], d["timestamps"], pb, tb,
                                              d["num_targets"]) * g).sum())
    dq, dk, dv, dpb, dtb = O.attention_backward(q, k, v, g, d["seq_offsets"], d["timestamps"], pb, tb,
                                                d["num_targets"])
    rng = np.random.default_rng(4)
    for arr, grad in [(q, dq), (k, dk), (v, dv)]:
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            assert abs(_fd(loss, arr, idx) - grad[idx]) < 1e-7 * max(1, abs(grad[idx]))
    for arr, grad in [(pb, dpb), (tb, dtb)]:
        used = np.nonzero(grad)[0][:5]
        assert len(used) > 0
        for b in used:
            assert abs(_fd(loss, arr, (b,)) - grad[b]) < 1e-7 * max(1, abs(grad[b]))


def test_layer_backward_finite_differences():
    H, dh, dm = 2, 3, 8
    p = _tiny_layer(12, dm, H, dh)
    rng = np.random.default_rng(13)
    offs = [0, 5, 9]
    x = rng.normal(size=(9, dm))
    ts = np.concatenate([np.cumsum(rng.integers(1, 3000, 5)), np.cumsum(rng.integers(1, 3000, 4))]).astype(np.int64)
    g = rng.normal(size=(9, dm))
    layers = [p, _tiny_layer(14, dm, H, dh)]
    loss = lambda: float((O.stack_forward(x, layers, offs, ts, H, dh) * g).sum())
    grads = O.stack_backward(x, layers, g, offs, ts, H, dh)
    checks = [(x, grads[0]["dx"])]
    for li, lp in enumerate(layers):
        gr = grads[li]
        checks += [(lp.w1, gr["dw1"]), (lp.b1, gr["db1"]), (lp.w2, gr["dw2"]), (lp.b2, gr["db2"]),
                   (lp.ln1_g, gr["dln1_g"]), (lp.ln1_b, gr["dln1_b"]), (lp.ln2_g, gr["dln2_g"]),
                   (lp.ln2_b, gr["dln2_b"]), (lp.pos_bias, gr["dpos_bias"]), (lp.time_bias, gr["dtime_bias"])]
    for arr, grad in checks:
        for _ in range(3):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            if arr is lp.pos_bias or arr is lp.time_bias:
                nz = np.nonzero(grad)[0]
                idx = (int(nz[rng.integers(0, len(nz))]),)
            fd = _fd(loss, arr, idx)
            assert abs(fd - grad[idx]) < 2e-6 * max(1, abs(grad[idx])), (idx, fd, grad[idx])


# ----------------------------------------------------------------------------
# Stochastic Length
# ----------------------------------------------------------------------------

def test_stochastic_length_rule():
    offs = np.array([0, 3, 13, 20, 30])
    keys = np.array([5, 1, 9,
                     7, 7, 3, 0, 9, 2, 2, 8, 1, 6,
                     4, 4, 4, 4, 4, 4, 4,
                     9, 8, 7, 6, 5, 4, 3, 2, 1, 0], dtype=np.uint32)
    coins = np.array([0, 10, 10, 99], dtype=np.uint32)
    gather, new_offs = O.stochastic_length_select(offs, coins, keys, 4, 50)
    # seq 0: n=3 <= 4 kept whole; seq 1: keys 0,1,2,2 at local 3,8,5,6 -> sorted
    # seq 2: all keys equal -> the first four; seq 3: coin 99 >= 50 -> kept whole
    want = [0, 1, 2, 3 + 3, 3 + 5, 3 + 6, 3 + 8, 13, 14, 15, 16] + list(range(20, 30))
    assert list(gather) == want
    assert list(new_offs) == [0, 3, 7, 11, 21]


def test_sampled_row_functions_match_dense():
    d = W.random_attention_inputs(21, [7, 12], 2, 4, "f32", num_targets=[0, 4], per_head_rab=True)
    dense = O.attention_forward(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], d["pos_bias"],
                                d["time_bias"], d["num_targets"])
    rows = [(0, 0, 0), (0, 6, 1), (1, 3, 0), (1, 9, 1), (1, 11, 0)]
    got = O.attention_rows(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], d["pos_bias"],
                           d["time_bias"], rows, d["num_targets"])
    for r, (s, i, h) in enumerate(rows):
        assert np.allclose(got[r], dense[d["seq_offsets"][s] + i, h], rtol=1e-12, atol=1e-14)
    p = _tiny_layer(22, 8, 2, 4)
    rng = np.random.default_rng(23)
    x = rng.normal(size=(19, 8))
    offs = [0, 7, 19]
    ts = np.concatenate([np.cumsum(rng.integers(1, 900, 7)), np.cumsum(rng.integers(1, 900, 12))]).astype(np.int64)
    y = O.layer_forward(x, p, offs, ts, 2, 4, num_targets=[0, 3])
    yr = O.layer_forward_rows(x, p, offs, ts, 2, 4, [(0, 3), (1, 0), (1, 11)], num_targets=[0, 3])
    assert np.allclose(yr, y[[3, 7, 18]], rtol=1e-12, atol=1e-12)


def test_interleaved_ranking_mask_hides_the_reaction():
    """Ranking over items interleaved with their reactions: the causal mask with
    the diagonal hides an item's own reaction (the next position) and every
    later event, so the oracle's item row does not move when they change, and
    it does move when an earlier reaction changes."""
    wl = W.interleave_item_action(W.make_workload(0, batch=2))
    s_ = wl.spec
    y = O.stack_forward(wl.x, wl.layers, wl.seq_offsets, wl.timestamps, s_.num_heads, s_.head_dim)
    a, z = int(wl.seq_offsets[0]), int(wl.seq_offsets[1])
    k = (z - a) // 4
    item = a + 2 * k
    rng = np.random.default_rng(3)
    x2 = wl.x.copy()
    x2[item + 1:z] = rng.standard_normal((z - item - 1, x2.shape[1]))   # a shift alone would cancel in LayerNorm
    y2 = O.stack_forward(x2, wl.layers, wl.seq_offsets, wl.timestamps, s_.num_heads, s_.head_dim)
    assert np.array_equal(y[a:item + 1], y2[a:item + 1])
    x3 = wl.x.copy()
    x3[item - 1] = rng.standard_normal(x3.shape[1])   # the previous item's reaction
    y3 = O.stack_forward(x3, wl.layers, wl.seq_offsets, wl.timestamps, s_.num_heads, s_.head_dim)
    assert not np.allclose(y[item], y3[item])
