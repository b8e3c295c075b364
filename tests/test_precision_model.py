"""The bf16 rounding model of the training step (tests/precision_model.py),
pinned to the oracle, and what it shows about the achievable gradient error.

CPU only.  The model is the oracle's layer with explicit bf16 roundings; with
every rounding switched off it must reproduce the oracle, and its errors then
say which bounds a bf16 tensor-core path can meet on the training workload."""
import numpy as np
import pytest

import oracle.hstu_oracle as O
import tests.precision_model as M
from hstu_sequential_transducer_02_b200 import workload as W

NAMES = ("dU", "dV", "dQ", "dK", "dpos_bias", "dtime_bias", "dw1", "dw2", "db1", "dln1_g", "dln1_b", "dln2_g",
         "dln2_b", "dx")


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - b) / np.linalg.norm(b))


@pytest.fixture(scope="module")
def c4():
    """The training workload the GPU tests use (B = 6, lengths x 1/8, 8 layers), after SL."""
    wl = W.make_workload(4, batch=6, scale=1 / 8, random_affine=True)
    e = wl.extras
    g, offs = O.stochastic_length_select(wl.seq_offsets, e["sl_coin"], e["sl_keys"], int(e["sl_len"]),
                                         int(e["sl_prob_u32"]))
    x0, ts, g0 = wl.x[g].astype(np.float64), wl.timestamps[g], e["grad_out"][g].astype(np.float64)
    s = wl.spec
    ref = O.stack_backward(x0, wl.layers, g0, offs, ts, s.num_heads, s.head_dim)
    yield wl, x0, ts, g0, offs, ref
    M.set_rounding(M.ROUNDING_POINTS)


def _worst(wl, got, ref):
    return max(_rel(got[li][n], ref[li][n]) for li in range(len(wl.layers)) for n in NAMES)


def test_bf16_rounding_of_the_model():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.0 - 2 ** -7, 1e-40, 3.0e38])
    got = M.bf16(x)
    assert got[0] == 1.0 and got[1] == 1.0          # tie to even
    assert got[2] == 1.0 + 2 ** -6                  # tie to even (odd neighbour below)
    assert got[3] == -2.0                           # halfway between -2 and -2 - 2^-6: to even
    assert abs(got[4]) < 1e-37
    assert got[5] == (1 + 98 / 128) * 2.0 ** 127    # 3e38 = 1.7632 * 2^127 -> 7-bit mantissa 98/128
    assert np.all(got.astype(np.float32).view(np.uint32) & 0xFFFF == 0)


def test_model_without_rounding_is_the_oracle(c4):
    wl, x0, ts, g0, offs, ref = c4
    M.set_rounding([])
    s = wl.spec
    got = M.stack_backward(x0, wl.layers, g0, offs, ts, s.num_heads, s.head_dim, band=False)
    # only the fp32 residual stream is rounded
    assert _worst(wl, got, ref) < 1e-5


def test_tensor_core_operands_alone_exceed_the_bf16_bound(c4):
    """Rounding only x-hat and U, V, Q, K (the forward's tensor-core operands)
    to bf16, all else exact, already moves the 8-layer stack's gradients beyond
    a relative Frobenius error of 1e-2."""
    wl, x0, ts, g0, offs, ref = c4
    M.set_rounding(["xhat", "uvqk"])
    s = wl.spec
    got = M.stack_backward(x0, wl.layers, g0, offs, ts, s.num_heads, s.head_dim, silu_p="f32", band=False)
    assert _worst(wl, got, ref) > 1e-2


def test_per_layer_error_of_the_bf16_path_is_within_bound(c4):
    """Every layer fed the oracle's own input and upstream gradient, with every
    bf16 rounding point of the path: each gradient within 1e-2."""
    wl, x0, ts, g0, offs, ref = c4
    s = wl.spec
    xs = [x0]
    for p in wl.layers[:-1]:
        xs.append(O.layer_forward(xs[-1], p, offs, ts, s.num_heads, s.head_dim))
    dys = [None] * len(wl.layers)
    dys[-1] = g0
    for li in range(len(wl.layers) - 1, 0, -1):
        dys[li - 1] = ref[li]["dx"]
    M.set_rounding(M.ROUNDING_POINTS)
    worst = 0.0
    for li in range(len(wl.layers)):
        r = M.layer_backward(xs[li], wl.layers[li], dys[li], offs, ts, s.num_heads, s.head_dim, silu_p="f32")
        worst = max(worst, max(_rel(r[n], ref[li][n]) for n in NAMES))
    assert worst < 1e-2


def test_one_term_candidates_exceed_the_max_abs_bound_from_operand_rounding():
    """M-FALCON candidates of a user without history attend only to themselves.
    Through two layers, rounding only x-hat, or only U, V, Q, K, to bf16 (the
    tensor cores' operands), all else exact, moves their outputs by more than
    3e-2 (the specification's bf16 max-abs bound) against the oracle, while the
    relative Frobenius error stays within 1e-2."""
    hist_lens, counts, mb = [64, 0, 37], [5, 9, 3], 7
    wl = W.make_workload(3, scale=1 / 32, batch=3, lengths=hist_lens)
    e = wl.extras
    s = wl.spec
    co = e["cand_offsets"]
    sel = np.concatenate([np.arange(co[u], co[u] + counts[u]) for u in range(3)]).astype(np.int64)
    cand_offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    args = (wl.seq_offsets, wl.x, wl.timestamps, cand_offsets, e["cand_x"][sel], e["cand_ts"][sel], mb,
            s.num_heads, s.head_dim)
    ref = O.mfalcon_rank([wl.layers[0]] * 2, *args)
    try:
        for pts in (["xhat"], ["uvqk"]):
            M.set_rounding(pts)
            got = M.mfalcon_rank([wl.layers[0]] * 2, *args)
            assert np.max(np.abs(got - ref)) > 3e-2, pts
            assert _rel(got, ref) < 1e-2, pts
    finally:
        M.set_rounding(M.ROUNDING_POINTS)
