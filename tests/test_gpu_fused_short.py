"""GPU parity of the fused short-sequence layer (hstu_layer_fwd with
HSTU_FLAG_SHORT_SEQUENCES: the whole layer in one kernel over work units of at
most 128 token rows holding whole sequences) against the fp64 oracle, on the
short-sequence workload's recipe with its lengths cut to at most 128."""
import numpy as np
import pytest
import torch

import oracle.hstu_oracle as O
from hstu_sequential_transducer_02_b200 import workload as W
from tests.helpers import assert_close, dev, layer_to_dev

pytestmark = pytest.mark.gpu


def _b():
    from hstu_sequential_transducer_02_b200 import binding
    return binding


def _run(wl, short, num_targets=None):
    b = _b()
    s = wl.spec
    layers = [b.Layer(layer_to_dev(p, torch.bfloat16), s.d_model, s.num_heads, s.head_dim, short_sequences=short)
              for p in wl.layers]
    y = dev(wl.x, torch.bfloat16)
    offs, ts = dev(wl.seq_offsets), dev(wl.timestamps)
    nt = None if num_targets is None else dev(np.asarray(num_targets, np.int32))
    b.trace_enable(True)
    for ly in layers:
        y = ly.forward(y, offs, ts, num_targets=nt)
    torch.cuda.synchronize()
    trace = b.trace_read()
    b.trace_enable(False)
    status = [b.workspace_status(ly._ws["fwd"]) for ly in layers]
    return y.float().cpu().numpy(), trace, status


def _ref(wl, num_targets=None):
    s = wl.spec
    return O.stack_forward(wl.x, wl.layers, wl.seq_offsets, wl.timestamps, s.num_heads, s.head_dim,
                           num_targets=num_targets)


def test_fused_short_layer_two_layers():
    """32 sequences of 2 .. 128 tokens (the short-sequence recipe, lengths / 8),
    random LayerNorm affines and biases, two layers: one fused kernel per layer."""
    wl = W.make_workload(1, scale=1 / 8, random_affine=True)
    assert int(np.max(np.diff(wl.seq_offsets))) <= 128
    got, trace, status = _run(wl, True)
    assert trace.get("fused_short_layer", {}).get("count") == 2 and "attn_fwd_tc" not in trace
    assert status == [0, 0]
    assert_close(got, _ref(wl), "bf16", "fused short layer")


def test_fused_short_layer_targets_and_per_head_bias():
    """M-FALCON targets (a candidate sees the history and itself, at position N)
    and one relative-bias table per head; lengths 1, 7, 64, 127, 128 and an empty
    sequence."""
    lens = [1, 7, 64, 0, 127, 128, 90]
    wl = W.make_workload(1, lengths=lens, per_head_rab=True, random_affine=True)
    nt = np.minimum(np.array([0, 3, 10, 0, 100, 40, 0]), lens).astype(np.int32)
    got, trace, status = _run(wl, True, nt)
    assert trace.get("fused_short_layer", {}).get("count") == 2
    assert status == [0, 0]
    assert_close(got, _ref(wl, nt), "bf16", "fused short layer, targets, per-head bias")


def test_fused_short_layer_all_candidates():
    """A sequence made only of candidates (each sees nothing but itself, N = 1):
    the one-term attention is where bf16 operand rounding alone moves the output
    past 3e-2 (tests/test_precision_model.py), so relative Frobenius within 1e-2
    and max-abs within 1.25 times that of the rounding model of the bf16 path."""
    import tests.precision_model as M
    from tests.helpers import errors
    lens = [127, 64]
    wl = W.make_workload(1, lengths=lens, per_head_rab=True, random_affine=True)
    nt = np.array([127, 5], dtype=np.int32)
    got, _, status = _run(wl, True, nt)
    assert status == [0, 0]
    ref = _ref(wl, nt)
    M.set_rounding(M.ROUNDING_POINTS)
    s = wl.spec
    y = wl.x.astype(np.float64)
    for p in wl.layers:
        y = M.layer_forward(y, p, wl.seq_offsets, wl.timestamps, s.num_heads, s.head_dim, silu_p="f32", band=False,
                            num_targets=nt, io="bf16")[0]
    ma, rel = errors(got, ref)
    ma_model = errors(y, ref)[0]
    print(f"all candidates: GPU max-abs {ma:.3e} rel-fro {rel:.3e}; rounding model max-abs {ma_model:.3e}")
    assert rel <= 1e-2 and ma <= max(3e-2, 1.25 * ma_model)


def test_fused_short_layer_matches_layer_path():
    """The fused kernel and the multi-kernel layer both match the oracle, and so
    agree with each other to within twice the bf16 bounds."""
    from tests.helpers import errors
    wl = W.make_workload(1, scale=1 / 8, batch=20)
    fused, _, _ = _run(wl, True)
    plain, trace, _ = _run(wl, False)
    assert "fused_short_layer" not in trace
    ref = _ref(wl)
    assert_close(fused, ref, "bf16", "fused")
    assert_close(plain, ref, "bf16", "layer path")
    ma, rel = errors(fused, plain)
    assert rel <= 2e-2 and ma <= 6e-2


def test_fused_short_layer_reports_long_sequence():
    """A sequence longer than 128 tokens is not computed and is reported in the
    status word; the other sequences are computed as usual."""
    wl = W.make_workload(1, lengths=[50, 200, 30])
    wl.layers = wl.layers[:1]
    got, _, status = _run(wl, True)
    assert status == [_b().ERR_BAD_OFFSETS]
    ref = _ref(wl)
    offs = wl.seq_offsets
    for s_ in (0, 2):
        a, z = offs[s_], offs[s_ + 1]
        assert_close(got[a:z], ref[a:z], "bf16", f"sequence {s_}")


def test_fused_short_layer_packs_many_sequences():
    """Units holding many sequences: 300 sequences of 1 .. 12 tokens, a run of 200
    empty sequences inside one 128-row window (more sequence offsets than rows),
    sequences of exactly 128 tokens starting on and off a window boundary, and
    sequences crossing window boundaries; targets on some of them."""
    rng = np.random.default_rng(7)
    lens = list(rng.integers(1, 13, size=150))
    lens += [0] * 200 + [128, 5, 128, 127, 1, 90, 77]
    lens += list(rng.integers(1, 13, size=150)) + [0, 64, 128]
    wl = W.make_workload(1, lengths=lens, random_affine=True)
    wl.layers = wl.layers[:1]
    lens_a = np.asarray(lens)
    nt = np.where(np.arange(len(lens)) % 7 == 3, np.minimum(2, lens_a), 0).astype(np.int32)
    got, trace, status = _run(wl, True, nt)
    assert trace.get("fused_short_layer", {}).get("count") == 1
    assert status == [0]
    assert_close(got, _ref(wl, nt), "bf16", "fused short layer, many sequences per unit")
