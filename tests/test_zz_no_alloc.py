"""The attention forward entry point that allocates nothing
(hstu_attn_fwd_noalloc), for callers that cannot allocate device memory where
they run the attention: call after call it must give the same result as
hstu_attn_fwd, which takes a caller-provided workspace, and match the fp64
oracle (near the diagonal it evaluates the relative bias per element where
hstu_attn_fwd reads a precomputed bf16 band, so the two agree to within the
bf16 tolerance, not bit for bit).

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test.  It also passes when run alone in a
fresh process: the first call on the device does the library's one-time set-up.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle.hstu_oracle as O
from hstu_sequential_transducer_02_b200 import workload as W
from tests.helpers import assert_close, dev, torch_dtype

pytestmark = pytest.mark.gpu


def _lib():
    from hstu_sequential_transducer_02_b200 import binding as b
    f = b._lib.hstu_attn_fwd_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(b.AttnDesc), ctypes.POINTER(b.Jagged), ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    return b, f


def _call_noalloc(b, f, q, k, v, offs, ts, pb, tb, H, nt, out, total_tokens=None):
    dh = q.shape[1] // H
    desc = b.attn_desc(H, dh, b.DTYPE_F32 if q.dtype == torch.float32 else b.DTYPE_BF16, pb.dim() == 2)
    jb = b.jagged(offs, ts, q.shape[0] if total_tokens is None else total_tokens, nt)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(ctypes.byref(desc), ctypes.byref(jb), p(q), q.stride(0), p(k), k.stride(0), p(v), v.stride(0), p(pb),
             p(tb), p(out), out.stride(0), stream)


@pytest.mark.parametrize("dtype_name,dh,per_head,targets", [("bf16", 128, False, [0, 30, 0, 200]),
                                                             ("bf16", 64, True, None),
                                                             ("f32", 32, False, [3, 0, 0, 1])])
def test_noalloc_matches_workspace_entry_point(dtype_name, dh, per_head, targets):
    b, f = _lib()
    H = 2
    d = W.random_attention_inputs(101 + dh, [300, 129, 1, 640], H, dh, dtype_name, num_targets=targets,
                                  per_head_rab=per_head)
    td = torch_dtype(dtype_name)
    T = d["q"].shape[0]
    q, k, v = (dev(d[n].reshape(T, H * dh), td) for n in ("q", "k", "v"))
    offs, ts, pb, tb = dev(d["seq_offsets"]), dev(d["timestamps"]), dev(d["pos_bias"]), dev(d["time_bias"])
    nt = None if targets is None else dev(d["num_targets"])
    ref = b.attn_fwd(q, k, v, offs, ts, pb, tb, H, num_targets=nt)
    torch.cuda.synchronize()
    ref = ref.float().cpu().numpy().astype(np.float64)
    oracle = O.attention_forward(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], d["pos_bias"],
                                 d["time_bias"], d["num_targets"]).reshape(T, H * dh)
    for _ in range(2):  # two calls in a row share (and overwrite) the library's scratch array
        out = torch.full((T, H * dh), float("nan"), dtype=td, device="cuda")
        assert _call_noalloc(b, f, q, k, v, offs, ts, pb, tb, H, nt, out) == b.OK
        torch.cuda.synchronize()
        assert_close(out, ref, dtype_name, "no-alloc vs workspace entry point")
        assert_close(out, oracle, dtype_name, "no-alloc vs oracle")


def test_noalloc_refuses_problems_beyond_its_scratch():
    b, f = _lib()
    H, dh = 8, 64
    T = 64
    q = torch.zeros(T, H * dh, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    offs = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    ts = torch.zeros(T, dtype=torch.int64, device="cuda")
    pb = torch.zeros(128, dtype=torch.float32, device="cuda")
    # a capacity of 2^30 rows asks for far more work-list space than the array holds
    rc = _call_noalloc(b, f, q, q, q, offs, ts, pb, pb, H, None, out, total_tokens=1 << 30)
    assert rc == b.ERR_WORKSPACE
    torch.cuda.synchronize()
