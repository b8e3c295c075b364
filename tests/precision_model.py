"""A rounding model of the bf16 training step, for choosing parity bounds.

TEST INFRASTRUCTURE ONLY.  It restates the fp64 oracle's layer forward and
backward (oracle/hstu_oracle.py: the same equations, in the same order) and
rounds to bf16 at every point where a bf16 kernel path stores a value or feeds
one to a tensor core.  It imports the oracle for the pieces it reuses unchanged
(masks, buckets, LayerNorm) and nothing from the CUDA package.

Rounding points (bf16 weights and activations, fp32 residual stream, fp32
accumulation everywhere):

forward   x-hat = LN1(x);  U, V, Q, K = SiLU(z) and z itself (kept for the
          backward);  P = SiLU(S) as the A operand of P V;  A V / N;
          the gate LN2(A V) * U.
backward  dY (operand of the f2 products);  dg = dY W2;  dO and dU from the
          gate's backward;  P and dS as operands of dV, dK, dQ;  dV, dK, dQ;
          dz = da * SiLU'(z).

`silu_p` chooses how the forward's P is formed: "f32" rounds the exact SiLU
once; "bf16pair" evaluates h = S/2 in bf16, tanh(h) rounded to bf16 and
h + h * tanh(h) rounded to bf16 (a SiLU computed on bf16 pairs, at best).
`band` rounds half of the relative bias to bf16 where |i - j| < 128 (a
precomputed near-diagonal bias band).
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np

import oracle.hstu_oracle as O


def bf16(a) -> np.ndarray:
    """Round to the nearest bf16 (ties to even), through float32; returns float64."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    bits = a32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    r = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


ROUNDING_POINTS = ("xhat", "uvqk", "z", "p_fwd", "attn_out", "gate", "dy", "dg", "dU", "dO", "p_bwd", "ds",
                   "dqkv", "dz")
_enabled = set(ROUNDING_POINTS)


def set_rounding(points) -> None:
    """Round only at the named points (all of ROUNDING_POINTS by default)."""
    global _enabled
    _enabled = set(points)


def _r(name: str, a) -> np.ndarray:
    return bf16(a) if name in _enabled else np.asarray(a, np.float64)


def f32(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def _p_forward(S, silu_p: str):
    if "p_fwd" not in _enabled:
        return O.silu(S)
    if silu_p == "f32":
        return bf16(O.silu(S))
    h = bf16(0.5 * S)
    t = bf16(np.tanh(h))
    return bf16(h + h * t)


def _rab(ts, n, nt, pos_bias, time_bias, band: bool):
    rab, pb, tb = O.rab_matrix(ts, n, nt, pos_bias, time_bias)
    if band:
        i = np.arange(n)[:, None]
        j = np.arange(n)[None, :]
        near = (i - j) < 128
        rab = np.where(near, 2.0 * bf16(0.5 * rab), f32(rab))
    return rab


def attention_forward(q, k, v, offs, ts, pos_bias, time_bias, silu_p="bf16pair", band=True, num_targets=None):
    T, H, dv = v.shape
    out = np.zeros((T, H, dv))
    for s in range(len(offs) - 1):
        a, b = int(offs[s]), int(offs[s + 1])
        n = b - a
        if n == 0:
            continue
        nt = 0 if num_targets is None else int(num_targets[s])
        N = max(n - nt, 1)
        mask = O.attention_mask(n, nt)
        for h in range(H):
            rab = _rab(ts[a:b], n, nt, O._head_table(pos_bias, h), O._head_table(time_bias, h), band and nt == 0)
            S = q[a:b, h] @ k[a:b, h].T + rab
            P = np.where(mask, _p_forward(S, silu_p), 0.0)
            out[a:b, h] = _r('attn_out', (P @ v[a:b, h]) / N)
    return out


def attention_backward(q, k, v, dout, offs, ts, pos_bias, time_bias):
    T, H, dh = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dpos, dtime = np.zeros(128), np.zeros(128)
    for s in range(len(offs) - 1):
        a, b = int(offs[s]), int(offs[s + 1])
        n = b - a
        if n == 0:
            continue
        mask = O.attention_mask(n, 0)
        rab, pb, tb = O.rab_matrix(ts[a:b], n, 0, pos_bias, time_bias)
        for h in range(H):
            S = q[a:b, h] @ k[a:b, h].T + rab
            P = _r('p_bwd', np.where(mask, O.silu(S), 0.0) / n)
            dO = dout[a:b, h]
            dP = dO @ v[a:b, h].T
            dS = np.where(mask, dP * O.silu_grad(S), 0.0) / n
            dpos += np.bincount(pb.ravel(), weights=dS.ravel(), minlength=128)
            dtime += np.bincount(tb.ravel(), weights=dS.ravel(), minlength=128)
            dSb = _r('ds', dS)
            dv[a:b, h] = _r('dqkv', P.T @ dO)
            dk[a:b, h] = _r('dqkv', dSb.T @ q[a:b, h])
            dq[a:b, h] = _r('dqkv', dSb @ k[a:b, h])
    return dq, dk, dv, dpos, dtime


def layer_forward(x, p, offs, ts, H, dh, silu_p="bf16pair", band=True, num_targets=None, io="f32"):
    """One layer; `io` is the type of the residual stream (X and Y): "f32" or "bf16"."""
    T = x.shape[0]
    xh = _r('xhat', O.layer_norm(x, p.ln1_g, p.ln1_b))
    z = xh @ np.asarray(p.w1, np.float64).T + np.asarray(p.b1, np.float64)
    a = _r('uvqk', O.silu(z))
    U, V, Q, K = O.split_uvqk(a, H, dh)
    Oa = attention_forward(Q, K, V, offs, ts, p.pos_bias, p.time_bias, silu_p, band, num_targets)
    on = O.layer_norm(Oa.reshape(T, H * dh), p.ln2_g, p.ln2_b)
    g = _r('gate', on * U.reshape(T, -1))
    y = x + g @ np.asarray(p.w2, np.float64).T + np.asarray(p.b2, np.float64)
    y = bf16(y) if io == "bf16" else f32(y)
    return y, dict(xh=xh, z=_r('z', z), U=U, V=V, Q=Q, K=K, O=Oa, on=on, g=g)


def mfalcon_rank(layers, hist_offsets, hist_x, hist_ts, cand_offsets, cand_x, cand_ts, microbatch, H, dh,
                 silu_p="f32"):
    """M-FALCON scoring with a bf16 residual stream, microbatch by microbatch
    (the oracle's mfalcon_rank with the roundings of the bf16 path)."""
    d = np.asarray(hist_x).shape[1]
    out = np.zeros((int(cand_offsets[-1]), d))
    for u in range(len(hist_offsets) - 1):
        ha, hb = int(hist_offsets[u]), int(hist_offsets[u + 1])
        ca, cb = int(cand_offsets[u]), int(cand_offsets[u + 1])
        for c0 in range(ca, cb, microbatch):
            c1 = min(c0 + microbatch, cb)
            y = np.concatenate([hist_x[ha:hb], cand_x[c0:c1]], axis=0).astype(np.float64)
            ts = np.concatenate([np.asarray(hist_ts[ha:hb]), np.asarray(cand_ts[c0:c1])]).astype(np.int64)
            for p in layers:
                y = layer_forward(y, p, [0, y.shape[0]], ts, H, dh, silu_p, False, [c1 - c0], io="bf16")[0]
            out[c0:c1] = y[hb - ha:]
    return out


def layer_backward(x, p, dy, offs, ts, H, dh, silu_p="bf16pair", band=True) -> Dict[str, np.ndarray]:
    T = x.shape[0]
    hd = H * dh
    _, it = layer_forward(x, p, offs, ts, H, dh, silu_p, band)
    w1 = np.asarray(p.w1, np.float64)
    w2 = np.asarray(p.w2, np.float64)
    dyb = _r('dy', dy)
    dw2 = dyb.T @ it["g"]
    db2 = dy.sum(axis=0)
    dg = _r('dg', dyb @ w2)
    Uf = it["U"].reshape(T, hd)
    dU = _r('dU', dg * it["on"])
    dO, dln2_g, dln2_b = O._layer_norm_backward(it["O"].reshape(T, hd), p.ln2_g, dg * Uf, 1e-5)
    dO = _r('dO', dO)
    dQ, dK, dV, dpos, dtime = attention_backward(it["Q"], it["K"], it["V"], dO.reshape(T, H, dh), offs, ts,
                                                 p.pos_bias, p.time_bias)
    da = np.concatenate([dU, dV.reshape(T, hd), dQ.reshape(T, hd), dK.reshape(T, hd)], axis=1)
    dz = _r('dz', da * O.silu_grad(it["z"]))
    dw1 = dz.T @ it["xh"]
    db1 = dz.sum(axis=0)
    dxh = dz @ w1
    dx_ln, dln1_g, dln1_b = O._layer_norm_backward(x, p.ln1_g, dxh, 1e-5)
    dx = f32(dy + dx_ln)
    return dict(dx=dx, dw1=dw1, db1=db1, dw2=dw2, db2=db2, dln1_g=dln1_g, dln1_b=dln1_b, dln2_g=dln2_g,
                dln2_b=dln2_b, dpos_bias=dpos, dtime_bias=dtime, dU=dU.reshape(T, H, dh), dV=dV, dQ=dQ, dK=dK)


def stack_backward(x, layers: Sequence, dy, offs, ts, H, dh, silu_p="bf16pair", band=True) -> List[Dict]:
    xs = [f32(x)]
    for p in layers[:-1]:
        xs.append(layer_forward(xs[-1], p, offs, ts, H, dh, silu_p, band)[0])
    grads = [None] * len(layers)
    g = f32(dy)
    for li in range(len(layers) - 1, -1, -1):
        grads[li] = layer_backward(xs[li], layers[li], g, offs, ts, H, dh, silu_p, band)
        g = grads[li]["dx"]
    return grads
