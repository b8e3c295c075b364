"""fp64 CPU oracle for the HSTU layer, its attention, M-FALCON ranking and
Stochastic Length.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
baseline leg of the benchmark may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from the product package.

It is a plain, slow, direct statement of what the HSTU pages describe, written
with NumPy in float64: per sequence and per head it builds the dense n x n score
matrix, applies the relative bias, the pointwise SiLU, the mask and the 1/N
scale, and multiplies by V.  No blocking, fusion or reordering beyond that.

Sources (titles of the pages; sections as printed there):
* "Actions Speak Louder than Words" summary (Chinese), "1.2 HSTU架构核心组件":
  the three sub-layers (pointwise projection, pointwise aggregated attention
  without softmax, relative attention bias from position and time); "2.3
  M-FALCON算法"; "2.1 随机长度 (Stochastic Length)".
* "生成式推荐（一）：HSTU" (CSDN), section "高性能自注意力Encoder：HSTU":
  f1 and f2 are single linear layers, phi1 = phi2 = SiLU, Norm = LayerNorm,
  output Norm(A(X)V(X)) * U(X); "Pointwise aggregated attention" (no
  normalisation over the sequence); "M-FALCON" (the mask and the rab are
  changed so that the b_m candidates' attention is identical).
* "Meta HSTU" case study (Russian), "Что меняется внутри HSTU": Q, K, V and U are
  built jointly, aggregation with position and time offsets, normalisation after
  aggregation, element-wise product with U, output transform, residual
  connections; "M-FALCON переиспользует историю"; "Разная длина истории".

The pages lost the equations themselves in extraction.  The layer equations
used here are the specification's:
    U, V, Q, K = Split(SiLU(f1(LayerNorm(X))))
    A V        = (SiLU(Q K^T + rab^{p,t}) / N  (.) mask) V
    Y          = X + f2(LayerNorm(A V) (.) U)
with position bucket clamp(i - j, 0, 127) and time bucket
clamp(floor(ln(max(1, |t_i - t_j|)) / 0.301), 0, 127).

Readings adopted where the pages are silent (each is listed in the design
notes as well):
* N is the number of history (non-candidate) tokens of the sequence, at least 1.
* No 1/sqrt(d) scaling of Q K^T.
* The causal mask includes the diagonal (j == i).
* An M-FALCON candidate sits at position N (the history length) for the
  position bias; it sees history j < N and itself (pos bucket 0, dt = 0).
* Split order along the 4*H*dh columns is U, V, Q, K; inside each block the
  columns are head-major (head h owns columns h*dh .. h*dh + dh - 1).
* LayerNorm uses the biased variance and eps = 1e-5; LN2 spans all heads.
* Linear layers have biases; weights are stored (out, in): y = x W^T + b.
* Stochastic Length: a sequence longer than L is subsampled when its coin is
  below p (integer compare on uint32 draws); it then keeps the L tokens with
  the smallest uint32 keys (ties to the lower index), in original order.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

NUM_POS_BUCKETS = 128
NUM_TIME_BUCKETS = 128


# ----------------------------------------------------------------------------
# elementwise pieces
# ----------------------------------------------------------------------------

def silu(x):
    """SiLU(x) = x * sigmoid(x) (phi1 = phi2 = SiLU, CSDN page, HSTU encoder section)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def silu_grad(x):
    """d/dx [x * sigmoid(x)] = sigmoid(x) * (1 + x * (1 - sigmoid(x)))."""
    x = np.asarray(x, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-x))
    return s * (1.0 + x * (1.0 - s))


def time_bucket(dt, time_div: float = 0.301, num_buckets: int = NUM_TIME_BUCKETS):
    """Time bucket of a timestamp difference in seconds.

    clamp(floor(ln(max(1, |dt|)) / time_div), 0, num_buckets - 1), evaluated in
    fp64 with the C library's natural logarithm.
    """
    dt = np.abs(np.asarray(dt, dtype=np.int64)).astype(np.float64)
    dt = np.maximum(dt, 1.0)
    b = np.floor(np.log(dt) / time_div)
    return np.clip(b, 0, num_buckets - 1).astype(np.int64)


def pos_bucket(delta, num_buckets: int = NUM_POS_BUCKETS):
    """Position bucket: clamp(pos_i - pos_j, 0, num_buckets - 1)."""
    return np.clip(np.asarray(delta, dtype=np.int64), 0, num_buckets - 1)


def layer_norm(x, gamma, beta, eps: float = 1e-5):
    """Row LayerNorm with biased variance (Norm = LayerNorm, CSDN page)."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


# ----------------------------------------------------------------------------
# positions and masks of one sequence
# ----------------------------------------------------------------------------

def history_length(n: int, num_targets: int) -> int:
    return n - num_targets


def positions(n: int, num_targets: int = 0) -> np.ndarray:
    """Position index of each token: history tokens 0..N-1, every candidate N."""
    N = history_length(n, num_targets)
    return np.minimum(np.arange(n, dtype=np.int64), N)


def attention_mask(n: int, num_targets: int = 0) -> np.ndarray:
    """Boolean [n, n] mask: causal over the history (diagonal included); an
    M-FALCON candidate i >= N sees the history j < N and itself only."""
    N = history_length(n, num_targets)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    return (j <= i) & ((j < N) | (j == i))


def rab_matrix(ts, n: int, num_targets: int, pos_bias, time_bias, time_div: float = 0.301):
    """rab^{p,t}_{ij} = pos_bias[pb(i,j)] + time_bias[tb(i,j)] for one sequence/head."""
    p = positions(n, num_targets)
    pb = pos_bucket(p[:, None] - p[None, :])
    ts = np.asarray(ts, dtype=np.int64)
    tb = time_bucket(ts[:, None] - ts[None, :], time_div)
    return np.asarray(pos_bias, np.float64)[pb] + np.asarray(time_bias, np.float64)[tb], pb, tb


def _head_table(table, h):
    t = np.asarray(table)
    return t if t.ndim == 1 else t[h]


# ----------------------------------------------------------------------------
# attention (pointwise aggregated attention)
# ----------------------------------------------------------------------------

def attention_forward(q, k, v, seq_offsets, timestamps, pos_bias, time_bias,
                      num_targets=None, time_div: float = 0.301):
    """O_i = (1/N) * sum_{j : mask(i,j)} SiLU(q_i . k_j + rab_ij) v_j, per sequence and head.

    q, k: [T, H, dqk]; v: [T, H, dv]; returns O [T, H, dv] in fp64.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, _ = q.shape
    out = np.zeros((T, H, v.shape[2]), dtype=np.float64)
    offs = np.asarray(seq_offsets, dtype=np.int64)
    for s in range(len(offs) - 1):
        a, b = int(offs[s]), int(offs[s + 1])
        n = b - a
        if n == 0:
            continue
        nt = 0 if num_targets is None else int(num_targets[s])
        N = max(history_length(n, nt), 1)
        mask = attention_mask(n, nt)
        for h in range(H):
            rab, _, _ = rab_matrix(timestamps[a:b], n, nt, _head_table(pos_bias, h),
                                   _head_table(time_bias, h), time_div)
            S = q[a:b, h, :] @ k[a:b, h, :].T + rab
            P = np.where(mask, silu(S), 0.0) / N
            out[a:b, h, :] = P @ v[a:b, h, :]
    return out


def attention_forward_pairwise(q, k, v, seq_offsets, timestamps, pos_bias, time_bias,
                               num_targets=None, time_div: float = 0.301):
    """The same sum written as an explicit loop over (i, j) pairs (tiny inputs only)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, _ = q.shape
    out = np.zeros((T, H, v.shape[2]))
    offs = [int(o) for o in seq_offsets]
    for s in range(len(offs) - 1):
        a, b = offs[s], offs[s + 1]
        n = b - a
        nt = 0 if num_targets is None else int(num_targets[s])
        N = max(n - nt, 1)
        for h in range(H):
            pt = _head_table(pos_bias, h)
            tt = _head_table(time_bias, h)
            for i in range(n):
                pi = min(i, n - nt)
                acc = np.zeros(v.shape[2])
                for j in range(n):
                    if j > i:
                        continue
                    if i >= n - nt and j >= n - nt and j != i:
                        continue
                    pj = min(j, n - nt)
                    pb = min(max(pi - pj, 0), NUM_POS_BUCKETS - 1)
                    dt = abs(int(timestamps[a + i]) - int(timestamps[a + j]))
                    tb = int(math.floor(math.log(max(dt, 1)) / time_div))
                    tb = min(max(tb, 0), NUM_TIME_BUCKETS - 1)
                    sc = float(np.dot(q[a + i, h], k[a + j, h])) + float(pt[pb]) + float(tt[tb])
                    acc += sc / (1.0 + math.exp(-sc)) * v[a + j, h]
                out[a + i, h] = acc / N
    return out


def attention_rows(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, rows, num_targets=None,
                   time_div: float = 0.301):
    """The same O_i for selected (sequence, row, head) triples only, one row at a
    time, so that very long sequences can be checked on sampled outputs.
    Returns [len(rows), dv]."""
    out = np.zeros((len(rows), np.asarray(v).shape[2]))
    offs = np.asarray(seq_offsets, dtype=np.int64)
    for r, (s, i, h) in enumerate(rows):
        a, b = int(offs[s]), int(offs[s + 1])
        n = b - a
        nt = 0 if num_targets is None else int(num_targets[s])
        N = max(history_length(n, nt), 1)
        j = np.arange(n)
        att = (j <= i) & ((j < n - nt) | (j == i))
        p = np.minimum(np.arange(n), n - nt)
        pb = pos_bucket(p[i] - p)
        tb = time_bucket(np.asarray(timestamps[a:b], np.int64)[i] - np.asarray(timestamps[a:b], np.int64), time_div)
        rab = np.asarray(_head_table(pos_bias, h), np.float64)[pb] + np.asarray(_head_table(time_bias, h), np.float64)[tb]
        sc = np.asarray(k[a:b, h], np.float64) @ np.asarray(q[a + i, h], np.float64) + rab
        w = np.where(att, silu(sc), 0.0) / N
        out[r] = w @ np.asarray(v[a:b, h], np.float64)
    return out


def attention_backward(q, k, v, dout, seq_offsets, timestamps, pos_bias, time_bias,
                       num_targets=None, time_div: float = 0.301):
    """Gradients of sum(O * dout) with respect to q, k, v and the two rab tables.

    With P_ij = mask_ij SiLU(S_ij) / N and O = P V:
      dV = P^T dO;  dP = dO V^T;  dS = dP * mask * SiLU'(S) / N;
      dQ = dS K;    dK = dS^T Q;  d_pos[b] = sum of dS over pairs in position bucket b,
      d_time[b] likewise over time buckets.
    Returns dq, dk, dv, d_pos_bias, d_time_bias (rab grads shaped like the tables).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    T, H, _ = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dpos = np.zeros(np.asarray(pos_bias).shape)
    dtime = np.zeros(np.asarray(time_bias).shape)
    offs = np.asarray(seq_offsets, dtype=np.int64)
    for s in range(len(offs) - 1):
        a, b = int(offs[s]), int(offs[s + 1])
        n = b - a
        if n == 0:
            continue
        nt = 0 if num_targets is None else int(num_targets[s])
        N = max(history_length(n, nt), 1)
        mask = attention_mask(n, nt)
        for h in range(H):
            rab, pb, tb = rab_matrix(timestamps[a:b], n, nt, _head_table(pos_bias, h),
                                     _head_table(time_bias, h), time_div)
            S = q[a:b, h] @ k[a:b, h].T + rab
            P = np.where(mask, silu(S), 0.0) / N
            dO = dout[a:b, h]
            dv[a:b, h] += P.T @ dO
            dP = dO @ v[a:b, h].T
            dS = np.where(mask, dP * silu_grad(S), 0.0) / N
            dq[a:b, h] += dS @ k[a:b, h]
            dk[a:b, h] += dS.T @ q[a:b, h]
            gp = np.bincount(pb.ravel(), weights=dS.ravel(), minlength=NUM_POS_BUCKETS)
            gt = np.bincount(tb.ravel(), weights=dS.ravel(), minlength=NUM_TIME_BUCKETS)
            if dpos.ndim == 1:
                dpos += gp
                dtime += gt
            else:
                dpos[h] += gp
                dtime[h] += gt
    return dq, dk, dv, dpos, dtime


# ----------------------------------------------------------------------------
# the layer
# ----------------------------------------------------------------------------

def split_uvqk(a, num_heads: int, head_dim: int):
    """Split the 4*H*dh projection output into U, V, Q, K, each [T, H, dh]."""
    T = a.shape[0]
    hd = num_heads * head_dim
    U = a[:, 0 * hd:1 * hd].reshape(T, num_heads, head_dim)
    V = a[:, 1 * hd:2 * hd].reshape(T, num_heads, head_dim)
    Q = a[:, 2 * hd:3 * hd].reshape(T, num_heads, head_dim)
    K = a[:, 3 * hd:4 * hd].reshape(T, num_heads, head_dim)
    return U, V, Q, K


def layer_forward(x, p, seq_offsets, timestamps, num_heads: int, head_dim: int,
                  num_targets=None, eps: float = 1e-5, time_div: float = 0.301,
                  return_intermediates: bool = False):
    """One HSTU layer in fp64.

    x: [T, d]; p: object with w1 [4Hdh, d], b1, ln1_g, ln1_b, ln2_g, ln2_b,
    w2 [d, Hdh], b2, pos_bias, time_bias.
    """
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    xh = layer_norm(x, p.ln1_g, p.ln1_b, eps)
    z = xh @ np.asarray(p.w1, np.float64).T + np.asarray(p.b1, np.float64)
    a = silu(z)
    U, V, Q, K = split_uvqk(a, num_heads, head_dim)
    O = attention_forward(Q, K, V, seq_offsets, timestamps, p.pos_bias, p.time_bias,
                          num_targets, time_div)
    o2 = O.reshape(T, num_heads * head_dim)
    on = layer_norm(o2, p.ln2_g, p.ln2_b, eps)
    g = on * U.reshape(T, -1)
    y = x + g @ np.asarray(p.w2, np.float64).T + np.asarray(p.b2, np.float64)
    if return_intermediates:
        return y, dict(xh=xh, z=z, a=a, U=U, V=V, Q=Q, K=K, O=O, on=on, g=g)
    return y


def layer_forward_rows(x, p, seq_offsets, timestamps, num_heads: int, head_dim: int, rows,
                       num_targets=None, eps: float = 1e-5, time_div: float = 0.301):
    """Y for selected (sequence, row) pairs of one layer: the projection of the
    whole sequence, then attention, LayerNorm, gate and f2 for those rows only.
    Returns [len(rows), d]."""
    x = np.asarray(x, np.float64)
    offs = np.asarray(seq_offsets, dtype=np.int64)
    out = np.zeros((len(rows), x.shape[1]))
    cache = {}
    for r, (s, i) in enumerate(rows):
        a, b = int(offs[s]), int(offs[s + 1])
        if s not in cache:
            xh = layer_norm(x[a:b], p.ln1_g, p.ln1_b, eps)
            act = silu(xh @ np.asarray(p.w1, np.float64).T + np.asarray(p.b1, np.float64))
            cache[s] = split_uvqk(act, num_heads, head_dim)
        U, V, Q, K = cache[s]
        loc = np.array([0, b - a])
        nt = None if num_targets is None else [num_targets[s]]
        o = np.concatenate([attention_rows(Q, K, V, loc, timestamps[a:b], p.pos_bias, p.time_bias, [(0, i, h)],
                                           nt, time_div)[0] for h in range(num_heads)])
        on = layer_norm(o[None, :], p.ln2_g, p.ln2_b, eps)[0]
        out[r] = x[a + i] + (on * U[i].reshape(-1)) @ np.asarray(p.w2, np.float64).T + np.asarray(p.b2, np.float64)
    return out


def stack_forward(x, layers: Sequence, seq_offsets, timestamps, num_heads, head_dim,
                  num_targets=None, eps=1e-5, time_div=0.301):
    y = np.asarray(x, np.float64)
    for p in layers:
        y = layer_forward(y, p, seq_offsets, timestamps, num_heads, head_dim, num_targets, eps, time_div)
    return y


def _layer_norm_backward(x, gamma, dy, eps):
    """Backward of row LayerNorm y = xhat * gamma + beta; returns dx, dgamma, dbeta."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    r = 1.0 / np.sqrt(var + eps)
    xhat = (x - mu) * r
    dgamma = (dy * xhat).sum(axis=0)
    dbeta = dy.sum(axis=0)
    dxh = dy * np.asarray(gamma, np.float64)
    dx = r * (dxh - dxh.mean(axis=-1, keepdims=True) - xhat * (dxh * xhat).mean(axis=-1, keepdims=True))
    return dx, dgamma, dbeta


def layer_backward(x, p, dy, seq_offsets, timestamps, num_heads: int, head_dim: int,
                   num_targets=None, eps: float = 1e-5, time_div: float = 0.301) -> Dict[str, np.ndarray]:
    """Hand-derived fp64 backward of `layer_forward` for the loss sum(Y * dy)."""
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    T = x.shape[0]
    hd = num_heads * head_dim
    y, it = layer_forward(x, p, seq_offsets, timestamps, num_heads, head_dim, num_targets, eps,
                          time_div, return_intermediates=True)
    w1 = np.asarray(p.w1, np.float64)
    w2 = np.asarray(p.w2, np.float64)
    # y = x + g W2^T + b2
    dw2 = dy.T @ it["g"]
    db2 = dy.sum(axis=0)
    dg = dy @ w2
    # g = on * U
    Uf = it["U"].reshape(T, hd)
    dU = dg * it["on"]
    don = dg * Uf
    # on = LN2(O)
    dO, dln2_g, dln2_b = _layer_norm_backward(it["O"].reshape(T, hd), p.ln2_g, don, eps)
    dQ, dK, dV, dpos, dtime = attention_backward(it["Q"], it["K"], it["V"], dO.reshape(T, num_heads, head_dim),
                                                 seq_offsets, timestamps, p.pos_bias, p.time_bias,
                                                 num_targets, time_div)
    da = np.concatenate([dU, dV.reshape(T, hd), dQ.reshape(T, hd), dK.reshape(T, hd)], axis=1)
    dz = da * silu_grad(it["z"])
    dw1 = dz.T @ it["xh"]
    db1 = dz.sum(axis=0)
    dxh = dz @ w1
    dx_ln, dln1_g, dln1_b = _layer_norm_backward(x, p.ln1_g, dxh, eps)
    dx = dy + dx_ln
    return dict(dx=dx, dw1=dw1, db1=db1, dw2=dw2, db2=db2, dln1_g=dln1_g, dln1_b=dln1_b,
                dln2_g=dln2_g, dln2_b=dln2_b, dpos_bias=dpos, dtime_bias=dtime,
                dU=dU.reshape(T, num_heads, head_dim), dV=dV, dQ=dQ, dK=dK, y=y)


def stack_backward(x, layers: Sequence, dy, seq_offsets, timestamps, num_heads, head_dim,
                   num_targets=None, eps=1e-5, time_div=0.301) -> List[Dict[str, np.ndarray]]:
    """Backward through a residual stack; returns per-layer gradient dicts (layer order)."""
    xs = [np.asarray(x, np.float64)]
    for p in layers[:-1]:
        xs.append(layer_forward(xs[-1], p, seq_offsets, timestamps, num_heads, head_dim,
                                num_targets, eps, time_div))
    grads: List[Dict[str, np.ndarray]] = [None] * len(layers)
    g = np.asarray(dy, np.float64)
    for li in range(len(layers) - 1, -1, -1):
        r = layer_backward(xs[li], layers[li], g, seq_offsets, timestamps, num_heads, head_dim,
                           num_targets, eps, time_div)
        grads[li] = r
        g = r["dx"]
    return grads


# ----------------------------------------------------------------------------
# M-FALCON ranking
# ----------------------------------------------------------------------------

def mfalcon_rank(layers: Sequence, hist_offsets, hist_x, hist_ts, cand_offsets, cand_x, cand_ts,
                 microbatch: int, num_heads: int, head_dim: int, eps=1e-5, time_div=0.301):
    """Score every candidate of every user in microbatches of b_m.

    For each user and each microbatch, the sequence [history ; b_m candidates]
    runs through the stack with the M-FALCON mask (candidates see the history
    and themselves); the final-layer rows of the candidates are returned,
    [sum of candidates, d].  ("2.3 M-FALCON算法" and the CSDN "M-FALCON"
    section: one forward pass scores the whole microbatch.)
    """
    hist_x = np.asarray(hist_x, np.float64)
    cand_x = np.asarray(cand_x, np.float64)
    d = hist_x.shape[1]
    out = np.zeros((int(cand_offsets[-1]), d))
    for u in range(len(hist_offsets) - 1):
        ha, hb = int(hist_offsets[u]), int(hist_offsets[u + 1])
        ca, cb = int(cand_offsets[u]), int(cand_offsets[u + 1])
        for c0 in range(ca, cb, microbatch):
            c1 = min(c0 + microbatch, cb)
            xs = np.concatenate([hist_x[ha:hb], cand_x[c0:c1]], axis=0)
            ts = np.concatenate([np.asarray(hist_ts[ha:hb]), np.asarray(cand_ts[c0:c1])]).astype(np.int64)
            offs = np.array([0, xs.shape[0]])
            y = stack_forward(xs, layers, offs, ts, num_heads, head_dim,
                              num_targets=np.array([c1 - c0]), eps=eps, time_div=time_div)
            out[c0:c1] = y[hb - ha:]
    return out


# ----------------------------------------------------------------------------
# Stochastic Length
# ----------------------------------------------------------------------------

def stochastic_length_select(seq_offsets, coins, keys, max_len: int, prob_u32: int):
    """Token indices kept by Stochastic Length, and the new offsets.

    A sequence longer than max_len is subsampled when coins[s] < prob_u32 (so
    with probability p = prob_u32 / 2^32); it then keeps the max_len tokens with
    the smallest keys (ties to the lower index), in their original order.
    Other sequences are kept whole.  ("2.1 随机长度": random sub-sequences of
    long histories in training, sometimes the whole history.)
    """
    offs = np.asarray(seq_offsets, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.uint32)
    kept = []
    new_len = []
    for s in range(len(offs) - 1):
        a, b = int(offs[s]), int(offs[s + 1])
        n = b - a
        if n > max_len and int(coins[s]) < int(prob_u32):
            order = sorted(range(n), key=lambda t: (int(keys[a + t]), t))[:max_len]
            idx = a + np.sort(np.asarray(order, dtype=np.int64))
        else:
            idx = np.arange(a, b, dtype=np.int64)
        kept.append(idx)
        new_len.append(len(idx))
    gather = np.concatenate(kept) if kept else np.zeros(0, np.int64)
    new_offs = np.zeros(len(new_len) + 1, dtype=np.int64)
    np.cumsum(new_len, out=new_offs[1:])
    return gather.astype(np.int64), new_offs.astype(np.int32)


# ----------------------------------------------------------------------------
# work accounting used by the measurement (not part of the computation)
# ----------------------------------------------------------------------------

def attention_pairs(seq_offsets, num_targets=None) -> int:
    """Number of unmasked (i, j) pairs over all sequences."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    total = 0
    for s in range(len(offs) - 1):
        n = int(offs[s + 1] - offs[s])
        nt = 0 if num_targets is None else int(num_targets[s])
        N = n - nt
        total += N * (N + 1) // 2 + nt * (N + 1)
    return total
