"""Seeded synthetic workloads for the HSTU layer and its M-FALCON ranking use.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no LayerNorm, no projection, no attention, no bucketing).
Both the fp64 oracle tests and the CUDA path consume its arrays, so both sides
see bit-identical inputs.

Shapes follow the workloads the HSTU pages describe: jagged, long-tailed user
histories with monotone timestamps ("Actions Speak Louder than Words" summary,
section 1.3 and 2.1; the Meta HSTU case study, "Разная длина истории"), plus the
five configurations the layer is specified on:

* 0  tiny fp32, 1 layer, B=4, n~U{8..64}, d=64, H=2, dh=32, causal
* 1  bf16, 2 layers, B=32, n~power law(1.5) on [16,1024], d=256, H=4, dh=64
* 2  bf16, 1 layer, B=8, n~U{4096..8192}, d=512, H=4, dh=128 (long history)
* 3  M-FALCON ranking: 16 users x (2048 history + 4096 candidates), b_m=512,
     d=256, H=2, dh=128, 1 layer
* 4  training: 8 layers, B=64, n~power law(1.5) on [64,4096], d=512, H=8,
     dh=64, Stochastic Length (L=1024, subsample probability 0.8)

Random streams (numpy PCG64, seed 20240 + config id, spawned in this order):
lengths, timestamps, X, weights, rab tables, extras (SL draws, candidates, G).

bf16 configurations round X and all weight matrices to bf16 (round to nearest
even) before they are returned, stored in float32 so that every consumer sees
the same values exactly.  rab tables, LayerNorm affine vectors and linear
biases stay fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

SEED_BASE = 20240
TIME_BASE = 1_700_000_000  # seconds; timestamps are int64 seconds from the epoch
GAP_MEAN_S = 600.0
RAB_STD = 0.02
NUM_POS_BUCKETS = 128
NUM_TIME_BUCKETS = 128
TIME_DIV = 0.301
LN_EPS = 1e-5


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bf16 (ties to even); returns float32."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    bits = a32.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = rounded.view(np.float32).copy()
    # keep NaN as NaN (never produced by this generator, but stay well defined)
    nan = np.isnan(a32)
    if nan.any():
        out[nan] = np.nan
    return out


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    return (a32.view(np.uint32) >> 16).astype(np.uint16)


@dataclass
class ConfigSpec:
    cid: int
    name: str
    num_layers: int
    d_model: int
    num_heads: int
    head_dim: int
    dtype: str                     # "f32" or "bf16"
    batch: int = 0
    len_kind: str = "uniform"      # "uniform" | "powerlaw" | "fixed"
    len_lo: int = 0
    len_hi: int = 0
    # M-FALCON
    users: int = 0
    hist_len: int = 0
    num_candidates: int = 0
    microbatch: int = 0
    # Stochastic Length
    sl_len: int = 0
    sl_prob: float = 0.0
    training: bool = False


CONFIGS: Dict[int, ConfigSpec] = {
    0: ConfigSpec(0, "tiny-fp32-1layer", 1, 64, 2, 32, "f32", batch=4,
                  len_kind="uniform", len_lo=8, len_hi=64),
    1: ConfigSpec(1, "bf16-2layer-powerlaw", 2, 256, 4, 64, "bf16", batch=32,
                  len_kind="powerlaw", len_lo=16, len_hi=1024),
    2: ConfigSpec(2, "long-history-bf16-1layer", 1, 512, 4, 128, "bf16", batch=8,
                  len_kind="uniform", len_lo=4096, len_hi=8192),
    3: ConfigSpec(3, "mfalcon-ranking-bf16", 1, 256, 2, 128, "bf16",
                  users=16, hist_len=2048, num_candidates=4096, microbatch=512),
    4: ConfigSpec(4, "train-8layer-bf16-sl", 8, 512, 8, 64, "bf16", batch=64,
                  len_kind="powerlaw", len_lo=64, len_hi=4096,
                  sl_len=1024, sl_prob=0.8, training=True),
}


@dataclass
class LayerParams:
    """One layer's parameters.  Linear weights use the (out, in) row-major layout."""
    w1: np.ndarray          # [4d, d]
    b1: np.ndarray          # [4d]
    ln1_g: np.ndarray       # [d]
    ln1_b: np.ndarray       # [d]
    ln2_g: np.ndarray       # [H*dv]
    ln2_b: np.ndarray       # [H*dv]
    w2: np.ndarray          # [d, H*dv]
    b2: np.ndarray          # [d]
    pos_bias: np.ndarray    # [128] (shared across heads) or [H, 128]
    time_bias: np.ndarray   # [128] or [H, 128]


@dataclass
class Workload:
    spec: ConfigSpec
    seq_offsets: np.ndarray             # int32 [B+1]
    timestamps: np.ndarray              # int64 [T]
    x: np.ndarray                       # float32 [T, d] (bf16 values for bf16 configs)
    layers: List[LayerParams]
    num_targets: Optional[np.ndarray] = None   # int32 [B]
    extras: Dict[str, np.ndarray] = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets).astype(np.int64)


# ----------------------------------------------------------------------------
# primitive draws
# ----------------------------------------------------------------------------

def _streams(seed: int, n: int = 6) -> List[np.random.Generator]:
    ss = np.random.SeedSequence(seed)
    return [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(n)]


def sample_lengths(rng: np.random.Generator, batch: int, kind: str, lo: int, hi: int,
                   exponent: float = 1.5) -> np.ndarray:
    """Sequence lengths: uniform integers on [lo, hi] or a truncated power law.

    The power law has density proportional to L^-exponent on [lo, hi]; it is
    sampled by inverting its continuous CDF, then floored and clamped.
    """
    if kind == "uniform":
        return rng.integers(lo, hi + 1, size=batch).astype(np.int64)
    if kind == "powerlaw":
        u = rng.random(batch)
        a = 1.0 - exponent
        lo_a, hi_a = lo ** a, hi ** a
        lens = (lo_a + u * (hi_a - lo_a)) ** (1.0 / a)
        return np.clip(np.floor(lens), lo, hi).astype(np.int64)
    raise ValueError(kind)


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    if off[-1] >= 2 ** 31:
        raise ValueError("total tokens exceed int32 offsets")
    return off.astype(np.int32)


def sample_timestamps(rng: np.random.Generator, lengths, gap_mean: float = GAP_MEAN_S) -> np.ndarray:
    """Per sequence: a start time plus the floored cumulative sum of Exp gaps.

    Timestamps are int64 seconds and non-decreasing within each sequence.
    """
    out = []
    for n in np.asarray(lengths, dtype=np.int64):
        start = TIME_BASE + int(rng.integers(0, 86_400 * 365))
        gaps = rng.exponential(gap_mean, size=int(n))
        out.append(start + np.floor(np.cumsum(gaps)).astype(np.int64))
    if not out:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate(out).astype(np.int64)


def xavier_uniform(rng: np.random.Generator, out_f: int, in_f: int) -> np.ndarray:
    a = np.sqrt(6.0 / (in_f + out_f))
    return rng.uniform(-a, a, size=(out_f, in_f))


def sample_layers(rng_w: np.random.Generator, rng_rab: np.random.Generator, spec: ConfigSpec,
                  random_affine: bool = False, per_head_rab: bool = False) -> List[LayerParams]:
    d, H, dh = spec.d_model, spec.num_heads, spec.head_dim
    hv = H * dh
    rnd = round_to_bf16 if spec.dtype == "bf16" else (lambda a: np.asarray(a, dtype=np.float32))
    layers = []
    for _ in range(spec.num_layers):
        w1 = rnd(xavier_uniform(rng_w, 4 * hv, d))
        w2 = rnd(xavier_uniform(rng_w, d, hv))
        if random_affine:
            b1 = rnd(rng_w.normal(0, 0.1, 4 * hv))
            b2 = rnd(rng_w.normal(0, 0.1, d))
            g1 = rnd(1.0 + rng_w.normal(0, 0.2, d))
            be1 = rnd(rng_w.normal(0, 0.2, d))
            g2 = rnd(1.0 + rng_w.normal(0, 0.2, hv))
            be2 = rnd(rng_w.normal(0, 0.2, hv))
        else:
            b1 = np.zeros(4 * hv, np.float32)
            b2 = np.zeros(d, np.float32)
            g1 = np.ones(d, np.float32)
            be1 = np.zeros(d, np.float32)
            g2 = np.ones(hv, np.float32)
            be2 = np.zeros(hv, np.float32)
        shape = (H, NUM_POS_BUCKETS) if per_head_rab else (NUM_POS_BUCKETS,)
        pos_bias = rng_rab.normal(0, RAB_STD, size=shape).astype(np.float32)
        time_bias = rng_rab.normal(0, RAB_STD, size=shape).astype(np.float32)
        layers.append(LayerParams(w1.astype(np.float32), b1.astype(np.float32),
                                  g1.astype(np.float32), be1.astype(np.float32),
                                  g2.astype(np.float32), be2.astype(np.float32),
                                  w2.astype(np.float32), b2.astype(np.float32),
                                  pos_bias, time_bias))
    return layers


def sample_x(rng: np.random.Generator, rows: int, d: int, dtype: str) -> np.ndarray:
    x = rng.standard_normal((rows, d))
    return round_to_bf16(x) if dtype == "bf16" else x.astype(np.float32)


# ----------------------------------------------------------------------------
# whole workloads
# ----------------------------------------------------------------------------

def make_workload(cid: int, *, seed: Optional[int] = None, scale: float = 1.0,
                  random_affine: bool = False, per_head_rab: bool = False,
                  batch: Optional[int] = None, lengths=None) -> Workload:
    """Build the seeded workload of configuration `cid`.

    `scale` < 1 shrinks sequence lengths (and, for M-FALCON, history and
    candidate counts) so that the oracle finishes quickly while the shapes keep
    the same structure; `batch` overrides the number of sequences/users and
    `lengths` fixes explicit sequence lengths.
    """
    spec = CONFIGS[cid]
    seed = SEED_BASE + cid if seed is None else seed
    r_len, r_ts, r_x, r_w, r_rab, r_ext = _streams(seed)

    if spec.users:  # M-FALCON ranking
        users = batch if batch is not None else spec.users
        n = max(1, int(round(spec.hist_len * scale)))
        m = max(1, int(round(spec.num_candidates * scale)))
        hist_lens = np.full(users, n, dtype=np.int64) if lengths is None else np.asarray(lengths, np.int64)
        hist_offsets = offsets_from_lengths(hist_lens)
        hist_ts = sample_timestamps(r_ts, hist_lens)
        hist_x = sample_x(r_x, int(hist_offsets[-1]), spec.d_model, spec.dtype)
        layers = sample_layers(r_w, r_rab, spec, random_affine, per_head_rab)
        cand_counts = np.full(users, m, dtype=np.int64)
        cand_offsets = offsets_from_lengths(cand_counts)
        cand_x = sample_x(r_ext, int(cand_offsets[-1]), spec.d_model, spec.dtype)
        last = np.array([hist_ts[hist_offsets[u + 1] - 1] if hist_lens[u] > 0 else TIME_BASE
                         for u in range(users)], dtype=np.int64)
        t_req = last + np.floor(r_ext.exponential(GAP_MEAN_S, size=users)).astype(np.int64)
        cand_ts = np.repeat(t_req, cand_counts).astype(np.int64)
        return Workload(spec, hist_offsets, hist_ts, hist_x, layers,
                        extras=dict(cand_offsets=cand_offsets, cand_x=cand_x, cand_ts=cand_ts,
                                    request_ts=t_req,
                                    microbatch=np.array(spec.microbatch if scale == 1.0
                                                        else max(1, int(round(spec.microbatch * scale))))))

    B = batch if batch is not None else spec.batch
    if lengths is not None:
        lens = np.asarray(lengths, dtype=np.int64)
    else:
        lens = sample_lengths(r_len, B, spec.len_kind, spec.len_lo, spec.len_hi)
        if scale != 1.0:
            lens = np.maximum(1, np.floor(lens * scale)).astype(np.int64)
    offsets = offsets_from_lengths(lens)
    ts = sample_timestamps(r_ts, lens)
    x = sample_x(r_x, int(offsets[-1]), spec.d_model, spec.dtype)
    layers = sample_layers(r_w, r_rab, spec, random_affine, per_head_rab)
    extras: Dict[str, np.ndarray] = {}
    if spec.training:
        T = int(offsets[-1])
        extras["sl_coin"] = r_ext.integers(0, 2 ** 32, size=len(lens), dtype=np.uint64).astype(np.uint32)
        extras["sl_keys"] = r_ext.integers(0, 2 ** 32, size=T, dtype=np.uint64).astype(np.uint32)
        extras["grad_out"] = sample_x(r_ext, T, spec.d_model, spec.dtype)
        sl_len = spec.sl_len if scale == 1.0 else max(1, int(spec.sl_len * scale))
        extras["sl_len"] = np.array(sl_len)
        extras["sl_prob_u32"] = np.array(min(2 ** 32 - 1, int(round(spec.sl_prob * 2 ** 32))), dtype=np.uint64)
    return Workload(spec, offsets, ts, x, layers, extras=extras)


def select_sequences(wl: "Workload", seqs) -> "Workload":
    """The sub-batch of `wl` made of the sequences `seqs` (in that order): their
    rows of X and timestamps, new offsets, the same weights.  Per-token extras
    (gradient seeds, SL keys) and per-sequence extras (SL coins) follow their
    sequences; scalars are kept."""
    seqs = [int(s) for s in seqs]
    offs = np.asarray(wl.seq_offsets, dtype=np.int64)
    rows = np.concatenate([np.arange(offs[s], offs[s + 1]) for s in seqs]) if seqs else np.zeros(0, np.int64)
    lens = np.array([offs[s + 1] - offs[s] for s in seqs], dtype=np.int64)
    T = int(offs[-1])
    extras = {}
    for k, v in wl.extras.items():
        v = np.asarray(v)
        if v.ndim >= 1 and v.shape[0] == T:
            extras[k] = v[rows]
        elif v.ndim >= 1 and v.shape[0] == len(offs) - 1:
            extras[k] = v[np.asarray(seqs, dtype=np.int64)]
        else:
            extras[k] = v
    return Workload(wl.spec, offsets_from_lengths(lens), wl.timestamps[rows], wl.x[rows], wl.layers, extras=extras)


def interleave_item_action(wl: "Workload", seed: int = 7, delay_mean: float = 60.0) -> "Workload":
    """Ranking input with every item followed by the user's reaction to it (the
    ranking setting of the pages: the input alternates objects and the reactions
    that followed them).  Token k of each sequence of `wl` becomes the item at
    position 2k; its reaction, at 2k + 1, gets an N(0,1) embedding (rounded like
    the item embeddings) and the item's timestamp plus a floored Exp(delay_mean)
    delay.  Layers and weights are wl's."""
    rng = np.random.default_rng(seed)
    lens = wl.lengths
    d = wl.x.shape[1]
    offs2 = offsets_from_lengths(2 * lens)
    T2 = int(offs2[-1])
    x = np.empty((T2, d), dtype=np.float32)
    ts = np.empty(T2, dtype=np.int64)
    x[0::2] = wl.x
    x[1::2] = sample_x(rng, wl.total_tokens, d, wl.spec.dtype)
    ts[0::2] = wl.timestamps
    ts[1::2] = wl.timestamps + np.floor(rng.exponential(delay_mean, size=wl.total_tokens)).astype(np.int64)
    return Workload(wl.spec, offs2.astype(np.int32), ts, x, wl.layers)


def random_attention_inputs(seed: int, lengths, num_heads: int, head_dim: int, dtype: str,
                            num_targets=None, per_head_rab: bool = False, qk_std: float = 0.25,
                            gap_mean: float = GAP_MEAN_S):
    """Q, K, V, timestamps and rab tables for exercising attention alone.

    Q, K, V are drawn N(0, qk_std^2) (bf16-rounded when dtype is bf16) in the
    token-major [T, H, dh] layout.
    """
    r_len, r_ts, r_x, r_w, r_rab, r_ext = _streams(seed)
    lens = np.asarray(lengths, dtype=np.int64)
    offsets = offsets_from_lengths(lens)
    T = int(offsets[-1])
    ts = sample_timestamps(r_ts, lens, gap_mean)
    rnd = round_to_bf16 if dtype == "bf16" else (lambda a: np.asarray(a, dtype=np.float32))
    q = rnd(r_x.normal(0, qk_std, (T, num_heads, head_dim)))
    k = rnd(r_x.normal(0, qk_std, (T, num_heads, head_dim)))
    v = rnd(r_x.normal(0, 1.0, (T, num_heads, head_dim)))
    shape = (num_heads, NUM_POS_BUCKETS) if per_head_rab else (NUM_POS_BUCKETS,)
    pos_bias = r_rab.normal(0, RAB_STD * 10, size=shape).astype(np.float32)
    time_bias = r_rab.normal(0, RAB_STD * 10, size=shape).astype(np.float32)
    nt = None if num_targets is None else np.asarray(num_targets, dtype=np.int32)
    return dict(seq_offsets=offsets, timestamps=ts, q=q, k=k, v=v, pos_bias=pos_bias,
                time_bias=time_bias, num_targets=nt, dout=rnd(r_ext.normal(0, 1.0, (T, num_heads, head_dim))))
