#!/usr/bin/env python
"""Throughput of the HSTU layer hot path on B200.

A step is one forward pass of the long-history HSTU layer (B=8 sequences,
n ~ U{4096..8192}, d_model=512, 4 heads of 128, bf16) through the C-ABI call
hstu_layer_fwd: jagged schedule, LayerNorm, f1 + SiLU + split, pointwise
attention with the rab bias, LayerNorm(A V) * U, f2 + residual.

Prints one JSON line (rank 0).  `value` is tokens/s over all ranks with the
inputs resident in HBM; `e2e` repeats the measurement through the same call
with host (pinned) inputs copied in and the output copied out every step;
`roofline` reports the attention kernel's causal-FLOP rate against the measured
dense bf16 peak; `cpu_baseline` times the fp64 CPU oracle on a bounded sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch with torch.distributed.run; one batch of 8 N sequences is dealt
out over the ranks by sequence (longest-processing-time first on the attended
pairs and per-token work; no collective on the data path, weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hstu_sequential_transducer_02_b200 import workload as W  # noqa: E402

CONFIG_ID = 2
METRIC = "HSTU layer tokens/s and attention TFLOP/s as % of B200 BF16 dense peak (1 GPU)"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
E2E_CHUNKS = 4       # sequence chunks of the host-memory forward (copies overlap the computation)
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--oracle-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the M-FALCON and training-step measurements")
    ap.add_argument("--profile-attn-bwd", action="store_true",
                    help="for profilers: run the training workload's attention backward (1 + 3 launches) and exit")
    ap.add_argument("--profile-mfalcon", action="store_true",
                    help="for profilers: the M-FALCON ranking workload through mfalcon_rank (5 calls of 8 "
                         "microbatches, 8 attention launches each) and exit")
    ap.add_argument("--profile-training", action="store_true",
                    help="for profilers: the 8-layer training step (1 + 1 timed + 1 traced steps) and exit")
    ap.add_argument("--profile-short", action="store_true",
                    help="for profilers: run the fused short-sequence layer on 512 sequences of at most 128 "
                         "tokens (two layers, 3 + 2 forwards) and exit")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count() or 1
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------
# fp64 oracle on the host cores (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------

def oracle_sequence_time(wl, s: int, max_tokens=None):
    import oracle.hstu_oracle as O
    sp = wl.spec
    a, b = int(wl.seq_offsets[s]), int(wl.seq_offsets[s + 1])
    if max_tokens is not None:
        b = min(b, a + max_tokens)
    t0 = time.perf_counter()
    O.layer_forward(wl.x[a:b], wl.layers[0], [0, b - a], wl.timestamps[a:b], sp.num_heads, sp.head_dim)
    return b - a, time.perf_counter() - t0


def cpu_baseline(wl, seconds: float):
    """Oracle layer forward over whole sequences of the workload, in order, until
    `seconds` of CPU work have been spent (at least one sequence)."""
    tokens, elapsed, seqs = 0, 0.0, 0
    for s in range(len(wl.seq_offsets) - 1):
        n, t = oracle_sequence_time(wl, s)
        tokens += n
        elapsed += t
        seqs += 1
        if elapsed >= seconds:
            break
    return {"value": tokens / elapsed, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle, 1 layer forward over the first {seqs} whole sequence(s) "
                      f"({tokens} tokens, {elapsed:.1f} s) of the long-history workload"}


def run_reference(args, rank: int):
    if rank != 0:
        return
    wl = W.make_workload(CONFIG_ID)
    B = len(wl.seq_offsets) - 1
    for w in range(args.warmup):
        oracle_sequence_time(wl, w % B, max_tokens=256)
    tokens, elapsed = 0, 0.0
    for k in range(args.steps):
        n, t = oracle_sequence_time(wl, k % B)
        tokens += n
        elapsed += t
    value = tokens / elapsed
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "long-history HSTU layer, B=8, n~U{4096..8192}, d=512, H=4, dh=128, 1 layer; "
                               "one whole sequence per step (sequence k mod 8)",
                   "global_batch": 1, "seq_len": "4096-8192", "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps, one whole sequence each ({tokens} tokens)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# multi-rank plumbing (host logic; covered on CPU with gloo ranks)
# ----------------------------------------------------------------------------

def projection_pairs_per_token(spec) -> float:
    """The row-wise work of a token (f1: 2 d 4d FLOP, f2: 2 d d FLOP) in units of
    one attended pair (2 (dqk + dv) H FLOP): the per-token weight of the cost
    that deals sequences out to ranks."""
    d = spec.d_model
    return (2.0 * d * 4 * d + 2.0 * d * d) / (2.0 * 2 * spec.head_dim * spec.num_heads)


def rank_workload(rank: int, world: int = 1):
    """Rank `rank`'s shard of one global batch: the long-history recipe drawn
    for 8 * world sequences (with one rank, exactly the 8-sequence workload),
    dealt out over the ranks by hstu_lpt_partition (attended pairs plus the
    projections' per-token work, longest first to the least-loaded rank), so
    that per-rank work stays about fixed as ranks are added.  Every rank draws
    the same batch and computes the same assignment: nothing is exchanged."""
    spec = W.CONFIGS[CONFIG_ID]
    wl = W.make_workload(CONFIG_ID, batch=spec.batch * world)
    if world == 1:
        return wl
    from hstu_sequential_transducer_02_b200 import binding as hb
    rank_of, _ = hb.lpt_partition(wl.seq_offsets, world, token_weight=projection_pairs_per_token(spec))
    return W.select_sequences(wl, np.nonzero(rank_of == rank)[0])


def reduce_over_ranks(local_ms: float, local_tokens: int, world: int, device=None):
    """(max over ranks of the timed milliseconds, sum over ranks of the tokens).
    Every rank calls it at the same point with the same collective sequence."""
    if world == 1:
        return float(local_ms), int(local_tokens)
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    n = torch.tensor([local_tokens], dtype=torch.int64, device=device)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), int(n.item())


def unmasked_pairs(seq_offsets, num_targets=None) -> int:
    """Attended (i, j) pairs of a jagged batch: N(N+1)/2 causal pairs of the N
    history tokens plus (N+1) per candidate (history and itself)."""
    offs = np.asarray(seq_offsets, dtype=np.int64)
    n = np.diff(offs)
    nt = np.zeros_like(n) if num_targets is None else np.asarray(num_targets, np.int64)
    N = n - nt
    return int(np.sum(N * (N + 1) // 2 + nt * (N + 1)))


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    """Samples the SM clock and the clock-event reasons of one GPU every few
    milliseconds from a host thread (NVML reads only; nothing is changed)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.period = period_s
        self.rows = []
        self.thread = None
        self.stop_flag = False

    def _loop(self, nv, h):
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((sm, mx, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
        except Exception:
            return
        self.thread = threading.Thread(target=self._loop, args=(nv, h), daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.rows and time.time() - t0 < 2.0:  # first sample before the timed region
            time.sleep(0.001)
        self.rows = []

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=2)
        rows = self.rows
        if not rows:
            return None
        reasons = sorted({n for _, _, rs in rows for n, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "source": "NVML, 5 ms period, timed region only"}


KERNEL_SOURCES = {"attn_fwd_tc": ("attn_tc.cu", "sm100.cuh", "common.cuh", "kernels.cuh")}


def kernel_digest(kernel: str):
    """sha256 (first 16 hex digits) of the sources that make up `kernel`."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES.get(kernel, ()):
        with open(os.path.join(ROOT, "hstu_sequential_transducer_02_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic(kernel: str, path: str = None):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (`profiles/dram_traffic.txt`: kernel, bytes, source digest), or None when
    there is none or the kernel's sources changed after the capture."""
    p = path or os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == kernel and not line.startswith("#"):
                if parts[2] != kernel_digest(kernel):
                    return None
                try:
                    return float(parts[1])
                except ValueError:
                    return None
    return None


# ----------------------------------------------------------------------------
# further rows of the path, measured on their own workloads (1 GPU)
# ----------------------------------------------------------------------------

def mfalcon_pairs(hist_lens, cand_counts) -> int:
    """Attended pairs of one mfalcon_rank call with the history's keys and values
    cached across microbatches: each user's history causally once, then every
    candidate against its user's history and itself (the same pairs as one
    M-FALCON pass over [history ; all candidates])."""
    n = np.asarray(hist_lens, dtype=np.int64)
    m = np.asarray(cand_counts, dtype=np.int64)
    return int(np.sum(n * (n + 1) // 2 + m * (n + 1)))


def _trace_attention(trace, name, flops):
    a = trace.get(name)
    if not a or not a["count"]:
        return None
    ms = a["ms"] / a["count"]
    return {"kernel": name, "launches": a["count"], "ms_per_launch": ms,
            "tflops": flops / a["count"] / (ms / 1e3) / 1e12 if flops else None}  # flops: all traced launches


def _traced(hb, fn, steps):
    """Per-kernel device times of `steps` calls of fn, with the library's event
    tracing on (a pass of its own, outside any timed region)."""
    import torch
    torch.cuda.synchronize()
    hb.trace_enable(True)
    for _ in range(steps):
        fn()
    torch.cuda.synchronize()
    trace = hb.trace_read()
    hb.trace_enable(False)
    return trace


def _top_kernels(trace, steps, k=6):
    """The k kernels with the most traced device time: share and ms per step."""
    tot = sum(v["ms"] for v in trace.values()) or 1e-9
    top = sorted(trace.items(), key=lambda kv: -kv[1]["ms"])[:k]
    return {name: {"share": v["ms"] / tot, "ms_per_step": v["ms"] / steps, "launches_per_step": v["count"] / steps}
            for name, v in top}


def measure_mfalcon(hb, steps: int):
    """M-FALCON ranking (16 users, n = 2048 history, m = 4096 candidates in
    microbatches of b_m = 512, d_model = 256, 2 heads of 128, 1 layer):
    candidates scored per second through mfalcon_rank."""
    import torch
    wl = W.make_workload(3)
    sp, e = wl.spec, wl.extras
    td = torch.bfloat16
    layer = hb.Layer(hb.layer_weights_to_device(wl.layers[0], td), sp.d_model, sp.num_heads, sp.head_dim)
    bm = int(e["microbatch"])
    m_max = int(np.max(np.diff(e["cand_offsets"])))
    args = (torch.from_numpy(wl.seq_offsets).cuda(), torch.from_numpy(wl.x).to(td).cuda(),
            torch.from_numpy(wl.timestamps).cuda(), torch.from_numpy(e["cand_offsets"]).cuda(),
            torch.from_numpy(e["cand_x"]).to(td).cuda(), torch.from_numpy(e["cand_ts"]).cuda())
    out = hb.mfalcon_rank([layer], *args, bm, m_max)
    for _ in range(2):
        hb.mfalcon_rank([layer], *args, bm, m_max, out=out)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        hb.mfalcon_rank([layer], *args, bm, m_max, out=out)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    # per-kernel device times from a separate traced pass (events around every launch
    # would otherwise be inside the timed calls)
    trace = _traced(hb, lambda: hb.mfalcon_rank([layer], *args, bm, m_max, out=out), steps)
    U = len(wl.seq_offsets) - 1
    n = int(np.diff(wl.seq_offsets)[0])
    cands = int(e["cand_offsets"][-1])
    mbs = (m_max + bm - 1) // bm
    pairs = mfalcon_pairs(np.diff(wl.seq_offsets), np.diff(e["cand_offsets"]))
    flops = pairs * 2 * 2 * sp.head_dim * sp.num_heads
    return {"workload": f"M-FALCON: {U} users, n={n} history, m={cands // U} candidates, b_m={bm} "
                        f"({mbs} microbatches, history K/V cached across them), "
                        f"d_model={sp.d_model}, {sp.num_heads} heads x {sp.head_dim}, 1 layer",
            "candidates_per_s": cands / (ms / 1e3), "ms_per_call": ms, "calls": steps,
            "attention": _trace_attention(trace, "attn_fwd_tc", flops * steps),
            "top_kernels": _top_kernels(trace, steps)}


def _two_layer_ms(hb, wl, steps: int, short: bool) -> float:
    """Device milliseconds of the workload's two-layer forward through
    hstu_layer_fwd (short: with HSTU_FLAG_SHORT_SEQUENCES, one fused kernel per layer)."""
    import torch
    sp = wl.spec
    td = torch.bfloat16
    layers = [hb.Layer(hb.layer_weights_to_device(p_, td), sp.d_model, sp.num_heads, sp.head_dim,
                       short_sequences=short) for p_ in wl.layers]
    x = torch.from_numpy(wl.x).to(td).cuda()
    offs = torch.from_numpy(wl.seq_offsets).cuda()
    ts = torch.from_numpy(wl.timestamps).cuda()
    ys = [torch.empty_like(x) for _ in layers]

    def fwd():
        h = x
        for ly, y in zip(layers, ys):
            h = ly.forward(h, offs, ts, out=y)

    for _ in range(3):
        fwd()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        fwd()
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def measure_short_sequences(hb, steps: int):
    """The short-sequence workload (power-law lengths, d_model = 256, 4 heads of
    64, 2 layers, bf16): tokens per second of the two-layer forward.  The recipe as
    specified (32 sequences, lengths in [16, 1024]) runs through the multi-kernel
    layer; with its lengths cut to [2, 128] (x 1/8) the layer can run as one fused
    kernel per layer, measured next to the multi-kernel layer on 32 and 512
    sequences."""
    wl = W.make_workload(1)
    T = int(wl.seq_offsets[-1])
    ms = _two_layer_ms(hb, wl, steps, False)
    out = {"workload": f"short sequences: B=32, power-law n in [16,1024] (T={T} tokens, longest "
                       f"{int(np.max(np.diff(wl.seq_offsets)))}), d_model=256, 4 heads x 64, 2 layers, causal",
           "tokens_per_s": T / (ms / 1e3), "ms_per_forward": ms, "steps": steps, "lengths_at_most_128": {}}
    for B in (32, 512):
        w2 = W.make_workload(1, scale=1 / 8, batch=B)
        T2 = int(w2.seq_offsets[-1])
        f_ms = _two_layer_ms(hb, w2, steps, True)
        l_ms = _two_layer_ms(hb, w2, steps, False)
        out["lengths_at_most_128"][f"B={B}"] = {
            "tokens": T2, "fused_tokens_per_s": T2 / (f_ms / 1e3), "fused_ms": f_ms,
            "layer_path_tokens_per_s": T2 / (l_ms / 1e3), "layer_path_ms": l_ms}
    return out


def measure_training(hb, steps: int):
    """Training step of the 8-layer stack (64 sequences, power-law lengths in
    [64, 4096] cut by Stochastic Length to 1024 with p = 0.8, d_model = 512, 8
    heads of 64, fp32 residual stream): SL, forward with saved activations,
    backward from dY = G; tokens (after SL) per second."""
    import torch
    from hstu_sequential_transducer_02_b200.training import StackTrainer
    wl = W.make_workload(4)
    sp, e = wl.spec, wl.extras
    td, io = torch.bfloat16, torch.float32
    pool = {}   # one workspace per entry point for the whole stack: the preparation is shared
    layers = [hb.Layer(hb.layer_weights_to_device(p_, td), sp.d_model, sp.num_heads, sp.head_dim,
                       residual_fp32=True, workspaces=pool) for p_ in wl.layers]
    offs_in = torch.from_numpy(wl.seq_offsets).cuda()
    coins = torch.from_numpy(e["sl_coin"].view(np.int32)).cuda()
    keys = torch.from_numpy(e["sl_keys"].view(np.int32)).cuda()
    x_all = torch.from_numpy(wl.x).to(io).cuda()
    ts_all = torch.from_numpy(wl.timestamps).cuda()
    g_all = torch.from_numpy(e["grad_out"]).to(io).cuda()
    hv = sp.num_heads * sp.head_dim
    T_cap = wl.total_tokens
    x = torch.empty(T_cap, sp.d_model, dtype=io, device="cuda")
    ts = torch.empty(T_cap, dtype=torch.int64, device="cuda")
    gy = torch.empty_like(x)
    saved = [hb.Saved.alloc(T_cap, sp.d_model, hv, td, "cuda") for _ in layers]
    acts = [torch.empty_like(x) for _ in layers]

    trainer = StackTrainer(layers, share_prep=True)   # one rank: the gradient reduction is a no-op

    def step():
        offs, idx = hb.stochastic_length(offs_in, coins, keys, int(e["sl_len"]), int(e["sl_prob_u32"]))
        cnt = offs[-1:]
        hb.gather_rows(x_all, idx, cnt, x)
        hb.gather_rows(ts_all, idx, cnt, ts)
        hb.gather_rows(g_all, idx, cnt, gy)
        trainer.step(x, offs, ts, gy, saved, acts)
        return offs

    offs = step()
    torch.cuda.synchronize()
    T2 = int(offs[-1].item())
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    trace = _traced(hb, step, steps)   # per-kernel device times, from a separate pass
    return {"workload": f"training step: 8 layers, B=64, power-law n in [64,4096], SL to 1024 (p=0.8) -> "
                        f"T={T2} tokens, d_model={sp.d_model}, {sp.num_heads} heads x {sp.head_dim}, "
                        "fp32 residual stream, forward + backward",
            "tokens_per_s": T2 / (ms / 1e3), "ms_per_step": ms, "steps": steps,
            "top_kernels": _top_kernels(trace, steps)}

# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def profile_attn_bwd():
    """The attention backward alone on the training workload's shapes (the
    sequence lengths Stochastic Length leaves, 8 heads of 64, bf16): one launch,
    then three timed ones; prints their mean time.  A target for profilers."""
    import torch
    from hstu_sequential_transducer_02_b200 import binding as hb
    wl = W.make_workload(4)
    e = wl.extras
    offs, _ = hb.stochastic_length(torch.from_numpy(wl.seq_offsets).cuda(),
                                   torch.from_numpy(e["sl_coin"].view(np.int32)).cuda(),
                                   torch.from_numpy(e["sl_keys"].view(np.int32)).cuda(), int(e["sl_len"]),
                                   int(e["sl_prob_u32"]))
    lens = np.diff(offs.cpu().numpy())
    H, dh = wl.spec.num_heads, wl.spec.head_dim
    d = W.random_attention_inputs(3, lens, H, dh, "bf16", qk_std=0.5)
    T = int(sum(lens))
    q, k, v, do = (torch.from_numpy(d[n].reshape(T, H * dh)).to(torch.bfloat16).cuda() for n in ("q", "k", "v", "dout"))
    args = (torch.from_numpy(d["seq_offsets"]).cuda(), torch.from_numpy(d["timestamps"]).cuda(),
            torch.from_numpy(d["pos_bias"]).cuda(), torch.from_numpy(d["time_bias"]).cuda(), H)
    hb.attn_bwd(q, k, v, do, *args)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        hb.attn_bwd(q, k, v, do, *args)
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"attn_bwd_ms": e0.elapsed_time(e1) / 3, "tokens": T, "heads": H, "head_dim": dh}))


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.profile_attn_bwd:
        profile_attn_bwd()
        return
    if args.profile_mfalcon:
        from hstu_sequential_transducer_02_b200 import binding as hb
        r = measure_mfalcon(hb, 1)
        print(json.dumps({"ms_per_call": r["ms_per_call"], "attention": r["attention"]}))
        return
    if args.profile_training:
        from hstu_sequential_transducer_02_b200 import binding as hb
        r = measure_training(hb, 1)
        print(json.dumps({"ms_per_step": r["ms_per_step"], "tokens_per_s": r["tokens_per_s"]}))
        return
    if args.profile_short:
        from hstu_sequential_transducer_02_b200 import binding as hb
        wl = W.make_workload(1, scale=1 / 8, batch=512)
        print(json.dumps({"fused_two_layer_ms": _two_layer_ms(hb, wl, 2, True), "tokens": int(wl.seq_offsets[-1])}))
        return
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from hstu_sequential_transducer_02_b200 import binding as hb

    wl = rank_workload(rank, world)
    sp = wl.spec
    td = torch.bfloat16
    T = wl.total_tokens
    layer = hb.Layer(hb.layer_weights_to_device(wl.layers[0], td), sp.d_model, sp.num_heads, sp.head_dim)
    x = torch.from_numpy(wl.x).to(td).cuda()
    offs = torch.from_numpy(wl.seq_offsets).cuda()
    ts = torch.from_numpy(wl.timestamps).cuda()
    y = torch.empty_like(x)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    clean = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")

    def flush_l2():
        """Evict L2 between timed steps, outside the timed events: a 256 MiB
        write, then a 256 MiB read of another buffer, which writes the write's
        dirty lines back, so that a step neither hits in L2 nor pays for the
        flush's own write-back."""
        flush.zero_()
        clean.sum()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        layer.forward(x, offs, ts, out=y)
    torch.cuda.synchronize()
    barrier()

    def timed_pass(traced):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        hb.trace_enable(traced)
        torch.cuda.synchronize()
        barrier()
        for k in range(args.steps):
            flush_l2()
            starts[k].record()
            layer.forward(x, offs, ts, out=y)
            ends[k].record()
        torch.cuda.synchronize()
        barrier()
        trace = hb.trace_read() if traced else None
        hb.trace_enable(False)
        return [s.elapsed_time(e) for s, e in zip(starts, ends)], trace

    # the step time comes from a pass without the library's per-kernel events
    # (they cost ~4 % of a step); a second pass of the same steps records them
    clocks = ClockSampler(local_rank)
    clocks.start()
    step_ms, _ = timed_pass(False)
    _, trace = timed_pass(True)
    clk = clocks.stop()
    total_ms, T_all = reduce_over_ranks(sum(step_ms), T, world, "cuda")
    ms_per_step = total_ms / args.steps
    value = T_all / (ms_per_step / 1e3)

    # end to end through the host-memory entry point (hstu_layer_fwd_host): every
    # step copies the inputs in from page-locked host memory and Y out, in chunks
    # of sequences whose copies overlap the computation
    x_h = torch.from_numpy(wl.x).to(td).pin_memory()
    offs_h = torch.from_numpy(wl.seq_offsets.astype(np.int32))
    ts_h = torch.from_numpy(wl.timestamps).pin_memory()
    y_h = torch.empty(x_h.shape, dtype=td).pin_memory()
    n_chunks = min(E2E_CHUNKS, len(wl.seq_offsets) - 1)
    layer.forward_host(x_h, offs_h, ts_h, n_chunks, out=y_h)   # workspace and copy streams, outside the timing
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    barrier()
    for k in range(args.steps):
        flush_l2()
        e_s[k].record()
        layer.forward_host(x_h, offs_h, ts_h, n_chunks, out=y_h)
        e_e[k].record()
    torch.cuda.synchronize()
    barrier()
    e2e_ms, _ = reduce_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e_s, e_e)), T, world, "cuda")
    e2e_value = T_all / (e2e_ms / args.steps / 1e3)
    h2d = x_h.numel() * x_h.element_size() + offs_h.numel() * 4 + ts_h.numel() * 8
    d2h = y_h.numel() * y_h.element_size()

    # roofline of the attention kernel
    pairs = unmasked_pairs(wl.seq_offsets)
    attn_flops = pairs * 2 * (sp.head_dim + sp.head_dim) * sp.num_heads
    peaks, peak_src = load_peaks()
    attn_name = "attn_fwd_tc" if "attn_fwd_tc" in trace else "attn_fwd_simt"
    attn = trace.get(attn_name, {"count": 0, "ms": float("nan")})
    attn_ms = attn["ms"] / max(attn["count"], 1)
    achieved = attn_flops / (attn_ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    launches = int(sum(v["count"] for v in trace.values()))
    traffic = read_traffic(attn_name)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"long-history HSTU layer forward: B={8 * world} jagged sequences, "
                                   f"n~U{{4096..8192}} (T={T_all} tokens), d_model=512, 4 heads x 128, 1 layer, "
                                   "causal, seed 20242" + (f", dealt out over {world} GPUs by LPT" if world > 1 else ""),
                       "global_batch": 8 * world, "seq_len": "4096-8192", "parallelism": f"dp{world}",
                       "l2": "flushed between timed steps (256 MiB write, then a 256 MiB read that writes its "
                             "dirty lines back; both outside the timed events)",
                       "kernel_times": "per-kernel CUDA events on the launching streams in a second pass of the "
                                       "same steps; ms_per_step from the pass without them"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": attn_name, "peak_source": f"{peak_src} bf16 dense (burst)",
                         "flops_per_launch": attn_flops, "ms_per_launch": attn_ms,
                         "frac_of_datasheet_2250": achieved / DATASHEET_BF16_TFLOPS},
            "attention_tflops": achieved,
            "kernels": {k: {"launches": v["count"], "ms_per_launch": v["ms"] / max(v["count"], 1),
                            "share": v["ms"] / max(sum(u["ms"] for u in trace.values()), 1e-9)}
                        for k, v in trace.items()},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clk,
        }
        if world == 1 and not args.no_extra:
            line["mfalcon"] = measure_mfalcon(hb, 5)
            line["training"] = measure_training(hb, 3)
            line["short_sequences"] = measure_short_sequences(hb, 50)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.oracle_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
