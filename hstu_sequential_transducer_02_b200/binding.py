"""Python binding of libhstu (ctypes).  Argument marshalling only: every step
of the computation runs in the library's CUDA kernels.  PyTorch provides the
device memory (tensors, workspaces) and the current CUDA stream.

Importing this module loads libhstu.so from the package directory and raises
if it is missing; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhstu.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libhstu.so is not built ({LIB_PATH}); run python -m hstu_sequential_transducer_02_b200.build")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_BAD_OFFSETS = range(7)
DTYPE_F32, DTYPE_BF16 = 0, 1
FLAG_FORCE_SIMT = 1
FLAG_SHORT_SEQUENCES = 2
FLAG_REUSE_PREP = 4
NUM_BUCKETS = 128

_c_int = ctypes.c_int
_c_i32 = ctypes.c_int32
_c_i64 = ctypes.c_int64
_c_u32 = ctypes.c_uint32
_c_size = ctypes.c_size_t
_c_vp = ctypes.c_void_p
_c_dbl = ctypes.c_double
_c_flt = ctypes.c_float


class AttnDesc(ctypes.Structure):
    _fields_ = [("num_heads", _c_i32), ("dqk", _c_i32), ("dv", _c_i32), ("dtype", _c_i32),
                ("rab_head_stride", _c_i32), ("num_pos_buckets", _c_i32), ("num_time_buckets", _c_i32),
                ("flags", _c_i32), ("time_div", _c_dbl)]


class LayerDesc(ctypes.Structure):
    _fields_ = [("d_model", _c_i32), ("ln_eps", _c_flt), ("io_dtype", _c_i32), ("reserved", _c_i32),
                ("attn", AttnDesc)]


class Jagged(ctypes.Structure):
    _fields_ = [("batch", _c_i32), ("total_tokens", _c_i32), ("seq_offsets", _c_vp), ("num_targets", _c_vp),
                ("timestamps", _c_vp)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, _c_vp) for n in ("w1", "b1", "ln1_gamma", "ln1_beta", "ln2_gamma", "ln2_beta", "w2", "b2",
                                     "pos_bias", "time_bias")]


class LayerSaved(ctypes.Structure):
    _fields_ = [(n, _c_vp) for n in ("xhat", "ln1_mean", "ln1_rstd", "z", "uvqk", "attn_out", "ln2_mean",
                                     "ln2_rstd", "gate")]


class LayerGrads(ctypes.Structure):
    _fields_ = [(n, _c_vp) for n in ("dw1", "db1", "dln1_gamma", "dln1_beta", "dln2_gamma", "dln2_beta", "dw2",
                                     "db2", "dpos_bias", "dtime_bias", "duvqk")]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_P = ctypes.POINTER
_lib_status_string = _sig("hstu_status_string", ctypes.c_char_p, [_c_int])
_lib_version = _sig("hstu_version", _c_int, [])
_lib_thresholds = _sig("hstu_build_time_thresholds", _c_int, [_c_dbl, _c_i32, _P(_c_i64)])
_lib_ws_status = _sig("hstu_workspace_status", _c_int, [_c_vp, _P(_c_i32), _c_vp])
_lib_attn_fwd_ws = _sig("hstu_attn_fwd_workspace_size", _c_int, [_P(AttnDesc), _c_i32, _c_i32, _P(_c_size)])
_lib_attn_fwd = _sig("hstu_attn_fwd", _c_int,
                     [_P(AttnDesc), _P(Jagged), _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_vp, _c_vp,
                      _c_i64, _c_vp, _c_size, _c_vp])
_lib_attn_bwd_ws = _sig("hstu_attn_bwd_workspace_size", _c_int, [_P(AttnDesc), _c_i32, _c_i32, _P(_c_size)])
_lib_attn_bwd = _sig("hstu_attn_bwd", _c_int,
                     [_P(AttnDesc), _P(Jagged), _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_vp, _c_vp,
                      _c_i64, _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_vp, _c_vp, _c_size, _c_vp])
_lib_layer_fwd_ws = _sig("hstu_layer_fwd_workspace_size", _c_int, [_P(LayerDesc), _c_i32, _c_i32, _P(_c_size)])
_lib_layer_fwd = _sig("hstu_layer_fwd", _c_int,
                      [_P(LayerDesc), _P(LayerWeights), _P(Jagged), _c_vp, _c_vp, _P(LayerSaved), _c_vp, _c_size,
                       _c_vp])
_lib_layer_fwd_host_ws = _sig("hstu_layer_fwd_host_workspace_size", _c_int,
                              [_P(LayerDesc), _c_i32, _c_i32, _c_i32, _P(_c_size)])
_lib_layer_fwd_host = _sig("hstu_layer_fwd_host", _c_int,
                           [_P(LayerDesc), _P(LayerWeights), _c_i32, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i32,
                            _c_vp, _c_size, _c_vp])
_lib_layer_bwd_ws = _sig("hstu_layer_bwd_workspace_size", _c_int, [_P(LayerDesc), _c_i32, _c_i32, _P(_c_size)])
_lib_layer_bwd = _sig("hstu_layer_bwd", _c_int,
                      [_P(LayerDesc), _P(LayerWeights), _P(Jagged), _c_vp, _P(LayerSaved), _c_vp, _c_vp,
                       _P(LayerGrads), _c_vp, _c_size, _c_vp])
_lib_mf_ws = _sig("mfalcon_rank_workspace_size", _c_int, [_P(LayerDesc), _c_i32, _c_i32, _c_i32, _c_i32, _P(_c_size)])
_lib_mf = _sig("mfalcon_rank", _c_int,
               [_P(LayerDesc), _P(LayerWeights), _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_vp, _c_vp, _c_vp, _c_vp,
                _c_vp, _c_vp, _c_vp, _c_vp, _c_size, _c_vp])
_lib_sl_ws = _sig("hstu_stochastic_length_workspace_size", _c_int, [_c_i32, _c_i32, _P(_c_size)])
_lib_sl = _sig("hstu_stochastic_length", _c_int,
               [_c_i32, _c_i32, _c_vp, _c_vp, _c_vp, _c_i32, _c_u32, _c_vp, _c_vp, _c_vp, _c_size, _c_vp])
_lib_gather = _sig("hstu_gather_rows", _c_int, [_c_vp, _c_vp, _c_i64, _c_vp, _c_vp, _c_i32, _c_vp])
_lib_dbg_buckets = _sig("hstu_debug_rab_buckets", _c_int, [_P(AttnDesc), _P(Jagged), _c_vp, _c_i32, _c_vp, _c_vp])
_lib_dbg_timeout = _sig("hstu_debug_timeout_probe", _c_int, [_c_i64, _c_vp, _c_vp])

EXPORTED = ["hstu_status_string", "hstu_version", "hstu_build_time_thresholds", "hstu_workspace_status",
            "hstu_attn_fwd_workspace_size", "hstu_attn_fwd", "hstu_attn_bwd_workspace_size", "hstu_attn_bwd",
            "hstu_layer_fwd_workspace_size", "hstu_layer_fwd", "hstu_layer_fwd_host_workspace_size",
            "hstu_layer_fwd_host", "hstu_layer_bwd_workspace_size", "hstu_layer_bwd",
            "mfalcon_rank_workspace_size", "mfalcon_rank", "hstu_stochastic_length_workspace_size",
            "hstu_stochastic_length", "hstu_gather_rows", "hstu_debug_rab_buckets", "hstu_debug_timeout_probe"]


_lib_last_cuda_error = _sig("hstu_last_cuda_error", ctypes.c_char_p, [])
EXPORTED.append("hstu_last_cuda_error")


class HstuError(RuntimeError):
    def __init__(self, code: int, where: str):
        detail = f" [{_lib_last_cuda_error().decode()}]" if code == ERR_CUDA else ""
        super().__init__(f"{where}: {status_string(code)} ({code}){detail}")
        self.code = code


def status_string(code: int) -> str:
    return _lib_status_string(code).decode()


def version() -> int:
    return _lib_version()


def _check(code: int, where: str):
    if code != OK:
        raise HstuError(code, where)


def build_time_thresholds(time_div: float = 0.301, num_buckets: int = NUM_BUCKETS) -> List[int]:
    out = (_c_i64 * num_buckets)()
    _check(_lib_thresholds(time_div, num_buckets, out), "hstu_build_time_thresholds")
    return list(out)


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def attn_desc(num_heads: int, head_dim: int, dtype: int, per_head_rab: bool = False, force_simt: bool = False,
              time_div: float = 0.301) -> AttnDesc:
    return AttnDesc(num_heads, head_dim, head_dim, dtype, NUM_BUCKETS if per_head_rab else 0, NUM_BUCKETS,
                    NUM_BUCKETS, FLAG_FORCE_SIMT if force_simt else 0, time_div)


def layer_desc(d_model: int, num_heads: int, head_dim: int, dtype: int, per_head_rab: bool = False,
               force_simt: bool = False, eps: float = 1e-5, time_div: float = 0.301,
               io_dtype: Optional[int] = None) -> LayerDesc:
    return LayerDesc(d_model, eps, dtype if io_dtype is None else io_dtype, 0,
                     attn_desc(num_heads, head_dim, dtype, per_head_rab, force_simt, time_div))


def jagged(seq_offsets: torch.Tensor, timestamps: torch.Tensor, total_tokens: int,
           num_targets: Optional[torch.Tensor] = None) -> Jagged:
    assert seq_offsets.dtype == torch.int32 and timestamps.dtype == torch.int64
    assert num_targets is None or num_targets.dtype == torch.int32
    return Jagged(seq_offsets.numel() - 1, total_tokens, _ptr(seq_offsets), _ptr(num_targets), _ptr(timestamps))


def _row_stride(t: torch.Tensor) -> int:
    assert t.stride(-1) == 1
    return t.stride(0)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def attn_fwd(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, num_heads: int, num_targets=None,
             force_simt: bool = False, time_div: float = 0.301, out=None, workspace=None, stream=None,
             return_workspace: bool = False):
    """q, k, v: [T, H*dh] (or [T, H, dh]) views with unit inner stride."""
    T = q.shape[0]
    dh = (q.shape[1] * (q.shape[2] if q.dim() == 3 else 1)) // num_heads
    dt = _dtype_code(q)
    d = attn_desc(num_heads, dh, dt, pos_bias.dim() == 2, force_simt, time_div)
    jb = jagged(seq_offsets, timestamps, T, num_targets)
    nbytes = _c_size()
    _check(_lib_attn_fwd_ws(ctypes.byref(d), jb.batch, T, ctypes.byref(nbytes)), "hstu_attn_fwd_workspace_size")
    ws = workspace if workspace is not None else _workspace(nbytes.value, q.device)
    if out is None:
        out = torch.empty(T, num_heads * dh, dtype=q.dtype, device=q.device)
    _check(_lib_attn_fwd(ctypes.byref(d), ctypes.byref(jb), _ptr(q), _row_stride(q), _ptr(k), _row_stride(k),
                         _ptr(v), _row_stride(v), _ptr(pos_bias), _ptr(time_bias), _ptr(out), _row_stride(out),
                         _ptr(ws), ws.numel(), _stream(stream)), "hstu_attn_fwd")
    return (out, ws) if return_workspace else out


def attn_bwd(q, k, v, dout, seq_offsets, timestamps, pos_bias, time_bias, num_heads: int, num_targets=None,
             time_div: float = 0.301, stream=None, force_simt: bool = False):
    """Returns dq, dk, dv ([T, H*dh], dtype of q) and the rab gradients (float, table shape)."""
    T = q.shape[0]
    dh = q.shape[1] // num_heads
    dt = _dtype_code(q)
    d = attn_desc(num_heads, dh, dt, pos_bias.dim() == 2, force_simt, time_div)
    jb = jagged(seq_offsets, timestamps, T, num_targets)
    nbytes = _c_size()
    _check(_lib_attn_bwd_ws(ctypes.byref(d), jb.batch, T, ctypes.byref(nbytes)), "hstu_attn_bwd_workspace_size")
    ws = _workspace(nbytes.value, q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dpos = torch.zeros_like(pos_bias, dtype=torch.float32)
    dtime = torch.zeros_like(time_bias, dtype=torch.float32)
    _check(_lib_attn_bwd(ctypes.byref(d), ctypes.byref(jb), _ptr(q), _row_stride(q), _ptr(k), _row_stride(k),
                         _ptr(v), _row_stride(v), _ptr(pos_bias), _ptr(time_bias), _ptr(dout), _row_stride(dout),
                         _ptr(dq), _row_stride(dq), _ptr(dk), _row_stride(dk), _ptr(dv), _row_stride(dv),
                         _ptr(dpos), _ptr(dtime), _ptr(ws), ws.numel(), _stream(stream)), "hstu_attn_bwd")
    return dq, dk, dv, dpos, dtime


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    st = _c_i32()
    _check(_lib_ws_status(_ptr(ws), ctypes.byref(st), _stream(stream)), "hstu_workspace_status")
    return st.value


# ----------------------------------------------------------------------------
# layer
# ----------------------------------------------------------------------------

_WEIGHT_NAMES = ("w1", "b1", "ln1_gamma", "ln1_beta", "ln2_gamma", "ln2_beta", "w2", "b2", "pos_bias", "time_bias")


def layer_weights(w: Dict[str, torch.Tensor]) -> LayerWeights:
    return LayerWeights(*[_ptr(w[n]) for n in _WEIGHT_NAMES])


@dataclass
class Saved:
    xhat: torch.Tensor
    ln1_mean: torch.Tensor
    ln1_rstd: torch.Tensor
    z: torch.Tensor
    uvqk: torch.Tensor
    attn_out: torch.Tensor
    ln2_mean: torch.Tensor
    ln2_rstd: torch.Tensor
    gate: Optional[torch.Tensor] = None   # LN2(A V) * U; None: the backward recomputes it

    @staticmethod
    def alloc(T: int, d_model: int, hv: int, dtype, device, keep_gate: bool = True) -> "Saved":
        f = dict(dtype=torch.float32, device=device)
        e = dict(dtype=dtype, device=device)
        return Saved(torch.empty(T, d_model, **e), torch.empty(T, **f), torch.empty(T, **f),
                     torch.empty(T, 4 * hv, **e), torch.empty(T, 4 * hv, **e), torch.empty(T, hv, **e),
                     torch.empty(T, **f), torch.empty(T, **f), torch.empty(T, hv, **e) if keep_gate else None)

    def c(self) -> LayerSaved:
        return LayerSaved(*[_ptr(getattr(self, n)) if getattr(self, n) is not None else None
                            for n in ("xhat", "ln1_mean", "ln1_rstd", "z", "uvqk", "attn_out", "ln2_mean", "ln2_rstd",
                                      "gate")])


class Layer:
    """One HSTU layer's descriptor and parameters (device tensors)."""

    def __init__(self, weights: Dict[str, torch.Tensor], d_model: int, num_heads: int, head_dim: int,
                 force_simt: bool = False, eps: float = 1e-5, time_div: float = 0.301,
                 residual_fp32: bool = False, short_sequences: bool = False, workspaces: Optional[dict] = None):
        """residual_fp32: X, Y (and dX, dY) are fp32 tensors while weights and
        activations use the weights' dtype.  short_sequences: every sequence has
        at most 128 tokens, and the forward runs as one fused kernel where the
        shapes allow it (HSTU_FLAG_SHORT_SEQUENCES).  workspaces: a dict shared by
        layers of the same shape that run one after the other on one stream, so
        that they use one workspace per entry point (and can reuse its attention
        preparation, see `reuse_prep`)."""
        self.w = weights
        self.dtype = weights["w1"].dtype
        self.io_dtype = torch.float32 if residual_fp32 else self.dtype
        self.d_model, self.num_heads, self.head_dim = d_model, num_heads, head_dim
        self.desc = layer_desc(d_model, num_heads, head_dim, _dtype_code(weights["w1"]),
                               weights["pos_bias"].dim() == 2, force_simt, eps, time_div,
                               io_dtype=DTYPE_F32 if residual_fp32 else None)
        if short_sequences:
            self.desc.attn.flags |= FLAG_SHORT_SEQUENCES
        self.cw = layer_weights(weights)
        self._ws = {} if workspaces is None else workspaces

    @property
    def hv(self) -> int:
        return self.num_heads * self.head_dim

    def _get_ws(self, key, fn, B, T, device):
        nbytes = _c_size()
        _check(fn(ctypes.byref(self.desc), B, T, ctypes.byref(nbytes)), "workspace_size")
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes.value or ws.device != device:
            ws = _workspace(nbytes.value, device)
            self._ws[key] = ws
        return ws

    def _desc_for(self, reuse_prep: bool):
        if not reuse_prep:
            return self.desc
        d = type(self.desc).from_buffer_copy(self.desc)
        d.attn.flags |= FLAG_REUSE_PREP
        return d

    def forward(self, x, seq_offsets, timestamps, num_targets=None, saved: Optional[Saved] = None, out=None,
                stream=None, reuse_prep: bool = False):
        """reuse_prep: the workspace holds the attention preparation of an earlier
        forward on the same batch (HSTU_FLAG_REUSE_PREP)."""
        T = x.shape[0]
        jb = jagged(seq_offsets, timestamps, T, num_targets)
        ws = self._get_ws("fwd", _lib_layer_fwd_ws, jb.batch, T, x.device)
        y = torch.empty_like(x) if out is None else out
        sv = saved.c() if saved is not None else None
        desc = self._desc_for(reuse_prep)
        _check(_lib_layer_fwd(ctypes.byref(desc), ctypes.byref(self.cw), ctypes.byref(jb), _ptr(x), _ptr(y),
                              ctypes.byref(sv) if sv is not None else None, _ptr(ws), ws.numel(), _stream(stream)),
               "hstu_layer_fwd")
        return y

    def forward_host(self, x, seq_offsets, timestamps, num_chunks: int, num_targets=None, out=None, device=None,
                     stream=None):
        """The forward from and to host memory (hstu_layer_fwd_host): x, out [T, d]
        and timestamps on the host (page-locked for the copies to overlap the
        computation), seq_offsets / num_targets host int32 tensors."""
        for t in (x, seq_offsets, timestamps) + ((num_targets,) if num_targets is not None else ()):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("forward_host takes contiguous host tensors")
        B = seq_offsets.numel() - 1
        T = int(seq_offsets[-1])
        dev = torch.device("cuda") if device is None else device
        nbytes = _c_size()
        _check(_lib_layer_fwd_host_ws(ctypes.byref(self.desc), B, T, num_chunks, ctypes.byref(nbytes)),
               "hstu_layer_fwd_host_workspace_size")
        ws = self._ws.get("fwd_host")
        if ws is None or ws.numel() < nbytes.value or ws.device != dev:
            ws = _workspace(nbytes.value, dev)
            self._ws["fwd_host"] = ws
        y = torch.empty_like(x) if out is None else out
        _check(_lib_layer_fwd_host(ctypes.byref(self.desc), ctypes.byref(self.cw), B, _ptr(seq_offsets),
                                   _ptr(num_targets) if num_targets is not None else None, _ptr(timestamps),
                                   _ptr(x), _ptr(y), num_chunks, _ptr(ws), ws.numel(), _stream(stream)),
               "hstu_layer_fwd_host")
        return y

    def backward(self, x, dy, saved: Saved, seq_offsets, timestamps, num_targets=None, grads=None, dx=None,
                 stream=None, keep_duvqk: bool = True, reuse_prep: bool = False):
        """reuse_prep: the workspace holds the attention preparation of an earlier
        backward on the same batch (HSTU_FLAG_REUSE_PREP)."""
        T = x.shape[0]
        jb = jagged(seq_offsets, timestamps, T, num_targets)
        ws = self._get_ws("bwd", _lib_layer_bwd_ws, jb.batch, T, x.device)
        dev = x.device
        if grads is None:
            grads = {n: torch.empty(self.w[n].shape, dtype=torch.float32, device=dev)
                     for n in ("w1", "b1", "ln1_gamma", "ln1_beta", "ln2_gamma", "ln2_beta", "w2", "b2", "pos_bias",
                               "time_bias")}
            grads["uvqk"] = torch.empty(T, 4 * self.hv, dtype=self.dtype, device=dev) if keep_duvqk else None
        g = LayerGrads(*[_ptr(grads[n]) for n in ("w1", "b1", "ln1_gamma", "ln1_beta", "ln2_gamma", "ln2_beta", "w2",
                                                  "b2", "pos_bias", "time_bias")], _ptr(grads.get("uvqk")))
        dx = torch.empty_like(x) if dx is None else dx
        sv = saved.c()
        desc = self._desc_for(reuse_prep)
        _check(_lib_layer_bwd(ctypes.byref(desc), ctypes.byref(self.cw), ctypes.byref(jb), _ptr(x),
                              ctypes.byref(sv), _ptr(dy), _ptr(dx), ctypes.byref(g), _ptr(ws), ws.numel(),
                              _stream(stream)), "hstu_layer_bwd")
        return dx, grads


# ----------------------------------------------------------------------------
# M-FALCON, Stochastic Length, diagnostics
# ----------------------------------------------------------------------------

def mfalcon_rank(layers: Sequence[Layer], hist_offsets, hist_x, hist_ts, cand_offsets, cand_x, cand_ts,
                 microbatch: int, max_candidates: int, workspace=None, stream=None, out=None):
    L = len(layers)
    desc = layers[0].desc
    arr = (LayerWeights * L)(*[ly.cw for ly in layers])
    U = hist_offsets.numel() - 1
    H = hist_x.shape[0]
    nbytes = _c_size()
    _check(_lib_mf_ws(ctypes.byref(desc), L, U, H, microbatch, ctypes.byref(nbytes)), "mfalcon_rank_workspace_size")
    ws = workspace if workspace is not None and workspace.numel() >= nbytes.value else _workspace(nbytes.value,
                                                                                                   cand_x.device)
    if out is None:
        out = torch.empty_like(cand_x)
    _check(_lib_mf(ctypes.byref(desc), arr, L, U, H, max_candidates, microbatch, _ptr(hist_offsets), _ptr(hist_x),
                   _ptr(hist_ts), _ptr(cand_offsets), _ptr(cand_x), _ptr(cand_ts), _ptr(out), _ptr(ws), ws.numel(),
                   _stream(stream)), "mfalcon_rank")
    return out


def mfalcon_workspace(layers: Sequence[Layer], num_users: int, hist_total: int, microbatch: int, device):
    nbytes = _c_size()
    _check(_lib_mf_ws(ctypes.byref(layers[0].desc), len(layers), num_users, hist_total, microbatch,
                      ctypes.byref(nbytes)), "mfalcon_rank_workspace_size")
    return _workspace(nbytes.value, device)


def stochastic_length(seq_offsets, coins, keys, max_len: int, prob_u32: int, stream=None):
    B = seq_offsets.numel() - 1
    T = keys.numel()
    nbytes = _c_size()
    _check(_lib_sl_ws(B, T, ctypes.byref(nbytes)), "hstu_stochastic_length_workspace_size")
    ws = _workspace(nbytes.value, seq_offsets.device)
    out_offs = torch.empty(B + 1, dtype=torch.int32, device=seq_offsets.device)
    out_idx = torch.empty(max(T, 1), dtype=torch.int32, device=seq_offsets.device)
    _check(_lib_sl(B, T, _ptr(seq_offsets), _ptr(coins), _ptr(keys), max_len, prob_u32 & 0xFFFFFFFF, _ptr(out_offs),
                   _ptr(out_idx), _ptr(ws), ws.numel(), _stream(stream)), "hstu_stochastic_length")
    return out_offs, out_idx


def gather_rows(src: torch.Tensor, index: torch.Tensor, count: torch.Tensor, out: torch.Tensor, stream=None):
    row_bytes = src[0].numel() * src.element_size() if src.dim() > 1 else src.element_size()
    _check(_lib_gather(_ptr(src), _ptr(out), row_bytes, _ptr(index), _ptr(count), out.shape[0], _stream(stream)),
           "hstu_gather_rows")
    return out


def debug_rab_buckets(seq_offsets, timestamps, pairs: torch.Tensor, num_targets=None, time_div: float = 0.301,
                      stream=None):
    d = attn_desc(1, 64, DTYPE_BF16, False, False, time_div)
    jb = jagged(seq_offsets, timestamps, timestamps.numel(), num_targets)
    out = torch.empty_like(pairs)
    _check(_lib_dbg_buckets(ctypes.byref(d), ctypes.byref(jb), _ptr(pairs), pairs.shape[0], _ptr(out),
                            _stream(stream)), "hstu_debug_rab_buckets")
    return out


def debug_timeout_probe(timeout_ns: int, status: torch.Tensor, stream=None):
    _check(_lib_dbg_timeout(timeout_ns, _ptr(status), _stream(stream)), "hstu_debug_timeout_probe")
    return status


# ----------------------------------------------------------------------------
# data-parallel sharding (host only)
# ----------------------------------------------------------------------------
_lib_lpt = _sig("hstu_lpt_partition", _c_int, [_c_i32, _c_vp, _c_vp, _c_i32, _c_dbl, _c_vp, _c_vp])
EXPORTED.append("hstu_lpt_partition")


def lpt_partition(seq_offsets, world: int, num_targets=None, token_weight: float = 0.0):
    """Rank of every sequence of a jagged batch (host arrays) and each rank's
    total cost, from hstu_lpt_partition: returns (rank_of int32[B], cost float64[world])."""
    import numpy as np
    offs = np.ascontiguousarray(seq_offsets, dtype=np.int32)
    B = offs.size - 1
    nt = None if num_targets is None else np.ascontiguousarray(num_targets, dtype=np.int32)
    rank_of = np.zeros(max(B, 1), dtype=np.int32)
    cost = np.zeros(max(world, 1), dtype=np.float64)
    _check(_lib_lpt(B, offs.ctypes.data_as(_c_vp), None if nt is None else nt.ctypes.data_as(_c_vp), world,
                    float(token_weight), rank_of.ctypes.data_as(_c_vp), cost.ctypes.data_as(_c_vp)),
           "hstu_lpt_partition")
    return rank_of[:B], cost[:world]


# ----------------------------------------------------------------------------
# tracing
# ----------------------------------------------------------------------------
_lib_trace_enable = _sig("hstu_trace_enable", _c_int, [_c_int])
_lib_trace_read = _sig("hstu_trace_read", _c_int, [_c_i32, _c_vp, _c_vp, _c_vp, _c_vp])
EXPORTED += ["hstu_trace_enable", "hstu_trace_read"]


def trace_enable(on: bool = True):
    _check(_lib_trace_enable(1 if on else 0), "hstu_trace_enable")


def trace_read(max_kernels: int = 64) -> Dict[str, Dict[str, float]]:
    """{kernel name: {"count": launches, "ms": summed device time}} since trace_enable."""
    names = ctypes.create_string_buffer(32 * max_kernels)
    counts = (_c_i32 * max_kernels)()
    ms = (ctypes.c_double * max_kernels)()
    n = _c_i32()
    _check(_lib_trace_read(max_kernels, names, counts, ms, ctypes.byref(n)), "hstu_trace_read")
    out = {}
    for i in range(min(n.value, max_kernels)):
        nm = names.raw[32 * i:32 * i + 32].split(b"\0", 1)[0].decode()
        out[nm] = {"count": int(counts[i]), "ms": float(ms[i])}
    return out


def layer_weights_to_device(p, dtype, device="cuda") -> Dict[str, torch.Tensor]:
    """Device tensors of one layer's parameters (an object with w1, b1, ln1_g,
    ln1_b, ln2_g, ln2_b, w2, b2, pos_bias, time_bias arrays); linear weights in
    `dtype`, everything else float32."""
    import numpy as np

    def t(a, dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(device)

    return dict(w1=t(p.w1, dtype), b1=t(p.b1, torch.float32), ln1_gamma=t(p.ln1_g, torch.float32),
                ln1_beta=t(p.ln1_b, torch.float32), ln2_gamma=t(p.ln2_g, torch.float32),
                ln2_beta=t(p.ln2_b, torch.float32), w2=t(p.w2, dtype), b2=t(p.b2, torch.float32),
                pos_bias=t(p.pos_bias, torch.float32), time_bias=t(p.time_bias, torch.float32))
