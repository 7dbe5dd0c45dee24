"""Python binding of the C-ABI library ``libgdn_b200.so`` (include/gdn.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the stream.  If the library is
missing this module raises; there is no other implementation to fall back to.

Tensors (all contiguous, on one CUDA device):
  q, k        [T, H_k*d_k]  (or [T, H_k, d_k])   activation dtype
  v, z        [T, H_v*d_v]                       activation dtype
  a, b        [T, H_v]                           activation dtype
  conv_state  [N, 2*H_k*d_k + H_v*d_v, 3]        activation dtype, updated in place
  rec_state   [N, H_v, d_v, d_k] float32         updated in place
  cu_seqlens  [N + 1] int32                      (prefill only)
  weights     dict: conv_w [C, 4], A_log [H_v], dt_bias [H_v], norm_w [d_v], float32
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn_b200.so")

_DT = {torch.bfloat16: 0, torch.float32: 1}


CUDA_ERROR = 3   # GDN_ERR_CUDA


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = "%s: %s (status %d)" % (what, status_string(status), status)
        if status == CUDA_ERROR:
            msg += " [%s]" % lib().gdn_last_cuda_error().decode()
        super().__init__(msg)
        self.status = status


class _CConfig(ctypes.Structure):
    _fields_ = [("n_k_heads", ctypes.c_int32), ("n_v_heads", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("conv_kernel", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("l2_eps", ctypes.c_float), ("norm_eps", ctypes.c_float),
                ("act_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("state_dtype", ctypes.c_int32), ("prefill_segments", ctypes.c_int32)]


class _CSegment(ctypes.Structure):
    _fields_ = [("dst", ctypes.c_void_p), ("width", ctypes.c_int32)]


class _CWeights(ctypes.Structure):
    _fields_ = [("conv_weight", ctypes.c_void_p), ("A_log", ctypes.c_void_p),
                ("dt_bias", ctypes.c_void_p), ("norm_weight", ctypes.c_void_p)]


_lib = None
EXPORTS = ("gdn_config_default", "gdn_prefill_workspace_size", "gdn_prefill_segments", "gdn_prefill", "gdn_decode",
           "gdn_decode_multi", "gdn_linear", "gdn_in_proj", "gdn_out_proj", "gdn_cp_workspace_size",
           "gdn_cp_local", "gdn_cp_finish", "gdn_prefill_host_workspace_size", "gdn_prefill_host",
           "gdn_check_device_error", "gdn_status_string", "gdn_last_cuda_error")
DECODE_MULTI_MAX_TOKENS = 16   # GDN_DECODE_MULTI_MAX_TOKENS
PREFILL_SPLIT = -1             # GDN_PREFILL_SPLIT: Config.prefill_segments value that splits the chain
LINEAR_MAX_SEGMENTS = 8        # GDN_LINEAR_MAX_SEGMENTS


def lib() -> ctypes.CDLL:
    """Load libgdn_b200.so (built in place by ``build.py``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libgdn_b200.so is not built; run `python -m "
                               "hybrid_linear_attention_mixer_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.gdn_config_default.argtypes = [vp]
        L.gdn_config_default.restype = None
        L.gdn_prefill_workspace_size.argtypes = [vp, i64, i32]
        L.gdn_prefill_workspace_size.restype = sz
        L.gdn_prefill_segments.argtypes = [vp, i64, i32]
        L.gdn_prefill_segments.restype = i32
        L.gdn_prefill.argtypes = [vp, vp] + [vp] * 8 + [vp, i32, i64, vp, vp, sz, vp]
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_decode.argtypes = [vp, vp] + [vp] * 8 + [i32, vp, vp]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_decode_multi.argtypes = [vp, vp] + [vp] * 8 + [i32, i32, vp, vp, vp, vp]
        L.gdn_decode_multi.restype = ctypes.c_int
        L.gdn_linear.argtypes = [vp, vp, i64, i32, i32, vp, i32, vp]
        L.gdn_linear.restype = ctypes.c_int
        L.gdn_in_proj.argtypes = [vp, vp, vp, i64, i32] + [vp] * 6 + [vp]
        L.gdn_in_proj.restype = ctypes.c_int
        L.gdn_out_proj.argtypes = [vp, vp, vp, i64, i32, vp, vp]
        L.gdn_out_proj.restype = ctypes.c_int
        L.gdn_cp_workspace_size.argtypes = [vp, i64]
        L.gdn_cp_workspace_size.restype = sz
        L.gdn_cp_local.argtypes = [vp, vp] + [vp] * 5 + [vp, i64, vp, vp, sz, vp]
        L.gdn_cp_local.restype = ctypes.c_int
        L.gdn_cp_finish.argtypes = [vp, vp, vp, vp, i32, i32, vp, i64, vp, vp, vp, sz, vp]
        L.gdn_cp_finish.restype = ctypes.c_int
        L.gdn_prefill_host_workspace_size.argtypes = [vp, i64, i32]
        L.gdn_prefill_host_workspace_size.restype = sz
        L.gdn_prefill_host.argtypes = [vp, vp] + [vp] * 8 + [vp, i32, i64, vp, vp, sz, vp]
        L.gdn_prefill_host.restype = ctypes.c_int
        L.gdn_check_device_error.argtypes = [vp]
        L.gdn_check_device_error.restype = ctypes.c_int
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_last_cuda_error.argtypes = []
        L.gdn_last_cuda_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().gdn_status_string(int(s)).decode()


@dataclass
class Config:
    """Layer shape; the defaults are the published layer (16 / 48 heads of 128, K = 4)."""
    n_k_heads: int = 16
    n_v_heads: int = 48
    d_k: int = 128
    d_v: int = 128
    conv_kernel: int = 4
    chunk: int = 64
    l2_eps: float = 1e-6
    norm_eps: float = 1e-6
    act_dtype: torch.dtype = torch.bfloat16
    out_dtype: torch.dtype = torch.bfloat16
    state_dtype: torch.dtype = torch.float32   # bf16: the recurrent state stored in bf16
    prefill_segments: int = 0                  # chunk ranges a prefill is pipelined over; 0: automatic;
                                               # PREFILL_SPLIT: one sequence's chain split in two

    @property
    def channels(self) -> int:
        return 2 * self.n_k_heads * self.d_k + self.n_v_heads * self.d_v

    def c(self) -> _CConfig:
        return _CConfig(self.n_k_heads, self.n_v_heads, self.d_k, self.d_v, self.conv_kernel,
                        self.chunk, self.l2_eps, self.norm_eps, _DT[self.act_dtype],
                        _DT[self.out_dtype], _DT[self.state_dtype], self.prefill_segments)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, device):
    if t.dtype != dtype:
        raise TypeError("%s: dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))


def _weights(w: dict, device) -> _CWeights:
    for n in ("conv_w", "A_log", "dt_bias", "norm_w"):
        _check(w[n], n, torch.float32, device)
    return _CWeights(w["conv_w"].data_ptr(), w["A_log"].data_ptr(), w["dt_bias"].data_ptr(),
                     w["norm_w"].data_ptr())


def workspace_size(cfg: Config, T_total: int, n_seqs: int) -> int:
    c = cfg.c()
    return int(lib().gdn_prefill_workspace_size(ctypes.byref(c), int(T_total), int(n_seqs)))


def prefill_segments(cfg: Config, T_total: int, n_seqs: int) -> int:
    """Chunk ranges a prefill of this size is pipelined over (1: one piece); a call
    launches 2 + 4 n kernels (6 for n = 1)."""
    c = cfg.c()
    return int(lib().gdn_prefill_segments(ctypes.byref(c), int(T_total), int(n_seqs)))


def prefill(cfg: Config, w: dict, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens,
            out=None, workspace=None, stream=None):
    """Packed variable-length prefill; returns out [T, H_v*d_v] (out_dtype)."""
    dev = q.device
    T = q.shape[0]
    for n, t in (("q", q), ("k", k), ("v", v), ("a", a), ("b", b), ("z", z),
                 ("conv_state", conv_state)):
        _check(t, n, cfg.act_dtype, dev)
    _check(rec_state, "rec_state", cfg.state_dtype, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev)
    n_seqs = cu_seqlens.shape[0] - 1
    if out is None:
        out = torch.empty((T, cfg.n_v_heads * cfg.d_v), dtype=cfg.out_dtype, device=dev)
    _check(out, "out", cfg.out_dtype, dev)
    need = workspace_size(cfg, T, n_seqs)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    c, cw = cfg.c(), _weights(w, dev)
    s = lib().gdn_prefill(ctypes.byref(c), ctypes.byref(cw), _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                          _ptr(b), _ptr(z), _ptr(conv_state), _ptr(rec_state), _ptr(cu_seqlens),
                          n_seqs, T, _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_prefill")
    return out


def decode(cfg: Config, w: dict, q, k, v, a, b, z, conv_state, rec_state, out=None, stream=None):
    """One token per sequence; returns out [N, H_v*d_v] (out_dtype)."""
    dev = q.device
    N = q.shape[0]
    for n, t in (("q", q), ("k", k), ("v", v), ("a", a), ("b", b), ("z", z),
                 ("conv_state", conv_state)):
        _check(t, n, cfg.act_dtype, dev)
    _check(rec_state, "rec_state", cfg.state_dtype, dev)
    if out is None:
        out = torch.empty((N, cfg.n_v_heads * cfg.d_v), dtype=cfg.out_dtype, device=dev)
    _check(out, "out", cfg.out_dtype, dev)
    c, cw = cfg.c(), _weights(w, dev)
    s = lib().gdn_decode(ctypes.byref(c), ctypes.byref(cw), _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                         _ptr(b), _ptr(z), _ptr(conv_state), _ptr(rec_state), N, _ptr(out),
                         _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_decode")
    return out


def decode_multi(cfg: Config, w: dict, q, k, v, a, b, z, conv_state, rec_state, n_tok: int, out=None,
                 state_snapshots=None, conv_snapshots=None, stream=None):
    """n_tok consecutive tokens per sequence (rows token-major within a sequence);
    returns out [N*n_tok, H_v*d_v].  Optional snapshots receive the recurrent state
    [n_tok, N, H_v, d_v, d_k] (state dtype) and the conv state [n_tok, N, C, K-1] after each token."""
    dev = q.device
    rows = q.shape[0]
    if n_tok <= 0 or rows % n_tok:
        raise ValueError("rows (%d) must be a positive multiple of n_tok (%d)" % (rows, n_tok))
    N = rows // n_tok
    for n, t in (("q", q), ("k", k), ("v", v), ("a", a), ("b", b), ("z", z),
                 ("conv_state", conv_state)):
        _check(t, n, cfg.act_dtype, dev)
    _check(rec_state, "rec_state", cfg.state_dtype, dev)
    if state_snapshots is not None:
        _check(state_snapshots, "state_snapshots", cfg.state_dtype, dev)
    if conv_snapshots is not None:
        _check(conv_snapshots, "conv_snapshots", cfg.act_dtype, dev)
    if out is None:
        out = torch.empty((rows, cfg.n_v_heads * cfg.d_v), dtype=cfg.out_dtype, device=dev)
    _check(out, "out", cfg.out_dtype, dev)
    c, cw = cfg.c(), _weights(w, dev)
    opt = lambda t: None if t is None else _ptr(t)
    s = lib().gdn_decode_multi(ctypes.byref(c), ctypes.byref(cw), _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                               _ptr(b), _ptr(z), _ptr(conv_state), _ptr(rec_state), N, int(n_tok),
                               _ptr(out), opt(state_snapshots), opt(conv_snapshots), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_decode_multi")
    return out


def linear(x, w, outs=None, stream=None):
    """y = x . w^T on the tensor cores: x [M, K] and w [N, K] bf16, fp32 accumulation.
    ``outs`` (optional) is a list of bf16 [M, width] tensors that receive consecutive
    column ranges of y (widths adding up to N); default one [M, N] tensor.  Returns
    the list of outputs."""
    dev = x.device
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[1]:
        raise ValueError("x [M, K] and w [N, K] expected, got %s and %s" % (tuple(x.shape), tuple(w.shape)))
    M, K = x.shape
    N = w.shape[0]
    _check(x, "x", torch.bfloat16, dev)
    _check(w, "w", torch.bfloat16, dev)
    if outs is None:
        outs = [torch.empty((M, N), dtype=torch.bfloat16, device=dev)]
    if not 1 <= len(outs) <= LINEAR_MAX_SEGMENTS:
        raise ValueError("1..%d output segments" % LINEAR_MAX_SEGMENTS)
    for i, o in enumerate(outs):
        _check(o, "outs[%d]" % i, torch.bfloat16, dev)
        if o.dim() != 2 or o.shape[0] != M:
            raise ValueError("outs[%d] must be [M, width]" % i)
    segs = (_CSegment * len(outs))(*[_CSegment(o.data_ptr(), o.shape[1]) for o in outs])
    s = lib().gdn_linear(_ptr(x), _ptr(w), M, N, K, segs, len(outs), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_linear")
    return outs


def in_proj(cfg: Config, hidden, w_in, out: dict | None = None, stream=None) -> dict:
    """The mixer's input projection: hidden [T, d_model] bf16, w_in [16,480, d_model]
    bf16 at the published shape (channels q | k | v | z | a | b).  Returns q, k
    [T, H_k*d_k], v, z [T, H_v*d_v], a, b [T, H_v], all bf16 (written into ``out``'s
    tensors when given)."""
    dev = hidden.device
    T, D = hidden.shape
    _check(hidden, "hidden", torch.bfloat16, dev)
    _check(w_in, "w_in", torch.bfloat16, dev)
    qk, vz, ab = cfg.n_k_heads * cfg.d_k, cfg.n_v_heads * cfg.d_v, cfg.n_v_heads
    if tuple(w_in.shape) != (2 * qk + 2 * vz + 2 * ab, D):
        raise ValueError("w_in shape %s, expected %s" % (tuple(w_in.shape), (2 * qk + 2 * vz + 2 * ab, D)))
    widths = (("q", qk), ("k", qk), ("v", vz), ("z", vz), ("a", ab), ("b", ab))
    o = out if out is not None else {n: torch.empty((T, wd), dtype=torch.bfloat16, device=dev) for n, wd in widths}
    for n, wd in widths:
        _check(o[n], n, torch.bfloat16, dev)
        if o[n].numel() != T * wd:
            raise ValueError("%s must hold [T, %d]" % (n, wd))
    c = cfg.c()
    s = lib().gdn_in_proj(ctypes.byref(c), _ptr(hidden), _ptr(w_in), T, D, _ptr(o["q"]), _ptr(o["k"]),
                          _ptr(o["v"]), _ptr(o["z"]), _ptr(o["a"]), _ptr(o["b"]), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_in_proj")
    return o


def out_proj(cfg: Config, o, w_out, y=None, stream=None):
    """The mixer's output projection: o [T, H_v*d_v] bf16 (the layer's output),
    w_out [d_model, H_v*d_v] bf16 -> y [T, d_model] bf16."""
    dev = o.device
    o2 = o.reshape(o.shape[0], -1)
    T = o2.shape[0]
    D = w_out.shape[0]
    _check(o2, "o", torch.bfloat16, dev)
    _check(w_out, "w_out", torch.bfloat16, dev)
    if w_out.shape[1] != cfg.n_v_heads * cfg.d_v or o2.shape[1] != w_out.shape[1]:
        raise ValueError("w_out must be [d_model, H_v*d_v] and o [T, H_v*d_v]")
    if y is None:
        y = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
    _check(y, "y", torch.bfloat16, dev)
    c = cfg.c()
    s = lib().gdn_out_proj(ctypes.byref(c), _ptr(o2), _ptr(w_out), T, D, _ptr(y), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_out_proj")
    return y


def cp_workspace_size(cfg: Config, T_seg: int) -> int:
    c = cfg.c()
    return int(lib().gdn_cp_workspace_size(ctypes.byref(c), T_seg))


def cp_local(cfg: Config, w: dict, q, k, v, a, b, conv_state, workspace=None, summary=None, stream=None):
    """Context-parallel phase 1 on this rank's segment: returns (summary, workspace).
    conv_state [C, K-1] holds the K-1 input rows before the segment (updated in
    place to the segment's last rows); summary [2, H_v, d_k, d_k] fp32 = (P, S_loc)."""
    dev = q.device
    T = q.shape[0]
    for n, t in (("q", q), ("k", k), ("v", v), ("a", a), ("b", b), ("conv_state", conv_state)):
        _check(t, n, cfg.act_dtype, dev)
    if workspace is None:
        workspace = torch.empty(cp_workspace_size(cfg, T), dtype=torch.uint8, device=dev)
    if summary is None:
        summary = torch.empty((2, cfg.n_v_heads, cfg.d_k, cfg.d_k), dtype=torch.float32, device=dev)
    _check(summary, "summary", torch.float32, dev)
    c, cw = cfg.c(), _weights(w, dev)
    s = lib().gdn_cp_local(ctypes.byref(c), ctypes.byref(cw), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b),
                           _ptr(conv_state), T, _ptr(summary), _ptr(workspace), workspace.numel(), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_cp_local")
    return summary, workspace


def cp_finish(cfg: Config, w: dict, z, summaries, rank: int, state_in, workspace, out=None, state_out=None,
              stream=None):
    """Context-parallel phase 2: summaries [R, 2, H_v, d_k, d_k] (every rank's, in rank
    order), state_in [H_v, d_v, d_k] the state before the whole sequence.  Returns
    (out [T_seg, H_v*d_v], state_out [H_v, d_v, d_k]: the state after this segment)."""
    dev = z.device
    T = z.shape[0]
    _check(z, "z", cfg.act_dtype, dev)
    _check(summaries, "summaries", torch.float32, dev)
    _check(state_in, "state_in", torch.float32, dev)
    if out is None:
        out = torch.empty((T, cfg.n_v_heads * cfg.d_v), dtype=cfg.out_dtype, device=dev)
    if state_out is None:
        state_out = torch.empty_like(state_in)
    c, cw = cfg.c(), _weights(w, dev)
    s = lib().gdn_cp_finish(ctypes.byref(c), ctypes.byref(cw), _ptr(z), _ptr(summaries), summaries.shape[0],
                            rank, _ptr(state_in), T, _ptr(out), _ptr(state_out), _ptr(workspace),
                            workspace.numel(), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_cp_finish")
    return out, state_out


def check_device_error(stream=None) -> None:
    """Synchronise the stream and raise GdnError if the device error word holds an
    error: a bounded wait that ran out, or a failed device check of a prefill's
    inputs (malformed cu_seqlens, conv output beyond fp16)."""
    s = lib().gdn_check_device_error(_stream(stream))
    if s != 0:
        raise GdnError(s, "device")


def prefill_host_workspace_size(cfg: Config, T_total: int, n_seqs: int) -> int:
    c = cfg.c()
    return int(lib().gdn_prefill_host_workspace_size(ctypes.byref(c), T_total, n_seqs))


def prefill_host(cfg: Config, w: dict, host: dict, conv_state, rec_state, workspace=None, stream=None):
    """End-to-end prefill from host buffers through gdn_prefill_host: ``host`` holds CPU
    tensors q, k, v, a, b, z (act dtype), cu_seqlens (int32) and out (out dtype), page-
    locked for the copies to overlap the work.  The states stay on the device.  Returns
    host['out'], complete once the stream is synchronised."""
    dev = rec_state.device
    q = host["q"]
    T = q.shape[0]
    cu = host["cu_seqlens"]
    N = cu.shape[0] - 1
    for n in ("q", "k", "v", "a", "b", "z", "cu_seqlens", "out"):
        t = host[n]
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError("host[%r] must be a contiguous CPU tensor" % n)
    for n in ("q", "k", "v", "a", "b", "z"):
        if host[n].dtype != cfg.act_dtype:
            raise TypeError("host[%r]: dtype %s, expected %s" % (n, host[n].dtype, cfg.act_dtype))
    if cu.dtype != torch.int32 or host["out"].dtype != cfg.out_dtype:
        raise TypeError("cu_seqlens must be int32 and out of the out dtype")
    _check(conv_state, "conv_state", cfg.act_dtype, dev)
    _check(rec_state, "rec_state", cfg.state_dtype, dev)
    if workspace is None:
        workspace = torch.empty(prefill_host_workspace_size(cfg, T, N), dtype=torch.uint8, device=dev)
    c, cw = cfg.c(), _weights(w, dev)
    s = lib().gdn_prefill_host(ctypes.byref(c), ctypes.byref(cw), _ptr(q), _ptr(host["k"]), _ptr(host["v"]),
                               _ptr(host["a"]), _ptr(host["b"]), _ptr(host["z"]), _ptr(conv_state),
                               _ptr(rec_state), _ptr(cu), N, T, _ptr(host["out"]), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    if s != 0:
        raise GdnError(s, "gdn_prefill_host")
    return host["out"]
