"""fp64 CPU oracle for the Gated DeltaNet token mixer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline of ``bench.py`` use this package; the product path never imports it.
It shares no code with the CUDA path.

Three independent formulations of the same layer live here:

* ``forward`` -- the C oracle (``gdn_oracle.c``): token by token, fp64,
  threaded over (sequence, value head).  This is the reference every GPU
  result is compared with.
* ``brute_force`` -- pure numpy, builds the explicit d_k x d_k transition
  matrix alpha (I - beta k k^T) for every token; for tiny inputs only.
* ``chunked`` -- pure numpy fp64 chunked (WY / UT) form of the same
  recurrence.  It pins the chunk algebra: it must equal the sequential form.

Sources: the layer shape (16 key heads, 48 value heads of dim 128, short conv
of kernel 4, fixed-size recurrent state) is from "Qwen3.8-Flash-Next"
(llm-architectures-explained), "Every architecture field", and
"Qwen3.8-Flash-Next anatomy" (frontier-model-atlas), "Decoder microscope";
rms_norm_eps and the float32 state type from "Raw config fields"
(llm-atlas-9r2).  The pages name the gated delta rule but do not print it; the
recurrence used is its standard statement
    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t q_t / sqrt(d_k),
    alpha_t = exp(-exp(A_log) softplus(a_t + dt_bias)),  beta_t = sigmoid(b_t).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")

F64, F32, BF16 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the C oracle in place (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC,
                               "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("n_k_heads", ctypes.c_int), ("n_v_heads", ctypes.c_int),
                ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("conv_kernel", ctypes.c_int),
                ("l2_eps", ctypes.c_double), ("norm_eps", ctypes.c_double)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.gdn_oracle_forward.restype = ctypes.c_int
    return _lib


@dataclass
class Shape:
    n_k_heads: int
    n_v_heads: int
    d_k: int
    d_v: int
    conv_kernel: int = 4
    l2_eps: float = 1e-6
    norm_eps: float = 1e-6

    @property
    def channels(self) -> int:
        return 2 * self.n_k_heads * self.d_k + self.n_v_heads * self.d_v


def _act(x):
    """Activation array as (contiguous array, dtype code).  uint16 means bf16 bits."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, F32
    return np.ascontiguousarray(x, dtype=np.float64), F64


def act_to_f64(x) -> np.ndarray:
    """bf16 bit patterns (uint16) or floats -> float64, exactly."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def forward(shape: Shape, w: dict, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens,
            heads=None, threads: int | None = None, want_o_pre: bool = False) -> dict:
    """Run the C oracle.

    q, k: [T, H_k*d_k]; v, z: [T, H_v*d_v]; a, b: [T, H_v]; all of one dtype
    (uint16 = bf16 bits, float32 or float64).  w: conv_w [C, K], A_log [H_v],
    dt_bias [H_v], norm_w [d_v].  conv_state [N, C, K-1]; rec_state
    [N, n_sel, d_v, d_k] for the value heads ``heads`` (all when None).
    Returns fp64 out [T, n_sel, d_v], conv_state, rec_state (and o_pre).
    """
    lib = _load()
    arrs = [_act(x) for x in (q, k, v, a, b, z)]
    dts = {d for _, d in arrs}
    if len(dts) != 1:
        raise ValueError("activations must share one dtype")
    act_dtype = dts.pop()
    T = arrs[0][0].shape[0]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seqs = cu.shape[0] - 1
    if heads is None:
        hs = None
        n_sel = shape.n_v_heads
    else:
        hs = np.ascontiguousarray(heads, dtype=np.int32)
        n_sel = hs.shape[0]
    cs = np.array(conv_state, dtype=np.float64, order="C", copy=True)
    rs = np.array(rec_state, dtype=np.float64, order="C", copy=True)
    if cs.shape != (n_seqs, shape.channels, shape.conv_kernel - 1):
        raise ValueError("conv_state shape %s" % (cs.shape,))
    if rs.shape != (n_seqs, n_sel, shape.d_v, shape.d_k):
        raise ValueError("rec_state shape %s" % (rs.shape,))
    out = np.zeros((T, n_sel, shape.d_v), dtype=np.float64)
    o_pre = np.zeros_like(out) if want_o_pre else None
    cfg = _Cfg(shape.n_k_heads, shape.n_v_heads, shape.d_k, shape.d_v, shape.conv_kernel,
               shape.l2_eps, shape.norm_eps)
    ws = {n: np.ascontiguousarray(w[n], dtype=np.float64)
          for n in ("conv_w", "A_log", "dt_bias", "norm_w")}
    P = ctypes.c_void_p
    if threads is None:
        threads = len(os.sched_getaffinity(0))
    rc = lib.gdn_oracle_forward(
        ctypes.byref(cfg),
        P(ws["conv_w"].ctypes.data), P(ws["A_log"].ctypes.data), P(ws["dt_bias"].ctypes.data),
        P(ws["norm_w"].ctypes.data),
        *[P(x.ctypes.data) for x, _ in arrs], ctypes.c_int(act_dtype),
        P(cs.ctypes.data), P(rs.ctypes.data), P(cu.ctypes.data), ctypes.c_int(n_seqs),
        P(hs.ctypes.data) if hs is not None else P(0), ctypes.c_int(n_sel),
        P(out.ctypes.data), P(o_pre.ctypes.data) if o_pre is not None else P(0),
        ctypes.c_int(int(threads)))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    res = {"out": out, "conv_state": cs, "rec_state": rs}
    if want_o_pre:
        res["o_pre"] = o_pre
    return res


# ---------------------------------------------------------------------------
# Segment state maps (context-parallel prefill)
# ---------------------------------------------------------------------------
# Over one segment the recurrence maps the initial state affinely:
#     S_end = S_0 . P + S_loc.
# With v = 0 every update is S <- alpha S (I - beta k k^T), linear in S, so the run
# from S_0 = I returns P (d_v = d_k required); the run from S_0 = 0 returns S_loc.

def segment_map(shape: Shape, w: dict, q, k, v, a, b, conv_state):
    """(P [H_v, d_k, d_k], S_loc [H_v, d_v, d_k]) of one segment, fp64.
    conv_state [C, K-1]: the inputs before the segment."""
    assert shape.d_k == shape.d_v, "P has the state's shape only when d_k == d_v"
    T = np.asarray(q).shape[0]
    cu = np.array([0, T], np.int32)
    cs = np.asarray(act_to_f64(conv_state))[None]
    Hv, d = shape.n_v_heads, shape.d_k
    z = np.zeros((T, Hv * shape.d_v))
    acts = [act_to_f64(x) for x in (q, k, v, a, b)]
    S_loc = forward(shape, w, *acts, z, cs, np.zeros((1, Hv, d, d)), cu)["rec_state"][0]
    cs0 = cs.copy()
    cs0[:, 2 * shape.n_k_heads * shape.d_k:] = 0.0          # the v channels of the conv window
    eye = np.broadcast_to(np.eye(d), (1, Hv, d, d)).copy()
    P = forward(shape, w, acts[0], acts[1], np.zeros_like(acts[2]), acts[3], acts[4], z, cs0, eye, cu)["rec_state"][0]
    return P, S_loc


def fold_segment_maps(state_in, maps):
    """The state after the segments whose (P, S_loc) are listed, from state_in."""
    S = np.asarray(state_in, dtype=np.float64)
    for P, S_loc in maps:
        S = S @ P + S_loc
    return S


# ---------------------------------------------------------------------------
# Projections around the mixer
# ---------------------------------------------------------------------------
# The hidden size is 2,560 ("Qwen3.8-Flash-Next" (llm-atlas-9r2), "Key facts";
# (llm-architectures-explained), "Every architecture field", row d_model).  The
# pages do not print how the mixer's inputs are projected from it; the reading
# taken is one bias-free linear map per side, the input map's output channels
# in the order q | k | v | z | a | b, the output map from the 6,144 channels of
# the layer's output back to the hidden size.

def linear(x, w) -> np.ndarray:
    """y = x . w^T in fp64, x [M, K], w [N, K] (bf16 bit patterns or floats).
    The plain definition; numpy's matmul is the one step."""
    return act_to_f64(x) @ act_to_f64(w).T


def in_proj_widths(shape: Shape):
    """(name, width) of the input projection's output channels, in order."""
    qk, vz = shape.n_k_heads * shape.d_k, shape.n_v_heads * shape.d_v
    return (("q", qk), ("k", qk), ("v", vz), ("z", vz), ("a", shape.n_v_heads), ("b", shape.n_v_heads))


def in_proj(shape: Shape, hidden, w_in) -> dict:
    """hidden [T, d_model] -> {q, k, v, z, a, b} fp64, split in the order above."""
    y = linear(hidden, w_in)
    out, c = {}, 0
    for name, wd in in_proj_widths(shape):
        out[name] = y[:, c:c + wd]
        c += wd
    assert c == y.shape[1], "w_in has %d rows, the split needs %d" % (y.shape[1], c)
    return out


def out_proj(o, w_out) -> np.ndarray:
    """o [T, H_v*d_v] -> y [T, d_model] fp64."""
    o = np.asarray(o)
    return linear(o.reshape(o.shape[0], -1), w_out)


# ---------------------------------------------------------------------------
# Pure-numpy formulations (small inputs only)
# ---------------------------------------------------------------------------

def _silu(x):
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def _sigmoid(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def features(shape: Shape, w: dict, q, k, v, a, b, conv_state, cu_seqlens):
    """Per-token post-conv features and gates, in numpy fp64.

    Returns qh, kh [T, H_k, d_k] (L2-normalised), vh [T, H_v, d_v],
    log_alpha [T, H_v], beta [T, H_v].  The conv runs over the concatenated
    q|k|v channels, each sequence seeded with its conv_state.
    """
    q, k, v, a, b = (act_to_f64(x) for x in (q, k, v, a, b))
    T = q.shape[0]
    K = shape.conv_kernel
    x = np.concatenate([q, k, v], axis=1)              # [T, C]
    cw = np.asarray(w["conv_w"], dtype=np.float64)      # [C, K]
    y = np.zeros_like(x)
    for s in range(len(cu_seqlens) - 1):
        t0, t1 = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        hist = np.asarray(conv_state[s], dtype=np.float64).T          # [K-1, C], oldest first
        xs = np.concatenate([hist, x[t0:t1]], axis=0)                 # [K-1+L, C]
        for t in range(t1 - t0):
            y[t0 + t] = np.sum(xs[t:t + K] * cw.T, axis=0)
    y = _silu(y)
    Hk, Hv, dk, dv = shape.n_k_heads, shape.n_v_heads, shape.d_k, shape.d_v
    qh = y[:, :Hk * dk].reshape(T, Hk, dk)
    kh = y[:, Hk * dk:2 * Hk * dk].reshape(T, Hk, dk)
    vh = y[:, 2 * Hk * dk:].reshape(T, Hv, dv)
    qh = qh / np.sqrt(np.sum(qh * qh, axis=-1, keepdims=True) + shape.l2_eps)
    kh = kh / np.sqrt(np.sum(kh * kh, axis=-1, keepdims=True) + shape.l2_eps)
    A = np.exp(np.asarray(w["A_log"], dtype=np.float64))
    dt = np.asarray(w["dt_bias"], dtype=np.float64)
    log_alpha = -A[None, :] * _softplus(a + dt[None, :])
    beta = _sigmoid(b)
    return qh, kh, vh, log_alpha, beta


def gated_rmsnorm(o, z, norm_w, eps):
    """out = o * rsqrt(mean(o^2) + eps) * w * SiLU(z), over the last axis."""
    z = act_to_f64(z)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + eps) * np.asarray(norm_w, np.float64) * _silu(z)


def brute_force(shape: Shape, w: dict, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens):
    """Token-by-token recurrence with the explicit matrix alpha (I - beta k k^T).

    Same signature and result layout as ``forward`` with all heads selected.
    """
    qh, kh, vh, la, beta = features(shape, w, q, k, v, a, b, conv_state, cu_seqlens)
    Hk, Hv, dk, dv = shape.n_k_heads, shape.n_v_heads, shape.d_k, shape.d_v
    G = Hv // Hk
    T = qh.shape[0]
    S_all = np.array(rec_state, dtype=np.float64, copy=True)
    o = np.zeros((T, Hv, dv))
    I = np.eye(dk)
    for s in range(len(cu_seqlens) - 1):
        for h in range(Hv):
            S = S_all[s, h]
            for t in range(int(cu_seqlens[s]), int(cu_seqlens[s + 1])):
                kk = kh[t, h // G][:, None]
                al, be = np.exp(la[t, h]), beta[t, h]
                S = al * S @ (I - be * (kk @ kk.T)) + be * vh[t, h][:, None] @ kk.T
                o[t, h] = S @ qh[t, h // G] / np.sqrt(dk)
            S_all[s, h] = S
    out = gated_rmsnorm(o, np.asarray(z).reshape(T, Hv, dv), w["norm_w"], shape.norm_eps)
    return {"out": out, "o_pre": o, "rec_state": S_all}


def chunked(shape: Shape, w: dict, q, k, v, a, b, z, conv_state, rec_state, cu_seqlens,
            chunk: int = 64):
    """fp64 chunked (WY / UT) form of the same recurrence.

    Inside a chunk of C tokens with start state S0, gate prefix sums
    g_r = sum_{i<=r} log alpha_i and u_r = beta_r (v_r - alpha_r S_{r-1} k_r):
        A_rj = beta_r exp(g_r - g_j) k_r.k_j  (j < r),  T = (I + A)^-1 diag(beta)
        W = T diag(exp g) K,  U~ = T V,  U = U~ - W S0^T
        O = (diag(exp g) Q S0^T + (Q K^T o M) U) / sqrt(d_k),  M_rj = exp(g_r - g_j), j <= r
        S_C = exp(g_C) S0 + U^T diag(exp(g_C - g)) K
    Only exp of non-positive arguments is ever formed.
    """
    qh, kh, vh, la, beta = features(shape, w, q, k, v, a, b, conv_state, cu_seqlens)
    Hk, Hv, dk, dv = shape.n_k_heads, shape.n_v_heads, shape.d_k, shape.d_v
    G = Hv // Hk
    T = qh.shape[0]
    S_all = np.array(rec_state, dtype=np.float64, copy=True)
    o = np.zeros((T, Hv, dv))
    for s in range(len(cu_seqlens) - 1):
        t0, t1 = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        for h in range(Hv):
            S = S_all[s, h]
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                Q, Kc, V = qh[c0:c1, h // G], kh[c0:c1, h // G], vh[c0:c1, h]
                g = np.cumsum(la[c0:c1, h])
                bt = beta[c0:c1, h]
                n = c1 - c0
                D = g[:, None] - g[None, :]
                low = np.tril(np.ones((n, n)), -1)
                Gm = np.exp(np.where(low > 0, D, 0.0)) * low
                Amat = bt[:, None] * Gm * (Kc @ Kc.T)
                Tm = np.linalg.solve(np.eye(n) + Amat, np.diag(bt))
                Wm = Tm @ (np.exp(g)[:, None] * Kc)
                U = Tm @ V - Wm @ S.T
                M = np.exp(np.where(np.tril(np.ones((n, n))) > 0, D, -np.inf))
                o[c0:c1, h] = (np.exp(g)[:, None] * (Q @ S.T) + ((Q @ Kc.T) * M) @ U) / np.sqrt(dk)
                S = np.exp(g[-1]) * S + U.T @ (np.exp(g[-1] - g)[:, None] * Kc)
            S_all[s, h] = S
    out = gated_rmsnorm(o, np.asarray(z).reshape(T, Hv, dv), w["norm_w"], shape.norm_eps)
    return {"out": out, "o_pre": o, "rec_state": S_all}
