"""Shared helpers of the GPU parity tests: run one workload through the C ABI
(via the Python binding) and through the fp64 oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from hybrid_linear_attention_mixer_b200 import gdn, inputs

# Tolerances of the layer's parity bar: output within 2e-2 of max|out| (bf16 output),
# final fp32 state within 1e-3 of max|S|.
OUT_TOL = 2e-2
STATE_TOL = 1e-3


def t_act(x: np.ndarray, dev) -> torch.Tensor:
    """numpy activation (uint16 bf16 bits or float32) -> torch tensor on dev."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(x).to(dev)


def shape_of(case) -> oracle.Shape:
    return oracle.Shape(case.n_k_heads, case.n_v_heads, case.d_k, case.d_v, case.conv_kernel,
                        case.l2_eps, case.norm_eps)


def config_of(case, out_dtype=None) -> gdn.Config:
    act = torch.bfloat16 if case.bf16 else torch.float32
    return gdn.Config(case.n_k_heads, case.n_v_heads, case.d_k, case.d_v, case.conv_kernel, 64,
                      case.l2_eps, case.norm_eps, act, out_dtype or act)


def weights_on(case, dev) -> dict:
    return {n: torch.from_numpy(np.ascontiguousarray(case.weights[n], dtype=np.float32)).to(dev)
            for n in ("conv_w", "A_log", "dt_bias", "norm_w")}


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def gpu_prefill(case, acts=None, conv_state=None, rec_state=None, cu=None, dev="cuda:0",
                out_dtype=None):
    """Run gdn_prefill; returns dict of fp64 numpy out [T, Hv, dv], conv_state, rec_state."""
    acts = case.acts if acts is None else acts
    cs = case.conv_state if conv_state is None else conv_state
    rs = case.rec_state if rec_state is None else rec_state
    cu = case.cu_seqlens if cu is None else cu
    cfg = config_of(case, out_dtype)
    w = weights_on(case, dev)
    d = {n: t_act(acts[n], dev) for n in "qkvabz"}
    cs_t = t_act(cs, dev)
    rs_t = torch.from_numpy(np.ascontiguousarray(rs, dtype=np.float32)).to(dev)
    cu_t = torch.from_numpy(np.ascontiguousarray(cu, dtype=np.int32)).to(dev)
    out = gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs_t, rs_t, cu_t)
    gdn.check_device_error()
    T = d["q"].shape[0]
    return {"out": to_f64(out).reshape(T, case.n_v_heads, case.d_v),
            "conv_state_t": cs_t, "conv_state": to_f64(cs_t), "rec_state": to_f64(rs_t)}


def oracle_run(case, acts=None, conv_state=None, rec_state=None, cu=None, heads=None, threads=None):
    acts = case.acts if acts is None else acts
    cs = case.conv_state if conv_state is None else conv_state
    rs = case.rec_state if rec_state is None else rec_state
    cu = case.cu_seqlens if cu is None else cu
    cs64 = oracle.act_to_f64(cs)
    rs_sel = rs if heads is None else rs[:, heads]
    return oracle.forward(shape_of(case), case.weights, *[acts[n] for n in "qkvabz"], cs64, rs_sel,
                          cu, heads=heads, threads=threads)


def rel_err(x, ref) -> float:
    den = float(np.abs(ref).max())
    return float(np.abs(x - ref).max()) / (den if den > 0 else 1.0)


def assert_parity(gpu: dict, ref: dict, heads=None, out_tol=OUT_TOL, state_tol=STATE_TOL, rows=None):
    g_out = gpu["out"] if heads is None else gpu["out"][:, heads]
    g_rs = gpu["rec_state"] if heads is None else gpu["rec_state"][:, heads]
    r_out = ref["out"]
    if rows is not None:
        g_out, r_out = g_out[rows], r_out[rows]
    eo = rel_err(g_out, r_out)
    es = rel_err(g_rs, ref["rec_state"])
    print("parity: out rel err %.3e (tol %.0e), state rel err %.3e (tol %.0e)" % (eo, out_tol, es, state_tol))
    assert np.isfinite(g_out).all() and np.isfinite(g_rs).all()
    assert eo <= out_tol, "out rel err %.3e > %.1e" % (eo, out_tol)
    assert es <= state_tol, "state rel err %.3e > %.1e" % (es, state_tol)
    return eo, es


def conv_state_bits(case, cs_t: torch.Tensor) -> np.ndarray:
    if case.bf16:
        return cs_t.view(torch.int16).cpu().numpy().view(np.uint16)
    return cs_t.cpu().numpy()


def expected_conv_state(case, acts, conv_state, cu) -> np.ndarray:
    """The last 3 raw inputs of each sequence (bit patterns), continuing the old state."""
    x = np.concatenate([acts["q"], acts["k"], acts["v"]], axis=1)
    out = np.empty_like(conv_state)
    for s in range(len(cu) - 1):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        hist = np.concatenate([conv_state[s].T, x[t0:t1]], axis=0)[-3:]
        out[s] = hist.T
    return out


def decode_steps(c, steps, dev="cuda:0", snapshots=False):
    """gdn_decode once per step; returns (outs, conv_state, rec_state[, state and conv
    state after every step])."""
    cfg = config_of(c)
    w = weights_on(c, dev)
    cs = t_act(c.conv_state, dev)
    rs = torch.from_numpy(c.rec_state).to(dev)
    outs, snaps, csnaps = [], [], []
    for st in steps:
        d = {n: t_act(st[n], dev) for n in "qkvabz"}
        o = gdn.decode(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs)
        outs.append(to_f64(o).reshape(-1, c.n_v_heads, c.d_v))
        if snapshots:
            snaps.append(rs.clone())
            csnaps.append(cs.clone())
    gdn.check_device_error()
    if snapshots:
        return outs, cs, rs, snaps, csnaps
    return outs, cs, to_f64(rs)


def as_sequences(c, steps, seqs):
    """Per-step one-token inputs of the chosen sequences, packed token-major within each
    sequence (one prefill of len(steps) tokens per sequence; the multi-token decode layout)."""
    n = len(steps)
    acts = {k: np.concatenate([np.stack([st[k][s] for st in steps]) for s in seqs]) for k in "qkvabz"}
    cu = np.arange(0, n * len(seqs) + 1, n, dtype=np.int32)
    return acts, cu
