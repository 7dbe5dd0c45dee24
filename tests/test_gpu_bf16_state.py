"""The recurrent state stored in bf16 (gdn_config.state_dtype = GDN_BF16).

The kernels read the stored state exactly, compute every step in fp32 as with an
fp32 state, and round what they store to bf16 (nearest even).  The reference is
the fp64 oracle with the same rounding points: the state is rounded to bf16
wherever a call stores it (after every gdn_decode step, at the end of a prefill
or multi-token call, and in each snapshot).  Both sides round at the same points
from values that differ by the fp32 path's own error, so a stored entry can land
one bf16 step (2^-8 of its size) apart, and such a step can be carried into the
next call: the state bar is two bf16 steps of max|S|, 2^-7.  The output bar and
the conv state (bit for bit) are those of the fp32 state.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
STATE_TOL_BF16 = 2.0 ** -7


def _round_bf16(x64: np.ndarray) -> np.ndarray:
    """fp64 state -> bf16 (via fp32, nearest even) -> fp64: the stored values."""
    return inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(x64.astype(np.float32))).astype(np.float64)


def _cfg(c, **kw):
    cfg = L.config_of(c, **kw)
    cfg.state_dtype = torch.bfloat16
    return cfg


def _state_bf16_on(c):
    bits = inputs.f32_to_bf16_bits(c.rec_state.astype(np.float32))
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(DEV), _round_bf16(c.rec_state)


def test_decode_steps_with_bf16_state():
    """4 decode steps at batch 32: the state is rounded to bf16 after every step."""
    c = inputs.make_case("decode_256", T=4, n_seqs=32)
    cfg, w = _cfg(c), L.weights_on(c, DEV)
    cs = L.t_act(c.conv_state, DEV)
    rs, ref_state = _state_bf16_on(c)
    ref_cs = c.conv_state
    seqs = list(range(c.n_seqs))
    for st in c.steps:
        d = {n: L.t_act(st[n], DEV) for n in "qkvabz"}
        out = gdn.decode(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs)
        acts, cu = L.as_sequences(c, [st], seqs)
        r = L.oracle_run(c, acts=acts, cu=cu, conv_state=ref_cs, rec_state=ref_state)
        ref_state = _round_bf16(r["rec_state"])
        ref_cs = np.concatenate([ref_cs[:, :, 1:],
                                 np.concatenate([st["q"], st["k"], st["v"]], axis=1)[:, :, None]], axis=2)
        assert L.rel_err(L.to_f64(out).reshape(-1, c.n_v_heads, c.d_v), r["out"]) <= L.OUT_TOL
        e = L.rel_err(L.to_f64(rs), ref_state)
        print("bf16 state decode step: state rel err %.3e (tol %.1e)" % (e, STATE_TOL_BF16))
        assert e <= STATE_TOL_BF16
    gdn.check_device_error()
    np.testing.assert_array_equal(L.conv_state_bits(c, cs), ref_cs)


def test_prefill_ragged_with_bf16_state():
    """Ragged varlen prefill from nonzero bf16 states: rounded once, at the end."""
    lens = [1, 63, 64, 65, 0, 130, 3, 200]
    base = inputs.make_case("prefill_4k", T=int(sum(lens)), seed=5)
    base.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(5)
    N = len(lens)
    base.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(N, base.channels, 3)).astype(np.float32))
    base.rec_state = _round_bf16(0.05 * rng.normal(size=(N, base.n_v_heads, base.d_v, base.d_k))).astype(np.float32)
    cfg, w = _cfg(base), L.weights_on(base, DEV)
    d = {n: L.t_act(base.acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(base.conv_state, DEV)
    rs, _ = _state_bf16_on(base)
    cu = torch.from_numpy(base.cu_seqlens).to(DEV)
    out = gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu)
    gdn.check_device_error()
    r = L.oracle_run(base)
    assert L.rel_err(L.to_f64(out).reshape(-1, base.n_v_heads, base.d_v), r["out"]) <= L.OUT_TOL
    e = L.rel_err(L.to_f64(rs), _round_bf16(r["rec_state"]))
    print("bf16 state prefill: state rel err %.3e (tol %.1e)" % (e, STATE_TOL_BF16))
    assert e <= STATE_TOL_BF16
    # the empty sequence keeps its stored state bit for bit
    assert torch.equal(rs[4].cpu(), _state_bf16_on(base)[0][4].cpu())


def test_decode_multi_with_bf16_state_and_snapshots():
    """4 drafted tokens for 8 sequences: the state is rounded at the end of the call and in
    each snapshot."""
    n_tok = 4
    c = inputs.make_case("decode_256", T=n_tok, n_seqs=8)
    cfg, w = _cfg(c), L.weights_on(c, DEV)
    seqs = list(range(c.n_seqs))
    acts, cu = L.as_sequences(c, c.steps, seqs)
    d = {n: L.t_act(acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(c.conv_state, DEV)
    rs, ref0 = _state_bf16_on(c)
    snap = torch.zeros((n_tok,) + tuple(rs.shape), dtype=torch.bfloat16, device=DEV)
    out = gdn.decode_multi(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, n_tok,
                           state_snapshots=snap)
    gdn.check_device_error()
    r = L.oracle_run(c, acts=acts, cu=cu, rec_state=ref0)
    assert L.rel_err(L.to_f64(out).reshape(-1, c.n_v_heads, c.d_v), r["out"]) <= L.OUT_TOL
    assert L.rel_err(L.to_f64(rs), _round_bf16(r["rec_state"])) <= STATE_TOL_BF16
    for t in range(1, n_tok + 1):
        pre, pcu = L.as_sequences(c, c.steps[:t], seqs)
        rt = L.oracle_run(c, acts=pre, cu=pcu, rec_state=ref0)
        assert L.rel_err(L.to_f64(snap[t - 1]), _round_bf16(rt["rec_state"])) <= STATE_TOL_BF16
