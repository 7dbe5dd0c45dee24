"""gdn_decode_multi: n_tok consecutive tokens per sequence in one pass over each
state (checking tokens that a multi-token-prediction head drafted).

* It equals n_tok consecutive gdn_decode calls: the conv states and their
  snapshots bit for bit, outputs and recurrent states (final and per token) up
  to the order of fp32 additions inside a state row's dot products.
* It matches the fp64 oracle run over the same tokens as one prefill per sequence,
  and every state snapshot matches the oracle run over that prefix of the tokens.
* The largest n_tok at the small head shape with fp32 activations, and at the
  published shape, whose 16-token buffers exceed the streamed kernel's shared
  memory (the call takes the register-streaming multi-token kernel instead).
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _multi(c, steps, n_tok, snapshots=True, out_dtype=None):
    cfg = L.config_of(c, out_dtype=out_dtype)
    w = L.weights_on(c, DEV)
    seqs = list(range(c.n_seqs))
    acts, _ = L.as_sequences(c, steps, seqs)
    d = {n: L.t_act(acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(c.rec_state).to(DEV)
    snap = csnap = None
    if snapshots:
        snap = torch.full((n_tok,) + tuple(rs.shape), float("nan"), device=DEV)
        csnap = torch.zeros((n_tok,) + tuple(cs.shape), dtype=cs.dtype, device=DEV)
    out = gdn.decode_multi(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, n_tok,
                           state_snapshots=snap, conv_snapshots=csnap)
    gdn.check_device_error()
    return out, cs, rs, snap, csnap


def _decode_steps_f32(c, steps):
    """gdn_decode once per step with fp32 outputs, keeping the states after every step."""
    cfg = L.config_of(c, out_dtype=torch.float32)
    w = L.weights_on(c, DEV)
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(c.rec_state).to(DEV)
    outs, snaps, csnaps = [], [], []
    for st in steps:
        d = {n: L.t_act(st[n], DEV) for n in "qkvabz"}
        outs.append(gdn.decode(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs).clone())
        snaps.append(rs.clone())
        csnaps.append(cs.clone())
    gdn.check_device_error()
    return outs, cs, rs, snaps, csnaps


@pytest.mark.parametrize("n_tok", [1, 4, 7, 16])
def test_decode_multi_equals_decode_steps(n_tok):
    c = inputs.make_case("decode_256", T=n_tok, n_seqs=64)
    outs, cs1, rs1, snaps, csnaps = _decode_steps_f32(c, c.steps)
    out, cs2, rs2, snap, csnap = _multi(c, c.steps, n_tok, out_dtype=torch.float32)
    go = L.to_f64(out).reshape(c.n_seqs, n_tok, -1)
    ro = np.stack([L.to_f64(o) for o in outs], axis=1)
    # fp32 additions in another order: a few units in the last place, compounded over the tokens
    assert L.rel_err(go, ro) <= 1e-5
    assert L.rel_err(L.to_f64(rs2), L.to_f64(rs1)) <= 1e-5
    assert torch.equal(cs2, cs1)
    for t in range(n_tok):
        assert L.rel_err(L.to_f64(snap[t]), L.to_f64(snaps[t])) <= 1e-5
        assert torch.equal(csnap[t], csnaps[t])


def test_decode_multi_oracle_and_snapshots():
    """5 drafted tokens for 6 sequences with nonzero states, all heads; each snapshot
    against the oracle over the first t tokens."""
    n_tok = 5
    c = inputs.make_case("decode_256", T=n_tok, n_seqs=6)
    out, cs, rs, snap, _ = _multi(c, c.steps, n_tok)
    seqs = list(range(c.n_seqs))
    acts, cu = L.as_sequences(c, c.steps, seqs)
    r = L.oracle_run(c, acts=acts, cu=cu)
    L.assert_parity({"out": L.to_f64(out).reshape(-1, c.n_v_heads, c.d_v), "rec_state": L.to_f64(rs)}, r)
    x = {k: acts[k].reshape(c.n_seqs, n_tok, -1) for k in "qkv"}
    expect = np.concatenate([c.conv_state[:, :, n_tok:],
                             np.concatenate([x["q"], x["k"], x["v"]], axis=2)[:, -3:].transpose(0, 2, 1)],
                            axis=2) if n_tok < 3 else \
        np.concatenate([x["q"], x["k"], x["v"]], axis=2)[:, -3:].transpose(0, 2, 1)
    np.testing.assert_array_equal(L.conv_state_bits(c, cs), expect)
    for t in range(1, n_tok + 1):
        pre, pcu = L.as_sequences(c, c.steps[:t], seqs)
        rt = L.oracle_run(c, acts=pre, cu=pcu)
        assert L.rel_err(L.to_f64(snap[t - 1]), rt["rec_state"]) <= L.STATE_TOL


def test_decode_multi_max_tokens_small_heads_fp32():
    """GDN_DECODE_MULTI_MAX_TOKENS tokens at 2 key / 6 value heads of 32, fp32 activations."""
    n_tok, N = gdn.DECODE_MULTI_MAX_TOKENS, 3
    c = inputs.make_case("tiny", T=n_tok * N)
    c.cu_seqlens = np.arange(0, n_tok * N + 1, n_tok, dtype=np.int32)
    c.conv_state = np.zeros((N, c.channels, 3), np.float32)
    c.rec_state = np.zeros((N, c.n_v_heads, c.d_v, c.d_k), np.float32)
    steps = [{k: c.acts[k].reshape(N, n_tok, -1)[:, t] for k in "qkvabz"} for t in range(n_tok)]
    out, cs, rs, _, _ = _multi(c, steps, n_tok, snapshots=False)
    r = L.oracle_run(c)
    L.assert_parity({"out": L.to_f64(out).reshape(-1, c.n_v_heads, c.d_v), "rec_state": L.to_f64(rs)}, r)
