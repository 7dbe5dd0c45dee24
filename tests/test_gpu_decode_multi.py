"""gdn_decode_multi: n_tok consecutive tokens per sequence in one pass over each
state (checking tokens that a multi-token-prediction head drafted).

* It equals n_tok consecutive gdn_decode calls bit for bit: outputs, final
  recurrent and conv states, and the per-token snapshots of both.
* It matches the fp64 oracle run over the same tokens as one prefill per sequence,
  and every state snapshot matches the oracle run over that prefix of the tokens.
* The largest n_tok at the small head shape with fp32 activations.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _multi(c, steps, n_tok, snapshots=True):
    cfg = L.config_of(c)
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


@pytest.mark.parametrize("n_tok", [1, 4, 7])
def test_decode_multi_bit_identical_to_decode_steps(n_tok):
    c = inputs.make_case("decode_256", T=n_tok, n_seqs=64)
    outs, cs1, rs1, snaps, csnaps = L.decode_steps(c, c.steps, snapshots=True)
    out, cs2, rs2, snap, csnap = _multi(c, c.steps, n_tok)
    go = L.to_f64(out).reshape(c.n_seqs, n_tok, c.n_v_heads, c.d_v)
    assert np.array_equal(go, np.stack(outs, axis=1))
    assert torch.equal(rs2, rs1)
    assert torch.equal(cs2, cs1)
    for t in range(n_tok):
        assert torch.equal(snap[t], snaps[t])
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
