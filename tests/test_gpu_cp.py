"""Context-parallel prefill kernels (gdn_cp_local, gdn_cp_finish) on one GPU.

The ranks are emulated one after another in this process: every segment's phase
1 runs, the summaries are stacked in rank order, then every segment's phase 2
runs.  Nothing waits on another launch, so one GPU serves all ranks.  Nonzero
initial states and slowly decaying gates make the state carried across each cut
matter: the 256K workload's -log alpha ~ U(1e-4, 0.1), and a slower U(1e-4, 1e-2)
under which a segment's transition P stays of order 0.1 over hundreds of tokens.
Checks, at the layer's parity bars:
* each segment's (P, S_loc) against the oracle's segment map: relative to max|P|
  where P is large enough to act on the state (max|P| >= 1e-2), else to within
  1e-5 absolute (a transition that small is lost under the state's own bar);
* the concatenated outputs and every rank's end state against one oracle run over
  the whole sequence (and its prefixes).
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
import oracle
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(T, seed=8, nla_range=None):
    c = inputs.make_case("prefill_256k", T=T, seed=seed, nla_range=nla_range)
    rng = np.random.default_rng(seed)
    c.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(1, c.channels, 3)).astype(np.float32))
    c.rec_state = (0.05 * rng.normal(size=(1, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)
    return c


def _run_cp(c, cuts):
    cfg = L.config_of(c)
    w = L.weights_on(c, DEV)
    x = np.concatenate([c.acts["q"], c.acts["k"], c.acts["v"]], axis=1)
    summaries, wss, conv_in = [], [], []
    for r in range(len(cuts) - 1):
        lo, hi = cuts[r], cuts[r + 1]
        cs = c.conv_state[0] if r == 0 else np.ascontiguousarray(x[lo - 3:lo].T)
        conv_in.append(cs)
        d = {n: L.t_act(np.ascontiguousarray(c.acts[n][lo:hi]), DEV) for n in "qkvab"}
        summary, ws = gdn.cp_local(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], L.t_act(cs, DEV))
        summaries.append(summary)
        wss.append(ws)
    S = torch.stack(summaries)
    rs0 = torch.from_numpy(c.rec_state[0]).to(DEV)
    outs, states = [], []
    for r in range(len(cuts) - 1):
        lo, hi = cuts[r], cuts[r + 1]
        out, st = gdn.cp_finish(cfg, w, L.t_act(np.ascontiguousarray(c.acts["z"][lo:hi]), DEV), S, r, rs0, wss[r])
        outs.append(L.to_f64(out))
        states.append(L.to_f64(st))
    gdn.check_device_error()
    return S, conv_in, outs, states


@pytest.mark.parametrize("cuts,nla", [([0, 700, 1303, 2000], None), ([0, 3, 67, 131, 400], None),
                                      ([0, 500], None), ([0, 260, 333, 900], (1e-4, 1e-2))])
def test_cp_matches_one_oracle_run(cuts, nla):
    T = cuts[-1]
    c = _case(T, nla_range=nla)
    S, conv_in, outs, states = _run_cp(c, cuts)
    shape = L.shape_of(c)
    errs = []
    # each segment's affine map
    for r in range(len(cuts) - 1):
        lo, hi = cuts[r], cuts[r + 1]
        P, S_loc = oracle.segment_map(shape, c.weights, *[c.acts[n][lo:hi] for n in "qkvab"], conv_in[r])
        pmax = float(np.abs(P).max())
        dP = float(np.abs(L.to_f64(S[r, 0]) - P).max())
        eS = L.rel_err(L.to_f64(S[r, 1]), S_loc)
        print("segment %d [%d, %d): max|P| %.2e, P err %.2e abs (%.2e rel), S_loc err %.2e"
              % (r, lo, hi, pmax, dP, dP / max(pmax, 1e-300), eS))
        errs.append(dP <= (L.STATE_TOL * pmax if pmax >= 1e-2 else 1e-5) and eS <= L.STATE_TOL)
    ref = L.oracle_run(c)
    out = np.concatenate(outs, axis=0).reshape(T, c.n_v_heads, c.d_v)
    eo = L.rel_err(out, ref["out"])
    es = L.rel_err(states[-1], ref["rec_state"][0])
    print("cp over %d ranks: out err %.2e, final state err %.2e" % (len(cuts) - 1, eo, es))
    for r, hi in enumerate(cuts[1:-1]):
        part = L.oracle_run(c, acts={n: x[:hi] for n, x in c.acts.items()}, cu=np.array([0, hi], np.int32))
        e = L.rel_err(states[r], part["rec_state"][0])
        print("  state after rank %d: err %.2e" % (r, e))
        errs.append(e <= L.STATE_TOL)
    assert all(errs) and eo <= L.OUT_TOL and es <= L.STATE_TOL


def test_cp_single_rank_equals_prefill():
    """One rank: the context-parallel path runs the same scan as gdn_prefill from the
    same state, so outputs and state agree to the scan's own rounding."""
    c = _case(300, seed=9)
    _, _, outs, states = _run_cp(c, [0, 300])
    g = L.gpu_prefill(c)
    assert L.rel_err(outs[0].reshape(300, c.n_v_heads, c.d_v), g["out"]) <= 1e-6
    assert L.rel_err(states[0], g["rec_state"][0]) <= 1e-6
