"""A prefill whose state chain is split in two (gdn_config.prefill_segments =
GDN_PREFILL_SPLIT, for one sequence).

The first half of the chunks runs from the real start state while the second
half runs, at the same time, from a zero state and as its transition map from
the identity; the second half's outputs are then corrected with the first
half's end state on the tensor cores (bf16 operands) and its end state folded
in fp32.  The arithmetic differs from one range's, so the results are checked
against the oracle (all heads) and against the one-range call within the
layer's tolerances, never bit for bit.  Workspaces are filled with NaN first,
so that any read of an element no kernel wrote shows.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SPLIT = -1


def _problem(T, seed, s0_scale):
    c = inputs.make_case("prefill_4k", T=T, seed=seed)
    rng = np.random.default_rng(seed)
    if s0_scale:
        c.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(1, c.channels, 3)).astype(np.float32))
        c.rec_state = (s0_scale * rng.normal(size=(1, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)
    return c


def _run(c, segments, poison=True):
    cfg = L.config_of(c)
    cfg.prefill_segments = segments
    w = L.weights_on(c, DEV)
    d = {n: L.t_act(c.acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(np.ascontiguousarray(c.rec_state)).to(DEV)
    cu = torch.from_numpy(c.cu_seqlens).to(DEV)
    ws = torch.empty(gdn.workspace_size(cfg, c.T, 1), dtype=torch.uint8, device=DEV)
    ws.fill_(0xFF if poison else 0)
    out = gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu, workspace=ws)
    torch.cuda.synchronize()
    gdn.check_device_error()
    return out, cs, rs


# 4096 tokens: 64 chunks, halves of 32.  4106: 65 chunks, a second half of 33 (an odd count,
# so the last correction CTA has one chunk) whose last chunk holds 10 tokens.
@pytest.mark.parametrize("T,seed,s0", [(4096, 91, 0.0), (4096, 92, 0.05), (4106, 93, 0.05)])
def test_split_chain_matches_the_oracle_and_one_range(T, seed, s0):
    c = _problem(T, seed, s0)
    cfg = L.config_of(c)
    cfg.prefill_segments = SPLIT
    assert gdn.prefill_segments(cfg, T, 1) == SPLIT
    out, cs, rs = _run(c, SPLIT)
    r = L.oracle_run(c, threads=16)
    g = {"out": L.to_f64(out).reshape(T, c.n_v_heads, c.d_v), "rec_state": L.to_f64(rs)}
    L.assert_parity(g, r)
    np.testing.assert_array_equal(L.conv_state_bits(c, cs), L.expected_conv_state(c, c.acts, c.conv_state,
                                                                                   c.cu_seqlens))
    one = _run(c, 1, poison=False)
    assert L.rel_err(L.to_f64(out), L.to_f64(one[0])) <= 1e-2
    assert L.rel_err(L.to_f64(rs), L.to_f64(one[2])) <= 1e-3
    assert torch.equal(cs, one[1])


def test_split_chain_device_checks_write_nothing():
    c = _problem(4096, 94, 0.05)
    cfg = L.config_of(c)
    cfg.prefill_segments = SPLIT
    w = L.weights_on(c, DEV)
    acts = dict(c.acts)
    v = inputs.bf16_bits_to_f32(acts["v"]).copy()
    v[4000:4010] = 3.0e6      # in the second half: the conv of these rows leaves the fp16 range
    acts["v"] = inputs.f32_to_bf16_bits(v)
    d = {n: L.t_act(acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(np.ascontiguousarray(c.rec_state)).to(DEV)
    out = torch.full((c.T, c.n_v_heads * c.d_v), 7.0, dtype=torch.bfloat16, device=DEV)
    before = (out.clone(), cs.clone(), rs.clone())
    for cu in (np.array([0, c.T], np.int32), np.array([0, c.T - 1], np.int32)):   # range error; cu[N] != T
        cu_t = torch.from_numpy(cu).to(DEV)
        gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu_t, out=out)
        import ctypes
        s = gdn.lib().gdn_check_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert s in (6, 7), gdn.status_string(s)
        for x, y in zip((out, cs, rs), before):
            assert torch.equal(x, y)


def test_split_chain_in_a_cuda_graph():
    c = _problem(4096, 95, 0.05)
    cfg = L.config_of(c)
    cfg.prefill_segments = SPLIT
    w = L.weights_on(c, DEV)
    d = {n: L.t_act(c.acts[n], DEV) for n in "qkvabz"}
    cs0 = L.t_act(c.conv_state, DEV)
    rs0 = torch.from_numpy(np.ascontiguousarray(c.rec_state)).to(DEV)
    cu = torch.from_numpy(c.cu_seqlens).to(DEV)
    ws = torch.empty(gdn.workspace_size(cfg, c.T, 1), dtype=torch.uint8, device=DEV)
    out = torch.empty((c.T, c.n_v_heads * c.d_v), dtype=torch.bfloat16, device=DEV)
    cs, rs = cs0.clone(), rs0.clone()

    def run():
        gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu, out=out, workspace=ws)

    run()
    torch.cuda.synchronize()
    gdn.check_device_error()
    ref = (out.clone(), cs.clone(), rs.clone())
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run()
    for _ in range(2):
        cs.copy_(cs0)
        rs.copy_(rs0)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        gdn.check_device_error()
        assert torch.equal(out, ref[0]) and torch.equal(cs, ref[1]) and torch.equal(rs, ref[2])
    del g
