"""A prefill pipelined over chunk ranges (gdn_config.prefill_segments).

The conv and intra-chunk kernels of each range run on the caller's stream while
the state chain walks the ranges before it on another stream; each chain's fp32
state passes from one range's scan launch to the next through the workspace.
No arithmetic changes with the ranges, so every range count must give the same
bits as the call run in one piece, and match the oracle.

A partial last chunk of a sequence reads, through its 64-row tile loads, rows
past the sequence's end: another sequence's tokens, which the next range's conv
may not have written yet.  Those rows are zeroed in shared memory before use; a
workspace filled with NaN before the call shows any read of a row that no conv
has written.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _problem(lens, seed, state_dtype=torch.float32):
    c = inputs.make_case("prefill_4k", T=sum(lens), seed=seed)
    c.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    N = len(lens)
    c.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(N, c.channels, 3)).astype(np.float32))
    c.rec_state = (0.05 * rng.normal(size=(N, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)
    d = {n: L.t_act(c.acts[n], DEV) for n in "qkvabz"}
    rs0 = torch.from_numpy(c.rec_state).to(DEV)
    if state_dtype == torch.bfloat16:
        rs0 = rs0.to(torch.bfloat16)
    return c, d, L.t_act(c.conv_state, DEV), rs0, torch.from_numpy(c.cu_seqlens).to(DEV)


def _run(c, d, cs0, rs0, cu, segments, state_dtype=torch.float32, poison=False):
    cfg = L.config_of(c)
    cfg.prefill_segments = segments
    cfg.state_dtype = state_dtype
    w = L.weights_on(c, DEV)
    cs, rs = cs0.clone(), rs0.clone()
    ws = torch.empty(gdn.workspace_size(cfg, c.T, len(c.cu_seqlens) - 1), dtype=torch.uint8, device=DEV)
    ws.fill_(0xFF if poison else 0)   # 0xffff is a NaN in fp16 and in fp32
    out = gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu, workspace=ws)
    torch.cuda.synchronize()
    gdn.check_device_error()
    return out, cs, rs


@pytest.mark.parametrize("state_dtype", [torch.float32, torch.bfloat16])
def test_range_counts_give_the_same_bits_as_one_piece(state_dtype):
    c, d, cs0, rs0, cu = _problem([4096], 81, state_dtype)
    ref = _run(c, d, cs0, rs0, cu, 1, state_dtype)
    for segments in (0, 2, 3, 7, 32):
        got = _run(c, d, cs0, rs0, cu, segments, state_dtype, poison=True)
        for x, y in zip(got, ref):
            assert torch.equal(x, y), segments
    if state_dtype == torch.float32:
        heads = [0, 17, 47]
        g = {"out": L.to_f64(ref[0]).reshape(c.T, c.n_v_heads, c.d_v), "rec_state": L.to_f64(ref[2])}
        L.assert_parity(g, L.oracle_run(c, heads=heads), heads=heads)


# The first sequence ends 10 tokens into its 16th chunk, right where the 2-range
# plan of 2,048 tokens in 2 ranges (32 chunks, ranges of 16) cuts: that chunk's tile loads
# reach rows 992..1023, which only the second range's conv writes.
# The last case packs 20 one-chunk sequences of 40 tokens before a long one, so that every
# range boundary among the first 20 chunks falls right after a partial chunk.
@pytest.mark.parametrize("lens,segments", [([970, 1078], 2), ([100, 1, 1500, 63, 384], 5),
                                           ([0, 2048, 0], 3), ([40] * 20 + [1000], 7)])
def test_partial_chunks_at_range_boundaries(lens, segments):
    c, d, cs0, rs0, cu = _problem(lens, 83 + len(lens))
    ref = _run(c, d, cs0, rs0, cu, 1)
    got = _run(c, d, cs0, rs0, cu, segments, poison=True)
    for x, y in zip(got, ref):
        assert torch.equal(x, y)
    heads = [5, 40]
    g = {"out": L.to_f64(got[0]).reshape(c.T, c.n_v_heads, c.d_v), "rec_state": L.to_f64(got[2])}
    L.assert_parity(g, L.oracle_run(c, heads=heads), heads=heads)
