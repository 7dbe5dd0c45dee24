"""The library's calls inside a CUDA graph.

gdn_prefill forks two small kernels onto an internal side stream and joins them
back with events, and gdn_cp_local runs its second scan on another; under stream
capture those forks become graph branches.  A captured prefill + decode step,
replayed, must give exactly what the same calls give when run directly from the
same starting states.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_prefill_and_decode_replay_from_a_graph():
    lens = [300, 0, 129]
    c = inputs.make_case("prefill_4k", T=sum(lens), seed=17)
    c.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cfg, w = L.config_of(c), L.weights_on(c, DEV)
    N = len(lens)
    rng = np.random.default_rng(17)
    cs0 = L.t_act(inputs.f32_to_bf16_bits(rng.normal(size=(N, c.channels, 3)).astype(np.float32)), DEV)
    rs0 = torch.from_numpy((0.05 * rng.normal(size=(N, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)).to(DEV)
    d = {n: L.t_act(c.acts[n], DEV) for n in "qkvabz"}
    step = {n: L.t_act(rng.normal(size=(N,) + c.acts[n].shape[1:]).astype(np.float32), DEV).to(torch.bfloat16)
            for n in "qkvabz"}
    cu = torch.from_numpy(c.cu_seqlens).to(DEV)
    ws = torch.empty(gdn.workspace_size(cfg, c.T, N), dtype=torch.uint8, device=DEV)
    out = torch.empty((c.T, c.n_v_heads * c.d_v), dtype=torch.bfloat16, device=DEV)
    dout = torch.empty((N, c.n_v_heads * c.d_v), dtype=torch.bfloat16, device=DEV)
    cs, rs = cs0.clone(), rs0.clone()

    def run():
        gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu, out=out, workspace=ws)
        gdn.decode(cfg, w, step["q"], step["k"], step["v"], step["a"], step["b"], step["z"], cs, rs, out=dout)

    run()                                   # eager (also sets up the library's streams and opt-ins)
    torch.cuda.synchronize()
    gdn.check_device_error()
    ref = (out.clone(), dout.clone(), cs.clone(), rs.clone())
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run()
    for _ in range(2):                      # replay twice from the same starting states
        cs.copy_(cs0)
        rs.copy_(rs0)
        out.zero_()
        dout.zero_()
        g.replay()
        torch.cuda.synchronize()
        gdn.check_device_error()
        assert torch.equal(out, ref[0]) and torch.equal(dout, ref[1])
        assert torch.equal(cs, ref[2]) and torch.equal(rs, ref[3])
    del g
