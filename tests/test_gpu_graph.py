"""The library's calls inside a CUDA graph.

gdn_prefill forks work onto internal side streams and joins it back with events
(the conv-state update; when pipelined over chunk ranges, the scans and the
norms too), and gdn_cp_local runs its second scan on another; under stream
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


@pytest.mark.parametrize("segments", [1, 3])   # 3: the prefill pipelined over three streams
def test_prefill_and_decode_replay_from_a_graph(segments):
    lens = [300, 0, 129]
    c = inputs.make_case("prefill_4k", T=sum(lens), seed=17)
    c.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cfg, w = L.config_of(c), L.weights_on(c, DEV)
    cfg.prefill_segments = segments
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


def test_capture_in_one_thread_beside_direct_calls_in_another():
    """One thread captures a prefill into a graph while another thread makes direct
    prefill calls on its own stream.  The side streams that a prefill forks onto
    belong to the calling thread, so neither call waits on, or is recorded into,
    the other thread's work: both give the results of the same calls run alone."""
    import threading

    def problem(seed, lens):
        c = inputs.make_case("prefill_4k", T=sum(lens), seed=seed)
        c.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        rng = np.random.default_rng(seed)
        N = len(lens)
        p = {"c": c, "cfg": L.config_of(c), "w": L.weights_on(c, DEV),
             "d": {n: L.t_act(c.acts[n], DEV) for n in "qkvabz"},
             "cu": torch.from_numpy(c.cu_seqlens).to(DEV),
             "cs0": L.t_act(inputs.f32_to_bf16_bits(rng.normal(size=(N, c.channels, 3)).astype(np.float32)), DEV),
             "rs0": torch.from_numpy((0.05 * rng.normal(size=(N, c.n_v_heads, c.d_v, c.d_k)))
                                     .astype(np.float32)).to(DEV),
             "ws": torch.empty(gdn.workspace_size(L.config_of(c), c.T, N), dtype=torch.uint8, device=DEV),
             "out": torch.empty((c.T, c.n_v_heads * c.d_v), dtype=torch.bfloat16, device=DEV)}
        p["cs"], p["rs"] = p["cs0"].clone(), p["rs0"].clone()
        return p

    def call(p, stream):
        d = p["d"]
        gdn.prefill(p["cfg"], p["w"], d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], p["cs"], p["rs"], p["cu"],
                    out=p["out"], workspace=p["ws"], stream=stream)

    def reset(p):
        p["cs"].copy_(p["cs0"])
        p["rs"].copy_(p["rs0"])
        p["out"].zero_()

    A, B = problem(23, [200, 77]), problem(29, [130, 0, 260])
    refs = {}
    for name, p in (("A", A), ("B", B)):    # each alone, eagerly
        call(p, torch.cuda.current_stream())
        torch.cuda.synchronize()
        gdn.check_device_error()
        refs[name] = (p["out"].clone(), p["cs"].clone(), p["rs"].clone())
        reset(p)
    torch.cuda.synchronize()

    start = threading.Barrier(2)
    errors, b_results = [], []
    g = torch.cuda.CUDAGraph()
    sa = torch.cuda.Stream()

    def thread_a():
        try:
            with torch.cuda.stream(sa):
                call(A, sa)                 # this thread's side streams and events exist before capture
                sa.synchronize()
                reset(A)
                sa.synchronize()
                start.wait()
                with torch.cuda.graph(g, stream=sa, capture_error_mode="thread_local"):
                    call(A, sa)
        except Exception as e:              # reported below
            errors.append(e)
            start.abort()

    def thread_b():
        try:
            sb = torch.cuda.Stream()
            with torch.cuda.stream(sb):
                call(B, sb)
                sb.synchronize()
                start.wait()
                for _ in range(3):          # direct calls while A captures
                    reset(B)
                    call(B, sb)
                sb.synchronize()
                b_results.append((B["out"].clone(), B["cs"].clone(), B["rs"].clone()))
        except Exception as e:
            errors.append(e)
            start.abort()

    ta, tb = threading.Thread(target=thread_a), threading.Thread(target=thread_b)
    ta.start()
    tb.start()
    ta.join()
    tb.join()
    assert not errors, errors
    torch.cuda.synchronize()
    gdn.check_device_error()
    for got, ref in zip(b_results[0], refs["B"]):
        assert torch.equal(got, ref)
    reset(A)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    gdn.check_device_error()
    for got, ref in zip((A["out"], A["cs"], A["rs"]), refs["A"]):
        assert torch.equal(got, ref)
    del g
