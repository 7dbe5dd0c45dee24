"""Host logic of context-parallel prefill (hybrid_linear_attention_mixer_b200.cp) on
2 and 3 gloo ranks on the CPU.

The two phases run as fp64 oracle stand-ins (segment maps, fold, per-segment
forward), so what is under test is the rank-to-rank plumbing: segment lengths,
the conv halo passed to the next rank, the rank order of the gathered maps, and
the final states on the last rank.  The result must equal one oracle run over
the whole sequence.
"""
import os
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

SHAPE = oracle.Shape(1, 2, 4, 4)


def _case(T, seed=3):
    rng = np.random.default_rng(seed)
    C = SHAPE.channels
    w = {"conv_w": rng.normal(0, 0.7, (C, 4)), "A_log": rng.uniform(-2, -1, 2),
         "dt_bias": rng.normal(0, 0.3, 2), "norm_w": rng.normal(1, 0.2, 4)}
    acts = {"q": rng.normal(size=(T, 4)), "k": rng.normal(size=(T, 4)), "v": rng.normal(size=(T, 8)),
            "z": rng.normal(size=(T, 8)), "a": rng.normal(size=(T, 2)), "b": rng.normal(size=(T, 2))}
    cs = rng.normal(size=(C, 3))
    rs = rng.normal(0, 0.5, (2, 4, 4))
    return w, acts, cs, rs


class OracleOps:
    """gdn_cp_local / gdn_cp_finish semantics, computed by the fp64 oracle."""

    def __init__(self, w):
        self.w = w

    def local(self, cfg, w, q, k, v, a, b, cs):
        P, S_loc = oracle.segment_map(SHAPE, self.w, q.numpy(), k.numpy(), v.numpy(), a.numpy(), b.numpy(),
                                      cs.numpy())
        ws = {"acts": (q, k, v, a, b), "cs_in": cs.clone()}
        cs.copy_(torch.cat([q[-3:], k[-3:], v[-3:]], dim=1).t())     # conv state after the segment
        return torch.from_numpy(np.stack([P, S_loc])), ws

    def finish(self, cfg, w, z, summaries, rank, state_in, ws):
        maps = [(summaries[j, 0].numpy(), summaries[j, 1].numpy()) for j in range(rank)]
        S0 = oracle.fold_segment_maps(state_in.numpy(), maps)
        q, k, v, a, b = (x.numpy() for x in ws["acts"])
        T = q.shape[0]
        r = oracle.forward(SHAPE, self.w, q, k, v, a, b, z.numpy(), ws["cs_in"].numpy()[None], S0[None],
                           np.array([0, T], np.int32))
        return torch.from_numpy(r["out"].reshape(T, -1)), torch.from_numpy(r["rec_state"][0])


def _rank_main(rank, world, port, cuts, outdir, T):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from hybrid_linear_attention_mixer_b200 import cp
        w, acts, cs, rs = _case(T)
        lo, hi = cuts[rank], cuts[rank + 1]
        seg = {n: torch.from_numpy(np.ascontiguousarray(x[lo:hi])) for n, x in acts.items()}
        try:
            out, state, cs_end = cp.prefill(None, None, seg["q"], seg["k"], seg["v"], seg["a"], seg["b"], seg["z"],
                                            torch.from_numpy(cs), torch.from_numpy(rs), ops=OracleOps(w))
            np.savez(os.path.join(outdir, "r%d.npz" % rank), out=out.numpy(), state=state.numpy(),
                     cs=cs_end.numpy())
        except ValueError as e:
            with open(os.path.join(outdir, "r%d.err" % rank), "w") as f:
                f.write(str(e))
    finally:
        dist.destroy_process_group()


def _run(cuts, T):
    world = len(cuts) - 1
    with tempfile.TemporaryDirectory() as d:
        port = 29500 + (os.getpid() % 2000) + 7 * world
        mp.start_processes(_rank_main, args=(world, port, cuts, d, T), nprocs=world, start_method="spawn",
                           join=True)
        return [dict(np.load(os.path.join(d, "r%d.npz" % r))) if os.path.exists(os.path.join(d, "r%d.npz" % r))
                else open(os.path.join(d, "r%d.err" % r)).read() for r in range(world)]


@pytest.mark.parametrize("cuts", [[0, 6, 13], [0, 4, 9, 13]])
def test_cp_prefill_equals_one_run(cuts):
    T = cuts[-1]
    res = _run(cuts, T)
    w, acts, cs, rs = _case(T)
    ref = oracle.forward(SHAPE, w, *[acts[n] for n in "qkvabz"], cs[None], rs[None], np.array([0, T], np.int32))
    out = np.concatenate([r["out"] for r in res], axis=0)
    np.testing.assert_allclose(out, ref["out"].reshape(T, -1), rtol=0, atol=1e-10)
    np.testing.assert_allclose(res[-1]["state"], ref["rec_state"][0], rtol=0, atol=1e-10)
    np.testing.assert_array_equal(res[-1]["cs"], ref["conv_state"][0])
    # every rank's state is the state after its own segment
    for r, hi in enumerate(cuts[1:-1]):
        part = oracle.forward(SHAPE, w, *[acts[n][:hi] for n in "qkvabz"], cs[None], rs[None],
                              np.array([0, hi], np.int32))
        np.testing.assert_allclose(res[r]["state"], part["rec_state"][0], rtol=0, atol=1e-10)


def test_cp_prefill_short_segment_fails_on_every_rank():
    res = _run([0, 2, 9], 9)        # rank 0 holds 2 rows < K-1 = 3
    assert all(isinstance(r, str) and "at least 3 rows" in r for r in res)
