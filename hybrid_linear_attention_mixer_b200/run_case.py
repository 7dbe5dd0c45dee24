"""Run one synthetic workload through the public API (no timing, no oracle).

    python -m hybrid_linear_attention_mixer_b200.run_case --case prefill_4k --iters 2
    python -m hybrid_linear_attention_mixer_b200.run_case --case prefill_256k --tokens 16384 --segments 1
    python -m hybrid_linear_attention_mixer_b200.run_case --case decode_256 --batch 64 --iters 3
    python -m hybrid_linear_attention_mixer_b200.run_case --proj --tokens 4096 --iters 1
    python -m hybrid_linear_attention_mixer_b200.run_case --case decode_256 --batch 64 --multi 4 --state bf16

A small, fixed-size target for profilers such as ncu: it builds the seeded
inputs of the named workload, runs the layer `iters` times on cuda:0 and checks
the device error word.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from hybrid_linear_attention_mixer_b200 import gdn, inputs


def _act(x, dev):
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(x).to(dev)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", default="prefill_4k", choices=inputs.CASES)
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--tokens", type=int, default=None, help="shrink a prefill workload to T tokens")
    ap.add_argument("--batch", type=int, default=None, help="decode batch (sequences)")
    ap.add_argument("--multi", type=int, default=0,
                    help="decode: this many consecutive tokens per sequence in one gdn_decode_multi call")
    ap.add_argument("--state", default="fp32", choices=("fp32", "bf16"), help="recurrent state storage")
    ap.add_argument("--segments", type=int, default=0,
                    help="prefill: chunk ranges the call is pipelined over (0: automatic, 1: one piece)")
    ap.add_argument("--proj", action="store_true",
                    help="run the input and output projections (hidden 2560) at --tokens instead")
    args = ap.parse_args()
    dev = torch.device("cuda:0")
    if args.proj:
        T = args.tokens or 4096
        pc = inputs.make_proj_case(T)
        cfg = gdn.Config()
        hid, w_in, w_out, o = (_act(x, dev) for x in (pc.hidden, pc.w_in, pc.w_out, pc.o))
        for _ in range(args.iters):
            gdn.in_proj(cfg, hid, w_in)
            gdn.out_proj(cfg, o, w_out)
        gdn.check_device_error()
        torch.cuda.synchronize()
        print("ok proj T=%d" % T)
        return
    if args.case == "decode_256":
        c = inputs.make_case(args.case, n_seqs=args.batch, T=max(1, args.multi))
    else:
        c = inputs.make_case(args.case, T=args.tokens)
    act = torch.bfloat16 if c.bf16 else torch.float32
    cfg = gdn.Config(c.n_k_heads, c.n_v_heads, c.d_k, c.d_v, c.conv_kernel, 64, c.l2_eps, c.norm_eps,
                     act, act, torch.bfloat16 if args.state == "bf16" else torch.float32, args.segments)
    w = {n: torch.from_numpy(np.ascontiguousarray(c.weights[n])).to(dev)
         for n in ("conv_w", "A_log", "dt_bias", "norm_w")}
    d = {n: _act(c.acts[n], dev) for n in "qkvabz"}
    cs = _act(c.conv_state, dev)
    rs = torch.from_numpy(c.rec_state).to(dev).to(cfg.state_dtype)
    if args.case == "decode_256" and args.multi > 0:
        m = {n: _act(np.stack([st[n] for st in c.steps], axis=1).reshape(c.n_seqs * args.multi, -1), dev)
             for n in "qkvabz"}
    for _ in range(args.iters):
        if args.case == "decode_256" and args.multi > 0:
            gdn.decode_multi(cfg, w, m["q"], m["k"], m["v"], m["a"], m["b"], m["z"], cs, rs, args.multi)
        elif args.case == "decode_256":
            gdn.decode(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs)
        else:
            cu = torch.from_numpy(c.cu_seqlens).to(dev)
            gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu)
    gdn.check_device_error()
    torch.cuda.synchronize()
    print("ok", args.case, "T=%d" % c.T, "seqs=%d" % c.n_seqs)


if __name__ == "__main__":
    main()
