#!/usr/bin/env python
"""Benchmark of the B200 Gated DeltaNet mixer (one layer).

A step is one pass of the whole hot path on synthetic inputs resident in HBM:
one packed prefill of a 4096-token sequence at the layer's shape (16 key / 48
value heads of 128: conv + SiLU + L2 norm, chunked gated delta rule, gated
RMSNorm) followed by 64 consecutive decode steps at batch 256 (fp32 state
[256, 48, 128, 128]).  The headline value is prefill tokens/s; decode is
reported as state-streaming HBM GB/s.  Times are CUDA events on the launching
stream, L2 flushed (256 MiB write) before each timed region, max over ranks.

Under torchrun every rank runs its own replica (independent sequences: weak
scaling, no data-path collective).

--impl reference times the fp64 CPU oracle (the correctness reference, a
deliberately slow baseline) on the host cores on the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (T=4K, 1 layer); decode state HBM GB/s at batch 256"
PREFILL_T = 4096
DECODE_N = 256
H_K, H_V, D = 16, 48, 128
C_CONV = 2 * H_K * D + H_V * D
# Algorithmic work per unit:
#   prefill dense FLOPs per token: H_k * 4*C*d + H_v * (6*C*d + 6*d^2), C = 64
PREFILL_FLOP_PER_TOKEN = H_K * 4 * 64 * D + H_V * (6 * 64 * D + 6 * D * D)
#   prefill bytes per call: q, k, v, z, a, b in and out, bf16, per token; the fp32 state read and
#   written once (at 168 FLOP/byte the call sits below the bf16 ridge: it is bound by these bytes)
PREFILL_BYTES_PER_TOKEN = (2 * H_K * D + 2 * H_V * D + 2 * H_V) * 2 + H_V * D * 2
PREFILL_STATE_BYTES = 2 * H_V * D * D * 4
#   decode bytes per step: fp32 state read + write, conv state read + write,
#   q/k/v/a/b/z in, out, parameters
DECODE_BYTES_PER_STEP = (2 * DECODE_N * H_V * D * D * 4 + 2 * DECODE_N * C_CONV * 3 * 2
                         + DECODE_N * (2 * H_K * D + 2 * H_V * D + 2 * H_V) * 2
                         + DECODE_N * H_V * D * 2 + (C_CONV * 4 + 2 * H_V + D) * 4)
#   multi-token decode bytes per call: the state and conv state once, inputs and outputs per token
MULTI_TOK = 4
MULTI_BYTES_PER_CALL = (2 * DECODE_N * H_V * D * D * 4 + 2 * DECODE_N * C_CONV * 3 * 2
                        + MULTI_TOK * DECODE_N * (2 * H_K * D + 2 * H_V * D + 2 * H_V) * 2
                        + MULTI_TOK * DECODE_N * H_V * D * 2 + (C_CONV * 4 + 2 * H_V + D) * 4)
#   decode with a bf16 state: the state bytes halve
BF16_BLOCK = 16
DECODE_BF16_BYTES_PER_STEP = DECODE_BYTES_PER_STEP - DECODE_N * H_V * D * D * 4
#   projections around the mixer (hidden size 2,560): dense FLOPs per call at PREFILL_T tokens
D_MODEL = 2560
PROJ_IN_N = 2 * H_K * D + 2 * H_V * D + 2 * H_V
PROJ_IN_FLOP = 2 * PREFILL_T * D_MODEL * PROJ_IN_N
PROJ_OUT_FLOP = 2 * PREFILL_T * H_V * D * D_MODEL
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# ncu DRAM bytes (read + write) per decode launch at batch 256, taken on the
# fp32-state decode kernel (gdn_decode_kernel) whose source text hashes to
# DECODE_SRC_SHA; null once that kernel's text changes.
DECODE_TRAFFIC = 1593363968          # mean of 3 launches at batch 256
DECODE_SRC_SHA = "4315b287d18a287c"
DECODE_KERNEL_TEXT = ("template <typename TA, typename TO, typename TS, int DK>\n"
                      "__global__ void __launch_bounds__(NT) gdn_decode_kernel", "// Multi-token rows")
# Tensor-pipe activity of the prefill's tensor-core kernels (ncu
# sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active, one --set full capture of the
# 4K prefill in one chunk range; the scan's average is over the SMs that run it), taken on the
# sources that hash to the given values; null once a file changes.
TENSOR_PIPE_NCU = {"gdn_intra_kernel": ("intra.cuh", "b1f14988bf943661", 0.0411),
                   "gdn_scan_kernel": ("scan.cuh", "4ce0eddd0125a8b0", 0.2811)}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_sha(name, section=None):
    """sha256 (16 hex digits) of a source file, or of the text from section[0] up to section[1]."""
    with open(os.path.join(ROOT, "hybrid_linear_attention_mixer_b200", "csrc", name)) as f:
        text = f.read()
    if section is not None:
        a = text.find(section[0])
        b = text.find(section[1], a) if a >= 0 else -1
        if b < 0:
            return None
        text = text[a:b]
    return hashlib.sha256(text.encode()).hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        sm, mx, reasons = [], None, set()
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) < 7:
                        continue
                    try:
                        sm.append(float(parts[0]))
                        mx = float(parts[1])
                    except ValueError:
                        continue
                    for n, v in zip(names, parts[3:7]):
                        if v.lower().startswith("active"):
                            reasons.add(n)
            os.unlink(self.path)
        except OSError:
            pass
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


def cpu_oracle_prefill(seconds=10.0):
    """fp64 oracle on the prefill workload, repeated for about `seconds`."""
    import oracle
    from hybrid_linear_attention_mixer_b200 import inputs
    c = inputs.make_case("prefill_4k")
    sh = oracle.Shape(c.n_k_heads, c.n_v_heads, c.d_k, c.d_v)
    cores = len(os.sched_getaffinity(0))
    cs = oracle.act_to_f64(c.conv_state)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(sh, c.weights, *[c.acts[n] for n in "qkvabz"], cs, c.rec_state, c.cu_seqlens,
                       threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": reps * PREFILL_T / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "prefill of 1 x %d tokens, all %d value heads, fp64, %d repetition(s) in %.1f s"
                      % (PREFILL_T, H_V, reps, el)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from hybrid_linear_attention_mixer_b200 import inputs
    c = inputs.make_case("prefill_4k")
    sh = oracle.Shape(c.n_k_heads, c.n_v_heads, c.d_k, c.d_v)
    cores = len(os.sched_getaffinity(0))
    cs = oracle.act_to_f64(c.conv_state)

    def step():
        oracle.forward(sh, c.weights, *[c.acts[n] for n in "qkvabz"], cs, c.rec_state, c.cu_seqlens,
                       threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    v = args.steps * PREFILL_T / el
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "prefill_4k: 1 sequence x 4096 tokens, 16/48 heads of 128, conv 4",
                       "global_batch": 1, "seq_len": PREFILL_T, "parallelism": "host threads"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": "the full prefill workload each step (fp64, %d threads)" % cores},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    import torch.distributed as dist
    from hybrid_linear_attention_mixer_b200 import gdn, inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    gdn.lib()

    def act(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)

    # ---- prefill workload: 1 x 4096 tokens ----
    pc = inputs.make_case("prefill_4k", seed=1 + rank)
    cfg = gdn.Config()
    w = {n: torch.from_numpy(pc.weights[n]).to(dev) for n in ("conv_w", "A_log", "dt_bias", "norm_w")}
    host = {n: act(pc.acts[n]).pin_memory() for n in "qkvabz"}
    host["cu_seqlens"] = torch.from_numpy(pc.cu_seqlens).pin_memory()
    P = {n: host[n].to(dev) for n in host}
    p_cs = act(pc.conv_state).to(dev)
    p_rs = torch.zeros((1, H_V, D, D), dtype=torch.float32, device=dev)
    p_out = torch.empty((PREFILL_T, H_V * D), dtype=torch.bfloat16, device=dev)
    p_ws = torch.empty(gdn.workspace_size(cfg, PREFILL_T, 1), dtype=torch.uint8, device=dev)
    host["out"] = torch.empty((PREFILL_T, H_V * D), dtype=torch.bfloat16).pin_memory()

    # ---- decode workload: batch 256, 64 consecutive steps ----
    dc = inputs.make_case("decode_256", seed=3 + rank, T=args.decode_steps)
    dw = {n: torch.from_numpy(dc.weights[n]).to(dev) for n in ("conv_w", "A_log", "dt_bias", "norm_w")}
    steps = [{n: act(st[n]).to(dev) for n in "qkvabz"} for st in dc.steps]
    d_cs = act(dc.conv_state).to(dev)
    d_rs = torch.from_numpy(dc.rec_state).to(dev)
    d_out = torch.empty((DECODE_N, H_V * D), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    stream = torch.cuda.current_stream()

    def prefill():
        gdn.prefill(cfg, w, P["q"], P["k"], P["v"], P["a"], P["b"], P["z"], p_cs, p_rs,
                    P["cu_seqlens"], out=p_out, workspace=p_ws, stream=stream)

    def decode_all():
        for st in steps:
            gdn.decode(cfg, dw, st["q"], st["k"], st["v"], st["a"], st["b"], st["z"], d_cs, d_rs,
                       out=d_out, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        prefill()
        flush.zero_()
        decode_all()
    gdn.check_device_error(stream)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = "GPU-" + str(props.uuid) if getattr(props, "uuid", None) else str(local)
    with ClockSampler(gpu_id) as clocks:
        time.sleep(0.3)
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            prefill()
            ev[i][1].record(stream)
            flush.zero_()
            ev[i][2].record(stream)
            decode_all()
            ev[i][3].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    gdn.check_device_error(stream)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in ev)
    t = torch.tensor([pre_ms, dec_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    pre_ms, dec_ms = float(t[0]), float(t[1])

    # ---- multi-token decode (draft verification): MULTI_TOK tokens per sequence, one pass ----
    mt = MULTI_TOK
    m_in = {n: torch.stack([st[n] for st in steps[:mt]], dim=1).reshape(DECODE_N * mt, -1).contiguous()
            for n in "qkvabz"}
    m_out = torch.empty((DECODE_N * mt, H_V * D), dtype=torch.bfloat16, device=dev)

    def decode_multi():
        gdn.decode_multi(cfg, dw, m_in["q"], m_in["k"], m_in["v"], m_in["a"], m_in["b"], m_in["z"],
                         d_cs, d_rs, mt, out=m_out, stream=stream)

    m_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for i in range(-args.warmup, args.steps):
        flush.zero_()
        if i >= 0:
            m_ev[i][0].record(stream)
        decode_multi()
        if i >= 0:
            m_ev[i][1].record(stream)
    torch.cuda.synchronize()
    gdn.check_device_error(stream)
    tm = torch.tensor([sum(a.elapsed_time(b) for a, b in m_ev)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
    multi_ms = float(tm[0])

    # ---- decode with the state stored in bf16: 16 consecutive steps per timed block ----
    cfg_b = gdn.Config(state_dtype=torch.bfloat16)
    b_rs = d_rs.to(torch.bfloat16)
    b_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for i in range(-args.warmup, args.steps):
        flush.zero_()
        if i >= 0:
            b_ev[i][0].record(stream)
        for st in steps[:BF16_BLOCK]:
            gdn.decode(cfg_b, dw, st["q"], st["k"], st["v"], st["a"], st["b"], st["z"], d_cs, b_rs,
                       out=d_out, stream=stream)
        if i >= 0:
            b_ev[i][1].record(stream)
    torch.cuda.synchronize()
    gdn.check_device_error(stream)
    tb = torch.tensor([sum(a.elapsed_time(b) for a, b in b_ev)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tb, op=dist.ReduceOp.MAX)
    bf16_step_s = float(tb[0]) / 1e3 / (args.steps * BF16_BLOCK)

    # ---- projections around the mixer at the prefill workload's 4096 tokens ----
    pj = inputs.make_proj_case(PREFILL_T, seed=5 + rank)
    hid, w_in, w_out = (act(x).to(dev) for x in (pj.hidden, pj.w_in, pj.w_out))
    pj_out = gdn.in_proj(cfg, hid, w_in, stream=stream)
    y_out = torch.empty((PREFILL_T, D_MODEL), dtype=torch.bfloat16, device=dev)

    def timed(fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(-args.warmup, args.steps):
            flush.zero_()
            if i >= 0:
                evs[i][0].record(stream)
            fn()
            if i >= 0:
                evs[i][1].record(stream)
        torch.cuda.synchronize()
        tt = torch.tensor([sum(a.elapsed_time(b) for a, b in evs)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        return float(tt[0]) / args.steps / 1e3          # seconds per call

    in_s = timed(lambda: gdn.in_proj(cfg, hid, w_in, out=pj_out, stream=stream))
    out_s = timed(lambda: gdn.out_proj(cfg, p_out, w_out, y=y_out, stream=stream))
    gdn.check_device_error(stream)
    # cuBLAS on the same shapes, for context only (not part of the product path)
    in_cublas_s = timed(lambda: torch.nn.functional.linear(hid, w_in))
    out_cublas_s = timed(lambda: torch.nn.functional.linear(p_out, w_out))

    # ---- context-parallel prefill: one sequence of PREFILL_T x N tokens, one segment per rank ----
    cp_cs = act(pc.conv_state[0]).to(dev)
    cp_rs = torch.zeros((H_V, D, D), dtype=torch.float32, device=dev)
    cp_seg = {n: P[n] for n in "qkvabz"}
    if world > 1:
        from hybrid_linear_attention_mixer_b200 import cp as cp_mod

        def cp_step():
            cp_mod.prefill(cfg, w, cp_seg["q"], cp_seg["k"], cp_seg["v"], cp_seg["a"], cp_seg["b"], cp_seg["z"],
                           cp_cs, cp_rs)
        cp_local_s = cp_finish_s = None
    else:
        cp_ws = torch.empty(gdn.cp_workspace_size(cfg, PREFILL_T), dtype=torch.uint8, device=dev)
        cp_sum = torch.empty((1, 2, H_V, D, D), dtype=torch.float32, device=dev)
        cp_cs1 = cp_cs.clone()

        def cp_local():
            cp_cs1.copy_(cp_cs)
            gdn.cp_local(cfg, w, cp_seg["q"], cp_seg["k"], cp_seg["v"], cp_seg["a"], cp_seg["b"], cp_cs1,
                         workspace=cp_ws, summary=cp_sum[0], stream=stream)

        def cp_finish():
            gdn.cp_finish(cfg, w, cp_seg["z"], cp_sum, 0, cp_rs, cp_ws, out=p_out, stream=stream)

        def cp_step():
            cp_local()
            cp_finish()
        cp_local_s, cp_finish_s = timed(cp_local), timed(cp_finish)
    cp_s = timed(cp_step)
    gdn.check_device_error(stream)

    # ---- packed variable-length (8 sequences) and long-context (1 x 262,144) prefills ----
    # (one rank's replica each; timed at N = 1 only, where they add about a minute of set-up)
    def prefill_block(name, seed):
        c = inputs.make_case(name, seed=seed)
        cfg_c = gdn.Config()
        wc = {n: torch.from_numpy(c.weights[n]).to(dev) for n in ("conv_w", "A_log", "dt_bias", "norm_w")}
        dc_ = {n: act(c.acts[n]).to(dev) for n in "qkvabz"}
        del c.acts
        N, T = c.n_seqs, c.T
        cu = torch.from_numpy(c.cu_seqlens).to(dev)
        cs = act(c.conv_state).to(dev)
        rs = torch.zeros((N, H_V, D, D), dtype=torch.float32, device=dev)
        out = torch.empty((T, H_V * D), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(gdn.workspace_size(cfg_c, T, N), dtype=torch.uint8, device=dev)
        sec = timed(lambda: gdn.prefill(cfg_c, wc, dc_["q"], dc_["k"], dc_["v"], dc_["a"], dc_["b"], dc_["z"], cs,
                                        rs, cu, out=out, workspace=ws, stream=stream))
        gdn.check_device_error(stream)
        nbytes = PREFILL_BYTES_PER_TOKEN * T + N * PREFILL_STATE_BYTES
        del dc_, out, ws
        torch.cuda.empty_cache()
        return {"workload": name, "tokens": T, "seqs": N, "seq_lens": np.diff(c.cu_seqlens).tolist(),
                "us_per_call": sec * 1e6, "value": T / sec, "unit": "tokens/s", "bytes_per_call": nbytes,
                "achieved_gbs": nbytes / sec / 1e9, "roofline_us": nbytes / (peaks()[0]["hbm_gbs"] * 1e3)}

    long_blocks = None
    if world == 1:
        long_blocks = {"varlen_8": prefill_block("varlen_8", 2), "prefill_256k": prefill_block("prefill_256k", 4)}

    # ---- end to end through the public API with host buffers ----
    h_ws = torch.empty(gdn.prefill_host_workspace_size(cfg, PREFILL_T, 1), dtype=torch.uint8, device=dev)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    for i in range(-args.warmup, args.steps):
        flush.zero_()
        if i >= 0:
            e2e_ev[i][0].record(stream)
        gdn.prefill_host(cfg, w, host, p_cs, p_rs, workspace=h_ws, stream=stream)
        if i >= 0:
            e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)
    te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
        dist.barrier()
    e2e_ms = float(te[0])
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v", "a", "b", "z", "cu_seqlens"))
    d2h = host["out"].numel() * host["out"].element_size()

    if rank == 0:
        pk, src = peaks()
        K = args.steps
        n_ranges = gdn.prefill_segments(cfg, PREFILL_T, 1)   # -1: the chain split in two
        # prefill kernels per call: the split chain launches chunk offsets, conv, conv-state update,
        # intra, the start states, three scans, the first half's norm, S0 to bf16, the second half's
        # correction and norm, and the state fold; n ranges launch 2 + 4 n (6 for one range)
        prefill_launches = 12 if n_ranges < 0 else 2 + 4 * n_ranges
        plan = "the state chain split in two (3 concurrent scans)" if n_ranges < 0 else \
            "pipelined over %d chunk ranges" % n_ranges
        value = PREFILL_T * world * K / (pre_ms / 1e3)
        dec_launch_s = dec_ms / 1e3 / (K * args.decode_steps)
        dec_gbs = DECODE_BYTES_PER_STEP / dec_launch_s / 1e9
        pre_tflops = PREFILL_FLOP_PER_TOKEN * PREFILL_T / (pre_ms / 1e3 / K) / 1e12
        pre_gbs = (PREFILL_BYTES_PER_TOKEN * PREFILL_T + PREFILL_STATE_BYTES) / (pre_ms / 1e3 / K) / 1e9
        traffic = DECODE_TRAFFIC if DECODE_SRC_SHA == src_sha("decode.cuh", DECODE_KERNEL_TEXT) else None
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": (pre_ms + dec_ms) / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp16-mma/fp32",
            "data": "synthetic (seeded; bf16 activations, fp32 state, random-init conv/gate/norm weights)",
            "config": {"workload": "prefill_4k + decode_256: prefill of 1 x 4096 tokens, then %d decode "
                                   "steps at batch 256; 16/48 heads of 128, conv 4, chunk 64"
                                   % args.decode_steps,
                       "global_batch": world, "seq_len": PREFILL_T, "parallelism": "dp%d" % world,
                       "l2": "flushed (256 MiB write) before each timed region"},
            "decode": {"value": dec_gbs, "unit": "GB/s", "us_per_step": dec_launch_s * 1e6,
                       "tokens_per_s": DECODE_N * world / dec_launch_s,
                       "bytes_per_step": DECODE_BYTES_PER_STEP},
            "decode_multi": {"tokens_per_seq": MULTI_TOK, "value": MULTI_BYTES_PER_CALL / (multi_ms / 1e3 / K) / 1e9,
                             "unit": "GB/s", "us_per_call": multi_ms * 1e3 / K,
                             "tokens_per_s": DECODE_N * MULTI_TOK * world / (multi_ms / 1e3 / K),
                             "bytes_per_call": MULTI_BYTES_PER_CALL},
            "decode_bf16_state": {"value": DECODE_BF16_BYTES_PER_STEP / bf16_step_s / 1e9, "unit": "GB/s",
                                  "us_per_step": bf16_step_s * 1e6, "tokens_per_s": DECODE_N * world / bf16_step_s,
                                  "bytes_per_step": DECODE_BF16_BYTES_PER_STEP},
            "projections": {
                "tokens": PREFILL_T, "d_model": D_MODEL, "unit": "TFLOP/s", "peak": pk["bf16_tflops"],
                "in": {"shape": [PREFILL_T, PROJ_IN_N, D_MODEL], "us": in_s * 1e6,
                       "value": PROJ_IN_FLOP / in_s / 1e12, "frac": PROJ_IN_FLOP / in_s / 1e12 / pk["bf16_tflops"],
                       "cublas_value": PROJ_IN_FLOP / in_cublas_s / 1e12},
                "out": {"shape": [PREFILL_T, D_MODEL, H_V * D], "us": out_s * 1e6,
                        "value": PROJ_OUT_FLOP / out_s / 1e12, "frac": PROJ_OUT_FLOP / out_s / 1e12 / pk["bf16_tflops"],
                        "cublas_value": PROJ_OUT_FLOP / out_cublas_s / 1e12}},
            "context_parallel": {
                "sequence_tokens": PREFILL_T * world, "segment_tokens": PREFILL_T, "ranks": world,
                "value": PREFILL_T * world / cp_s, "unit": "tokens/s", "us_per_call": cp_s * 1e6,
                "local_us": None if cp_local_s is None else cp_local_s * 1e6,
                "finish_us": None if cp_finish_s is None else cp_finish_s * 1e6,
                "exchange_bytes_per_rank": 2 * H_V * D * D * 4,
                "note": "one rank: phase 1 and phase 2 on one segment, no exchange"
                        if world == 1 else "NCCL all-gathers inside the timed call"},
            "prefill_ms": pre_ms / K,
            "prefill_varlen_8": None if long_blocks is None else dict(
                long_blocks["varlen_8"], frac=long_blocks["varlen_8"]["achieved_gbs"] / pk["hbm_gbs"]),
            "prefill_256k": None if long_blocks is None else dict(
                long_blocks["prefill_256k"], frac=long_blocks["prefill_256k"]["achieved_gbs"] / pk["hbm_gbs"]),
            "roofline": {"kernel": "gdn_decode_kernel", "bound": "hbm", "achieved": dec_gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": dec_gbs / pk["hbm_gbs"],
                         "traffic": traffic, "peak_source": src},
            "prefill_roofline": {"kernels": "whole prefill call (chunk offsets, conv, conv state, intra, scan, "
                                            "gated norm), " + plan,
                                 "bound": "hbm", "achieved": pre_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                 "frac": pre_gbs / pk["hbm_gbs"],
                                 "bytes_per_call": PREFILL_BYTES_PER_TOKEN * PREFILL_T + PREFILL_STATE_BYTES,
                                 "tensor_achieved_tflops": pre_tflops, "tensor_peak_tflops": pk["bf16_tflops"],
                                 "tensor_frac": pre_tflops / pk["bf16_tflops"], "peak_source": src},
            "tensor_pipe": dict({k: (v[2] if src_sha(v[0]) == v[1] else None) for k, v in TENSOR_PIPE_NCU.items()},
                                target=0.40, source="ncu captures in profiles/gdn_intra_kernel_prefill_4k.md and "
                                                    "profiles/gdn_scan_kernel_prefill_4k.md"),
            "clocks": clocks.summary(),
            "e2e": {"value": PREFILL_T * world * K / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            # per step: the prefill's kernels, then one kernel per decode step
            "gpu_launches": K * (prefill_launches + args.decode_steps),
            "context": {"pages_cost_model": "6.05 GiB KV+state at 256K tokens and 13.3 GFLOP/token "
                                            "decode at 4K (whole model, no hardware stated)"},
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_prefill()
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
