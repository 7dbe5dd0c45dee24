"""gdn_prefill_host: prefill from host buffers with the copies overlapping the work.

The tokens run in segments of a multiple of 64 rows; sequences that cross a cut
continue from the states the previous segment left on the device.  Checks:
* a varlen batch whose sequences cross several cuts (one of them empty, nonzero
  initial states) against the fp64 oracle at the layer's bars, conv state bit-exact;
* one 4096-token sequence against gdn_prefill on the device: the cuts fall on
  chunk boundaries and the state crosses each cut in fp32, so the chain is the same
  (measured bit-identical; the bar is 1e-6);
* pageable host memory (no overlap, same result) and a single short segment.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _host(c, pin=True):
    def cpu(x):
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 \
            else torch.from_numpy(np.ascontiguousarray(x))
        return t.pin_memory() if pin else t.clone()
    h = {n: cpu(c.acts[n]) for n in "qkvabz"}
    h["cu_seqlens"] = torch.from_numpy(c.cu_seqlens.astype(np.int32))
    h["cu_seqlens"] = h["cu_seqlens"].pin_memory() if pin else h["cu_seqlens"]
    out = torch.empty((c.T, c.n_v_heads * c.d_v), dtype=torch.bfloat16)
    h["out"] = out.pin_memory() if pin else out
    return h


def _run_host(c, pin=True):
    cfg = L.config_of(c)
    w = L.weights_on(c, DEV)
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(np.ascontiguousarray(c.rec_state, dtype=np.float32)).to(DEV)
    h = _host(c, pin)
    gdn.prefill_host(cfg, w, h, cs, rs)
    torch.cuda.synchronize()
    gdn.check_device_error()
    return (h["out"].float().numpy().astype(np.float64).reshape(c.T, c.n_v_heads, c.d_v), cs, L.to_f64(rs))


def test_prefill_host_varlen_across_cuts():
    lens = [1000, 0, 37, 900, 663]
    T = sum(lens)
    c = inputs.make_case("prefill_4k", T=T, seed=12)
    c.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(12)
    N = len(lens)
    c.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(N, c.channels, 3)).astype(np.float32))
    c.rec_state = (0.05 * rng.normal(size=(N, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)
    out, cs, rs = _run_host(c)
    r = L.oracle_run(c)
    L.assert_parity({"out": out, "rec_state": rs}, r)
    np.testing.assert_array_equal(L.conv_state_bits(c, cs),
                                  L.expected_conv_state(c, c.acts, c.conv_state, c.cu_seqlens))


def test_prefill_host_equals_device_prefill_on_chunk_aligned_cuts():
    c = inputs.make_case("prefill_4k", seed=13)
    out, cs, rs = _run_host(c)
    g = L.gpu_prefill(c)
    eo, es = L.rel_err(out, g["out"]), L.rel_err(rs, g["rec_state"])
    print("host vs device prefill: out %.2e, state %.2e" % (eo, es))
    assert eo <= 1e-6 and es <= 1e-6
    assert torch.equal(cs, g["conv_state_t"])


def test_prefill_host_pageable_and_single_segment():
    c = inputs.make_case("prefill_4k", T=300, seed=14)
    out_p, _, rs_p = _run_host(c, pin=False)
    out, _, rs = _run_host(c, pin=True)
    np.testing.assert_array_equal(out_p, out)
    np.testing.assert_array_equal(rs_p, rs)
    r = L.oracle_run(c)
    L.assert_parity({"out": out, "rec_state": rs}, r)
