"""Device-side checks and failure detection, on the GPU, with no fault.

* A bounded mbarrier wait that nothing completes gives up after its limit,
  records its code in the error word, and the kernel returns; the host maps the
  word to GDN_ERR_DEVICE_TIMEOUT and the context stays usable.  The wait runs in
  the test-only probe library, built from the same device.cuh code (wait,
  error word, host-side mapping) as the library's kernels.
* A malformed cu_seqlens (device memory, so the host cannot check it) is caught
  by the prefill's first kernel: GDN_ERR_SEQLENS, and neither out nor the states
  are written.
* A conv output beyond the fp16 range of the prefill workspace is caught by the
  conv kernel: GDN_ERR_RANGE, and again nothing is written.

Every input here stays inside every buffer even if the checks were missing.
"""
import ctypes

import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TIMEOUT, SEQLENS, RANGE = 4, 6, 7


def _probe():
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "csrc"))
    import build_probe
    lib = ctypes.CDLL(build_probe.build())
    lib.probe_wait_timeout.argtypes = [ctypes.c_ulonglong, ctypes.c_void_p, ctypes.POINTER(ctypes.c_float),
                                       ctypes.c_void_p]
    lib.probe_wait_timeout.restype = ctypes.c_int
    lib.probe_check_device_error.argtypes = [ctypes.c_void_p]
    lib.probe_check_device_error.restype = ctypes.c_int
    return lib


def test_bounded_wait_runs_out_reports_timeout_and_the_gpu_stays_usable():
    lib = _probe()
    gave_up = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    ms = ctypes.c_float(0.0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    limit_ns = 100_000   # 100 us
    s = lib.probe_wait_timeout(limit_ns, ctypes.c_void_p(gave_up.data_ptr()), ctypes.byref(ms), stream)
    assert s == TIMEOUT, s
    assert int(gave_up.item()) == 1
    assert 0.1 <= ms.value < 1000.0, ms.value       # it waited its limit, then returned
    assert lib.probe_check_device_error(stream) == 0  # read and cleared
    # the context is still usable: a decode step after it matches the oracle
    c = inputs.make_case("decode_256", T=1, seed=9, n_seqs=4)
    outs, _, rs = L.decode_steps(c, c.steps)
    r = L.oracle_run(c, acts=c.steps[0], cu=np.arange(0, 5, dtype=np.int32))
    assert L.rel_err(outs[0], r["out"]) <= L.OUT_TOL
    assert L.rel_err(rs, r["rec_state"]) <= L.STATE_TOL
    gdn.check_device_error()


def _prefill_raw(c, cu, acts=None, segments=0):
    """gdn_prefill with cu_seqlens given as is; returns the device tensors and the
    status gdn_check_device_error reports.  segments > 1 pipelines the call over
    that many chunk ranges, whose scans run before the last range's conv checks
    its outputs."""
    acts = c.acts if acts is None else acts
    cfg = L.config_of(c)
    cfg.prefill_segments = segments
    w = L.weights_on(c, DEV)
    d = {n: L.t_act(acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(np.ascontiguousarray(c.rec_state)).to(DEV)
    cu_t = torch.from_numpy(np.asarray(cu, np.int32)).to(DEV)
    T = d["q"].shape[0]
    out = torch.full((T, c.n_v_heads * c.d_v), 7.0, dtype=cfg.out_dtype, device=DEV)
    before = (out.clone(), cs.clone(), rs.clone())
    gdn.prefill(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs, cu_t, out=out)
    s = gdn.lib().gdn_check_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return s, (out, cs, rs), before


def _case(T, seed):
    c = inputs.make_case("prefill_4k", T=T, seed=seed)
    rng = np.random.default_rng(seed)
    N = 3
    c.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(N, c.channels, 3)).astype(np.float32))
    c.rec_state = (0.05 * rng.normal(size=(N, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)
    return c


@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("cu", [[0, 200, 100, 300],     # decreasing
                                [0, 100, 160, 250],     # does not end at T_total
                                [0, 100, 160, 290]])
def test_malformed_cu_seqlens_is_reported_and_nothing_is_written(cu, segments):
    c = _case(300, 61)
    s, after, before = _prefill_raw(c, cu, segments=segments)
    assert s == SEQLENS, gdn.status_string(s)
    for x, y in zip(after, before):
        assert torch.equal(x, y)
    # the next (well-formed) call on the same workspace-free path runs normally
    good = np.array([0, 100, 160, 300], np.int32)
    g = L.gpu_prefill(c, cu=good)
    r = L.oracle_run(c, cu=good)
    L.assert_parity(g, r)


# 200 tokens in 4 ranges of one chunk: [0, 1), [1, 2), [2, 3) and [3, end) of the global
# chunks of cu_seqlens [0, 70, 120, 200] (two, one and two chunks).  Rows 50..59 fall in
# the first range's conv; rows 185..194 (the second sequence's second chunk) in the last
# one's, which runs after the other ranges' scans.
@pytest.mark.parametrize("segments,rows", [(1, (50, 60)), (4, (50, 60)), (4, (185, 195))])
def test_conv_output_beyond_fp16_is_reported_and_nothing_is_written(segments, rows):
    c = _case(200, 62)
    acts = dict(c.acts)
    v = inputs.bf16_bits_to_f32(acts["v"]).copy()
    v[rows[0]:rows[1]] = 3.0e6   # the conv of these rows reaches millions on half the channels
    acts["v"] = inputs.f32_to_bf16_bits(v)
    cu = np.array([0, 70, 120, 200], np.int32)
    s, after, before = _prefill_raw(c, cu, acts=acts, segments=segments)
    assert s == RANGE, gdn.status_string(s)
    for x, y in zip(after, before):
        assert torch.equal(x, y)
    # large q and k are normalised, so they are in range
    acts = dict(c.acts)
    acts["q"] = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(c.acts["q"]) * 1.0e4)
    s, _, _ = _prefill_raw(c, cu, acts=acts, segments=segments)
    assert s == 0, gdn.status_string(s)
