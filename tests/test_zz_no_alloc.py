"""gdn_prefill_noalloc: the prefill entry point for callers that cannot allocate
device memory.  Some servers hand all device memory to their own pool at
start-up, and some latency-critical callers cannot take cudaMalloc's implicit
synchronisation; neither can pass a workspace.  This entry point keeps its
scratch in a fixed device array inside the library.

The test first leaves NaN in the shared array (a call at the largest size that
fits, whose gates, v and z are NaN), then calls the entry point through the C
ABI twice in a row, on different inputs, and checks each result against the
workspace entry point gdn_prefill bit for bit: the kernels are deterministic,
so any read of a stale scratch element would show.  This file sorts last so
that a run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import gdn_testlib as L
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SCRATCH_BYTES = 64 << 20      # GDN_NOALLOC_SCRATCH_BYTES in include/gdn.h
WORKSPACE_ERR = 5             # GDN_ERR_WORKSPACE


def _entry():
    f = gdn.lib().gdn_prefill_noalloc
    vp = ctypes.c_void_p
    f.argtypes = [vp, vp] + [vp] * 8 + [vp, ctypes.c_int32, ctypes.c_int64, vp, vp]
    f.restype = ctypes.c_int
    return f


def _case(lens, seed):
    c = inputs.make_case("prefill_4k", T=int(sum(lens)), seed=seed)
    rng = np.random.default_rng(seed)
    N = len(lens)
    c.cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    c.conv_state = inputs.f32_to_bf16_bits(rng.normal(size=(N, c.channels, 3)).astype(np.float32))
    c.rec_state = (0.05 * rng.normal(size=(N, c.n_v_heads, c.d_v, c.d_k))).astype(np.float32)
    return c


def _run_noalloc(f, c):
    cfg = L.config_of(c)
    w = L.weights_on(c, DEV)
    d = {n: L.t_act(c.acts[n], DEV) for n in "qkvabz"}
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.from_numpy(c.rec_state).to(DEV)
    cu = torch.from_numpy(c.cu_seqlens).to(DEV)
    T = d["q"].shape[0]
    out = torch.full((T, c.n_v_heads * c.d_v), float("nan"), dtype=torch.bfloat16, device=DEV)
    cc, cw = cfg.c(), gdn._weights(w, torch.device(DEV))
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = f(ctypes.byref(cc), ctypes.byref(cw), P(d["q"]), P(d["k"]), P(d["v"]), P(d["a"]), P(d["b"]),
          P(d["z"]), P(cs), P(rs), P(cu), c.cu_seqlens.shape[0] - 1, T, P(out),
          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert s == 0, gdn.status_string(s)
    gdn.check_device_error()
    return {"out": L.to_f64(out).reshape(T, c.n_v_heads, c.d_v), "conv_state_t": cs,
            "rec_state": L.to_f64(rs)}


def _largest_single_sequence():
    cfg = gdn.Config()
    fits = 1
    while gdn.workspace_size(cfg, fits + 1, 1) <= SCRATCH_BYTES:
        fits += 1
    return fits


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    f = _entry()
    # leave NaN in the shared array: NaN gates, v and z reach the records, v^ and the
    # o tiles (q and k stay finite, so the call's range check lets it run through)
    poison = _case([_largest_single_sequence()], 40)
    nan = inputs.f32_to_bf16_bits(np.full((1,), np.nan, np.float32))[0]
    for n in "abvz":
        poison.acts[n] = np.full_like(poison.acts[n], nan)
    _run_noalloc(f, poison)
    for lens, seed in (([300, 1, 65, 0, 130], 41), ([600, 63], 42)):
        c = _case(lens, seed)
        got = _run_noalloc(f, c)
        ref = L.gpu_prefill(c)          # gdn_prefill with a caller workspace
        assert np.isfinite(got["out"]).all()
        assert np.array_equal(got["out"], ref["out"])
        assert np.array_equal(got["rec_state"], ref["rec_state"])
        assert torch.equal(got["conv_state_t"], ref["conv_state_t"])


def test_noalloc_rejects_requests_beyond_its_scratch():
    f = _entry()
    c = _case([8], 43)
    cfg = gdn.Config()
    fits = _largest_single_sequence()
    assert fits == 823   # the limit include/gdn.h states for one sequence
    cc, cw = cfg.c(), gdn._weights(L.weights_on(c, DEV), torch.device(DEV))
    dummy = torch.zeros(16, device=DEV)
    P = ctypes.c_void_p(dummy.data_ptr())
    s = f(ctypes.byref(cc), ctypes.byref(cw), *[P] * 8, P, 1, fits + 1, P, None)
    assert s == WORKSPACE_ERR
