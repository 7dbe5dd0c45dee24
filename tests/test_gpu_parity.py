"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Bar: output within 2e-2 of max|out|, final fp32 state
within 1e-3 of max|S|, conv state bit-exact (it is a copy of inputs)."""
import ctypes
import os

import numpy as np
import pytest
import torch

import gdn_testlib as L
import oracle
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    gdn.lib()   # the native library must load: no other implementation exists
    yield


# ---------------------------------------------------------------------------
# tcgen05 operand layouts (test-only probe library)
# ---------------------------------------------------------------------------

def _probe():
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "csrc"))
    import build_probe
    lib = ctypes.CDLL(build_probe.build())
    lib.umma_probe.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.umma_probe.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("variant,K,N", [(0, 128, 64), (1, 64, 64), (2, 128, 64), (3, 64, 128),
                                         (4, 128, 64), (5, 64, 128), (6, 128, 64)])
def test_tcgen05_operand_layouts(variant, K, N):
    """Each operand form the prefill kernels use multiplies correctly: K-major and
    MN-major shared-memory tiles, and A read from tensor memory."""
    lib = _probe()
    rng = np.random.default_rng(variant)
    A = rng.normal(size=(128, K)).astype(np.float32)
    B = rng.normal(size=(N, K)).astype(np.float32)
    At, Bt = torch.from_numpy(A).to(DEV), torch.from_numpy(B).to(DEV)
    Dt = torch.full((128, N), float("nan"), device=DEV)
    rc = lib.umma_probe(variant, ctypes.c_void_p(At.data_ptr()), ctypes.c_void_p(Bt.data_ptr()),
                        ctypes.c_void_p(Dt.data_ptr()))
    assert rc == 0
    ref = A.astype(np.float16).astype(np.float64) @ B.astype(np.float16).astype(np.float64).T
    np.testing.assert_allclose(Dt.cpu().numpy(), ref, rtol=0, atol=1e-3 * np.abs(ref).max())


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------

def test_tiny_fp32_parity():
    """2 key / 6 value heads of dim 32, fp32 activations and output, T = 64."""
    c = inputs.make_case("tiny")
    g = L.gpu_prefill(c)
    r = L.oracle_run(c)
    L.assert_parity(g, r)
    np.testing.assert_array_equal(L.conv_state_bits(c, g["conv_state_t"]),
                                  L.expected_conv_state(c, c.acts, c.conv_state, c.cu_seqlens))


def test_tiny_bf16_output():
    c = inputs.make_case("tiny")
    g = L.gpu_prefill(c, out_dtype=torch.bfloat16)
    L.assert_parity(g, L.oracle_run(c))


def test_prefill_4k_parity_all_heads():
    """One 4096-token sequence at the layer's shape (16 / 48 heads of 128)."""
    c = inputs.make_case("prefill_4k")
    g = L.gpu_prefill(c)
    r = L.oracle_run(c)
    eo, es = L.assert_parity(g, r)
    print("prefill_4k out %.2e state %.2e" % (eo, es))


def _ragged_case(lens, seed=5, state_std=0.05):
    base = inputs.make_case("prefill_4k", T=int(sum(lens)), seed=seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    N = len(lens)
    cs = inputs.f32_to_bf16_bits(rng.normal(size=(N, base.channels, 3)).astype(np.float32))
    rs = (state_std * rng.normal(size=(N, base.n_v_heads, base.d_v, base.d_k))).astype(np.float32)
    base.cu_seqlens, base.conv_state, base.rec_state = cu, cs, rs
    return base


def test_ragged_varlen_with_states():
    """Tails of 1, 63, 64, 65 tokens, an empty sequence, sequences shorter than the
    conv window, and nonzero starting conv and recurrent states."""
    c = _ragged_case([1, 63, 64, 65, 0, 130, 3, 2, 200])
    g = L.gpu_prefill(c)
    r = L.oracle_run(c)
    L.assert_parity(g, r)
    np.testing.assert_array_equal(L.conv_state_bits(c, g["conv_state_t"]),
                                  L.expected_conv_state(c, c.acts, c.conv_state, c.cu_seqlens))
    # the empty sequence keeps both states bit for bit
    np.testing.assert_array_equal(g["rec_state"][4], c.rec_state[4].astype(np.float64))


def test_bf16_small_heads_ragged_streaming_conv():
    """bf16 activations at 2 key / 6 value heads of 64: q, k, v widths that are not
    multiples of 512 channels take the streaming conv kernel (the tiled one needs
    whole 512-channel slices); ragged lengths, an empty sequence, nonzero states."""
    Hk, Hv, d, K = 2, 6, 64, 4
    lens = [1, 63, 70, 0, 130, 2, 40]
    T, N = sum(lens), len(lens)
    w = inputs._weights(7, Hk, Hv, d, d, K)
    acts = inputs._acts(7, T, Hk, Hv, d, d, True, "model")
    rng = np.random.default_rng(7)
    C = 2 * Hk * d + Hv * d
    cs = inputs.f32_to_bf16_bits(rng.normal(size=(N, C, K - 1)).astype(np.float32))
    rs = (0.05 * rng.normal(size=(N, Hv, d, d))).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    c = inputs.Case("small_bf16", Hk, Hv, d, d, K, 64, True, cu, w, acts, cs, rs)
    g = L.gpu_prefill(c)
    L.assert_parity(g, L.oracle_run(c))
    np.testing.assert_array_equal(L.conv_state_bits(c, g["conv_state_t"]),
                                  L.expected_conv_state(c, c.acts, c.conv_state, c.cu_seqlens))


def test_varlen_8_full_size_sampled_heads():
    """The 8-sequence packed workload at full size; oracle on sampled value heads."""
    c = inputs.make_case("varlen_8")
    g = L.gpu_prefill(c)
    heads = [0, 1, 2, 25, 47]
    r = L.oracle_run(c, heads=heads)
    L.assert_parity(g, r, heads=heads)
    np.testing.assert_array_equal(L.conv_state_bits(c, g["conv_state_t"]),
                                  L.expected_conv_state(c, c.acts, c.conv_state, c.cu_seqlens))


def test_split_prefill_equals_one_prefill_on_gpu():
    """prefill(T1) then prefill(T2) on the GPU matches the oracle's prefill(T1+T2)."""
    c = inputs.make_case("prefill_4k", T=300, seed=9)
    T1 = 131
    a1 = {n: x[:T1] for n, x in c.acts.items()}
    a2 = {n: x[T1:] for n, x in c.acts.items()}
    g1 = L.gpu_prefill(c, acts=a1, cu=np.array([0, T1], np.int32))
    cs1 = L.conv_state_bits(c, g1["conv_state_t"])
    g2 = L.gpu_prefill(c, acts=a2, conv_state=cs1, rec_state=g1["rec_state"].astype(np.float32),
                       cu=np.array([0, 300 - T1], np.int32))
    r = L.oracle_run(c)
    out = np.concatenate([g1["out"], g2["out"]])
    assert L.rel_err(out, r["out"]) <= L.OUT_TOL
    assert L.rel_err(g2["rec_state"], r["rec_state"]) <= L.STATE_TOL


def test_prefill_256k_sampled_heads():
    """One 262,144-token sequence (weak decay: -log alpha ~ U(1e-4, 0.1)); the fp32
    state is carried across 4096 chunks; oracle on sampled value heads."""
    c = inputs.make_case("prefill_256k")
    g = L.gpu_prefill(c)
    heads = [0, 47]
    r = L.oracle_run(c, heads=heads)
    eo, es = L.assert_parity(g, r, heads=heads)
    print("prefill_256k out %.2e state %.2e" % (eo, es))


def test_zero_tokens_is_noop():
    c = inputs.make_case("tiny")
    cfg = L.config_of(c)
    w = L.weights_on(c, DEV)
    empty = {n: L.t_act(x[:0], DEV) for n, x in c.acts.items()}
    cs = L.t_act(c.conv_state, DEV)
    rs = torch.ones((1, c.n_v_heads, c.d_v, c.d_k), device=DEV)
    cu = torch.zeros(2, dtype=torch.int32, device=DEV)
    gdn.prefill(cfg, w, empty["q"], empty["k"], empty["v"], empty["a"], empty["b"], empty["z"], cs, rs, cu)
    gdn.check_device_error()
    assert torch.all(rs == 1)


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

_decode_steps = L.decode_steps
_as_sequences = L.as_sequences


def test_decode_batch256_four_steps_all_heads():
    c = inputs.make_case("decode_256", T=4)
    outs, cs, rs = _decode_steps(c, c.steps)
    seqs = list(range(c.n_seqs))
    acts, cu = _as_sequences(c, c.steps, seqs)
    r = L.oracle_run(c, acts=acts, cu=cu)
    ro = r["out"].reshape(c.n_seqs, 4, c.n_v_heads, c.d_v)
    go = np.stack(outs, axis=1)
    assert L.rel_err(go, ro) <= L.OUT_TOL
    assert L.rel_err(rs, r["rec_state"]) <= L.STATE_TOL
    x = {k: np.stack([st[k] for st in c.steps], axis=1) for k in "qkv"}   # [N, 4, ...]
    expect = np.concatenate([c.conv_state[:, :, 3:],
                             np.concatenate([x["q"], x["k"], x["v"]], axis=2)[:, 1:].transpose(0, 2, 1)],
                            axis=2)
    np.testing.assert_array_equal(L.conv_state_bits(c, cs), expect)


def test_decode_batch256_64_steps_sampled_sequences():
    """64 consecutive steps at batch 256 (the timed workload); oracle on sampled sequences."""
    c = inputs.make_case("decode_256")
    outs, cs, rs = _decode_steps(c, c.steps)
    seqs = [0, 77, 255]
    acts, cu = _as_sequences(c, c.steps, seqs)
    sub_cs = c.conv_state[seqs]
    sub_rs = c.rec_state[seqs]
    r = L.oracle_run(c, acts=acts, cu=cu, conv_state=sub_cs, rec_state=sub_rs)
    ro = r["out"].reshape(len(seqs), 64, c.n_v_heads, c.d_v)
    go = np.stack(outs, axis=1)[seqs]
    assert L.rel_err(go, ro) <= L.OUT_TOL
    assert L.rel_err(rs[seqs], r["rec_state"]) <= L.STATE_TOL


def test_decode_small_heads_dim32_fp32():
    """Decode at 2 key / 6 value heads of dim 32 with fp32 activations."""
    c = inputs.make_case("tiny", T=8)
    steps = [{k: c.acts[k][t:t + 1] for k in "qkvabz"} for t in range(8)]
    outs, cs, rs = _decode_steps(c, steps)
    r = L.oracle_run(c)
    assert L.rel_err(np.concatenate(outs), r["out"]) <= L.OUT_TOL
    assert L.rel_err(rs, r["rec_state"]) <= L.STATE_TOL


def test_prefill_then_decode_equals_longer_prefill():
    c = inputs.make_case("prefill_4k", T=200, seed=11)
    T1 = 190
    g = L.gpu_prefill(c, acts={n: x[:T1] for n, x in c.acts.items()}, cu=np.array([0, T1], np.int32))
    cfg = L.config_of(c)
    w = L.weights_on(c, DEV)
    cs = g["conv_state_t"]
    rs = torch.from_numpy(g["rec_state"].astype(np.float32)).to(DEV)
    outs = [g["out"]]
    for t in range(T1, 200):
        d = {n: L.t_act(c.acts[n][t:t + 1], DEV) for n in "qkvabz"}
        o = gdn.decode(cfg, w, d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], cs, rs)
        outs.append(L.to_f64(o).reshape(1, c.n_v_heads, c.d_v))
    gdn.check_device_error()
    r = L.oracle_run(c)
    assert L.rel_err(np.concatenate(outs), r["out"]) <= L.OUT_TOL
    assert L.rel_err(L.to_f64(rs), r["rec_state"]) <= L.STATE_TOL
