"""The projections around the mixer (gdn_linear, gdn_in_proj, gdn_out_proj) against
the fp64 oracle.

Bound, per element: the tensor cores multiply bf16 pairs exactly in fp32, add
the K products in fp32 (in some order), and round the sum once to bf16.  A K-term
fp32 sum in any order is within gamma_K * sum_k |x_k w_k| of the exact sum
(gamma_K = K u / (1 - K u)); u = 2^-23 is taken, one fp32 ulp per addition, so
that truncating adders are covered too.  The bf16 rounding adds at most 2^-8 of
the value (unit roundoff of 8 significant bits).  Hence
    |y_gpu - y| <= 2^-8 |y| + (1 + 2^-8) gamma_K sum_k |x_k w_k|.
With inputs in {-1, 0, 1} and K < 256 every partial sum is an integer below 2^24
and |y| <= 255 is a bf16 value, so the result is bit-exact.
"""
import numpy as np
import pytest
import torch

import gdn_testlib as L
import oracle
from hybrid_linear_attention_mixer_b200 import gdn, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bf16(x_bits: np.ndarray) -> torch.Tensor:
    return L.t_act(x_bits, DEV)


def _ternary(rng, shape) -> np.ndarray:
    return inputs.f32_to_bf16_bits(rng.integers(-1, 2, shape).astype(np.float32))


def _bound_ok(y_gpu: np.ndarray, x_bits, w_bits, y_ref: np.ndarray):
    x = np.abs(oracle.act_to_f64(x_bits))
    w = np.abs(oracle.act_to_f64(w_bits))
    K = x.shape[1]
    u = 2.0 ** -23
    gamma = K * u / (1 - K * u)
    lim = 2.0 ** -8 * np.abs(y_ref) + (1 + 2.0 ** -8) * gamma * (x @ w.T)
    err = np.abs(y_gpu - y_ref)
    worst = float((err / np.maximum(lim, 1e-300)).max())
    print("projection: max err %.3e, max err / bound %.3f, max rel %.3e"
          % (err.max(), worst, err.max() / max(np.abs(y_ref).max(), 1e-300)))
    return worst <= 1.0


# (M, N): with M > 128 the CTA-pair form runs; each of the first seven shapes makes
# its tile-width choice land on a different width (128, 144, 160, 192, 208, 224,
# 256 with 74 pairs on 148 SMs).  M <= 128 runs the one-CTA form (widths 128 and
# 256).  Every shape has ragged M, N and K tails.
SHAPES = [(1000, 200), (1000, 2312), (1000, 2600), (1000, 2888), (1000, 3464), (1000, 3752), (1000, 4040),
          (130, 264), (1, 8), (100, 264), (64, 20000)]


@pytest.mark.parametrize("M,N", SHAPES)
def test_linear_integer_inputs_bit_exact(M, N):
    K = 136
    rng = np.random.default_rng(M * 7 + N)
    xb, wb = _ternary(rng, (M, K)), _ternary(rng, (N, K))
    # output split over segments that cut across tiles: 8 | 120 | ... | 16 (when N allows)
    widths = [8, 120, N - 144, 16] if N > 144 else [N]
    outs = [torch.full((M, wd), float("nan"), dtype=torch.bfloat16, device=DEV) for wd in widths]
    gdn.linear(_bf16(xb), _bf16(wb), outs)
    gdn.check_device_error()
    y = np.concatenate([L.to_f64(o) for o in outs], axis=1)
    ref = oracle.linear(xb, wb)
    np.testing.assert_array_equal(y, ref)


@pytest.mark.parametrize("K", [8, 64, 72, 2560])
def test_linear_normal_inputs_within_bound(K):
    rng = np.random.default_rng(K)
    M, N = 257, 392
    xb = inputs.f32_to_bf16_bits(rng.normal(size=(M, K)).astype(np.float32))
    wb = inputs.f32_to_bf16_bits((rng.normal(size=(N, K)) / np.sqrt(K)).astype(np.float32))
    y = gdn.linear(_bf16(xb), _bf16(wb))[0]
    gdn.check_device_error()
    assert _bound_ok(L.to_f64(y), xb, wb, oracle.linear(xb, wb))


def _proj_case(T):
    return inputs.make_proj_case(T)


def test_in_proj_parity_ragged_T():
    T = 300
    pc = _proj_case(T)
    cfg = gdn.Config()
    shape = oracle.Shape(cfg.n_k_heads, cfg.n_v_heads, cfg.d_k, cfg.d_v)
    got = gdn.in_proj(cfg, _bf16(pc.hidden), _bf16(pc.w_in))
    gdn.check_device_error()
    ref = oracle.in_proj(shape, pc.hidden, pc.w_in)
    c = 0
    for name, wd in oracle.in_proj_widths(shape):
        assert tuple(got[name].shape) == (T, wd)
        assert _bound_ok(L.to_f64(got[name]), pc.hidden, pc.w_in[c:c + wd], ref[name]), name
        c += wd


def test_out_proj_parity_ragged_T():
    T = 300
    pc = _proj_case(T)
    cfg = gdn.Config()
    y = gdn.out_proj(cfg, _bf16(pc.o), _bf16(pc.w_out))
    gdn.check_device_error()
    assert tuple(y.shape) == (T, 2560)
    assert _bound_ok(L.to_f64(y), pc.o, pc.w_out, oracle.out_proj(pc.o, pc.w_out))


def test_projections_full_size_sampled_rows():
    """T = 4096 (the prefill workload's token count): both projections, checked on
    96 sampled rows (first, last and random) that the oracle computes one by one."""
    T = 4096
    pc = _proj_case(T)
    cfg = gdn.Config()
    shape = oracle.Shape(cfg.n_k_heads, cfg.n_v_heads, cfg.d_k, cfg.d_v)
    got = gdn.in_proj(cfg, _bf16(pc.hidden), _bf16(pc.w_in))
    y = gdn.out_proj(cfg, _bf16(pc.o), _bf16(pc.w_out))
    gdn.check_device_error()
    rows = np.unique(np.concatenate([[0, 127, 128, T - 1], np.random.default_rng(1).integers(0, T, 92)]))
    ref = oracle.in_proj(shape, pc.hidden[rows], pc.w_in)
    c = 0
    for name, wd in oracle.in_proj_widths(shape):
        assert _bound_ok(L.to_f64(got[name])[rows], pc.hidden[rows], pc.w_in[c:c + wd], ref[name]), name
        c += wd
    assert _bound_ok(L.to_f64(y)[rows], pc.o[rows], pc.w_out, oracle.out_proj(pc.o[rows], pc.w_out))


def test_mixer_with_projections_two_sequences():
    """hidden -> in_proj -> prefill (2 packed sequences) -> out_proj, against the oracle
    chain with the same bf16 rounding points (projection outputs and the layer output
    are stored in bf16 on both sides)."""
    T = 200
    cu = np.array([0, 77, T], np.int32)
    pc = _proj_case(T)
    case = inputs.make_case("prefill_4k", T=T, seed=3)
    cfg = gdn.Config()
    shape = L.shape_of(case)
    w = L.weights_on(case, DEV)
    p = gdn.in_proj(cfg, _bf16(pc.hidden), _bf16(pc.w_in))
    cs = torch.zeros((2, case.channels, 3), dtype=torch.bfloat16, device=DEV)
    rs = torch.zeros((2, case.n_v_heads, case.d_v, case.d_k), dtype=torch.float32, device=DEV)
    out = gdn.prefill(cfg, w, p["q"], p["k"], p["v"], p["a"], p["b"], p["z"], cs, rs,
                      torch.from_numpy(cu).to(DEV))
    y = gdn.out_proj(cfg, out, _bf16(pc.w_out))
    gdn.check_device_error()

    r_in = {n: inputs.f32_to_bf16_bits(x.astype(np.float32)) for n, x in oracle.in_proj(shape, pc.hidden, pc.w_in).items()}
    r = oracle.forward(shape, case.weights, *[r_in[n] for n in "qkvabz"],
                       np.zeros((2, case.channels, 3)), np.zeros((2, case.n_v_heads, case.d_v, case.d_k)), cu)
    o_bits = inputs.f32_to_bf16_bits(r["out"].reshape(T, -1).astype(np.float32))
    y_ref = oracle.out_proj(o_bits, pc.w_out)
    e = L.rel_err(L.to_f64(y), y_ref)
    print("mixer with projections: y rel err %.3e (tol %.1e)" % (e, L.OUT_TOL))
    assert e <= L.OUT_TOL
    assert L.rel_err(L.to_f64(rs), r["rec_state"]) <= L.STATE_TOL
