"""Seeded synthetic inputs for the Gated DeltaNet mixer.

This module only draws random numbers and rounds them to the storage type.  It
holds none of the layer's arithmetic, and both the CUDA path's tests and the
fp64 oracle take their inputs from it.

Activations are returned as numpy arrays: ``uint16`` arrays hold bf16 bit
patterns (round-to-nearest-even from float32), ``float32`` arrays hold fp32
activations.  Parameters are float32.  Every tensor is drawn from its own
PCG64 stream keyed by (seed, tensor name, row block), so that any row block
can be regenerated on its own and the draw does not depend on the order in
which tensors are made.

Workloads (head shape of the layer: 16 key heads, 48 value heads, d_k = d_v =
128, conv kernel 4 -- "Qwen3.8-Flash-Next" (llm-architectures-explained),
"Every architecture field"):

* ``tiny``        1 sequence, T = 64, 2 key / 6 value heads of dim 32, fp32
                  activations, alpha ~ U[0.9, 0.999], zero states, seed 0.
* ``prefill_4k``  1 sequence, T = 4096, bf16, zero states.
* ``varlen_8``    8 sequences, lengths ~ U{512..16384}, bf16, zero states.
* ``decode_256``  256 sequences x 1 token, fp32 state ~ N(0, 0.02) (std),
                  bf16 conv state; 64 consecutive steps.
* ``prefill_256k`` 1 sequence, T = 262144, -log alpha ~ U(1e-4, 0.1).

Projections around the mixer (``make_proj_case``): hidden states [T, 2560]
bf16 ~ N(0, 1) (hidden size 2,560: "Qwen3.8-Flash-Next" (llm-atlas-9r2), "Key
facts"); random-init bf16 weights w_in [16480, 2560] ~ N(0, 1/2560) and w_out
[2560, 6144] ~ N(0, 1/6144), so that every projected channel is ~ N(0, 1) like
the mixer's own synthetic inputs.
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

ROW_BLOCK = 1024


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even.  Finite inputs."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, name: str, block: int = 0) -> np.random.Generator:
    key = zlib.crc32(name.encode())
    return np.random.Generator(np.random.PCG64([seed, key, block]))


def _workers() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _normal_rows(seed, name, rows, cols, std=1.0, mean=0.0, bf16=True):
    """[rows, cols] N(mean, std^2), drawn in independent row blocks (threaded)."""
    out = np.empty((rows, cols), dtype=np.uint16 if bf16 else np.float32)

    def fill(blk):
        r0 = blk * ROW_BLOCK
        r1 = min(rows, r0 + ROW_BLOCK)
        x = _rng(seed, name, blk).standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0 or mean != 0.0:
            x = x * np.float32(std) + np.float32(mean)
        out[r0:r1] = f32_to_bf16_bits(x) if bf16 else x

    nblk = (rows + ROW_BLOCK - 1) // ROW_BLOCK
    if nblk <= 1:
        for blk in range(nblk):
            fill(blk)
    else:
        with ThreadPoolExecutor(min(_workers(), nblk)) as ex:
            list(ex.map(fill, range(nblk)))
    return out


def _inv_softplus_of_neg_log_alpha(neg_log_alpha: np.ndarray) -> np.ndarray:
    """a such that softplus(a) = -log(alpha): a = log(expm1(-log alpha)).

    With A_log = 0 and dt_bias = 0 the gate then reproduces the drawn alpha
    (up to the rounding of a to the activation type)."""
    return np.log(np.expm1(neg_log_alpha.astype(np.float64)))


@dataclass
class Case:
    name: str
    n_k_heads: int
    n_v_heads: int
    d_k: int
    d_v: int
    conv_kernel: int
    chunk: int
    bf16: bool                    # activations bf16 (else fp32)
    cu_seqlens: np.ndarray        # int32 [N+1]
    weights: dict                 # conv_w [C,K], A_log [Hv], dt_bias [Hv], norm_w [dv] (fp32)
    acts: dict                    # q,k [T,Hk*dk]; v,z [T,Hv*dv]; a,b [T,Hv]
    conv_state: np.ndarray        # [N, C, K-1] (uint16 bf16 or float32)
    rec_state: np.ndarray         # [N, Hv, dv, dk] float32
    l2_eps: float = 1e-6
    norm_eps: float = 1e-6
    steps: list = field(default_factory=list)   # decode: per-step activation dicts

    @property
    def channels(self) -> int:
        return 2 * self.n_k_heads * self.d_k + self.n_v_heads * self.d_v

    @property
    def n_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])


def _weights(seed, Hk, Hv, dk, dv, K, gates="model"):
    C = 2 * Hk * dk + Hv * dv
    w = {
        # no trained weights exist: conv taps ~ N(0, 1/4), norm weight 1 + 0.1 N(0,1)
        "conv_w": _rng(seed, "conv_w").standard_normal((C, K), dtype=np.float32) * np.float32(0.5),
        "norm_w": (1.0 + 0.1 * _rng(seed, "norm_w").standard_normal(dv)).astype(np.float32),
    }
    if gates == "model":
        w["A_log"] = _rng(seed, "A_log").uniform(0.0, 2.7, Hv).astype(np.float32)
        w["dt_bias"] = (0.1 * _rng(seed, "dt_bias").standard_normal(Hv)).astype(np.float32)
    else:  # alpha drawn directly: A_log = 0, dt_bias = 0
        w["A_log"] = np.zeros(Hv, np.float32)
        w["dt_bias"] = np.zeros(Hv, np.float32)
    return w


def _acts(seed, T, Hk, Hv, dk, dv, bf16, gates, alpha_range=None, nla_range=None, prefix=""):
    p = prefix
    acts = {
        "q": _normal_rows(seed, p + "q", T, Hk * dk, bf16=bf16),
        "k": _normal_rows(seed, p + "k", T, Hk * dk, bf16=bf16),
        "v": _normal_rows(seed, p + "v", T, Hv * dv, bf16=bf16),
        "z": _normal_rows(seed, p + "z", T, Hv * dv, bf16=bf16),
        "b": _normal_rows(seed, p + "b", T, Hv, bf16=bf16),
    }
    if gates == "model":
        acts["a"] = _normal_rows(seed, p + "a", T, Hv, bf16=bf16)
    else:
        a = np.empty((T, Hv), dtype=np.float32)
        for blk, r0 in enumerate(range(0, T, ROW_BLOCK)):
            r1 = min(T, r0 + ROW_BLOCK)
            g = _rng(seed, p + "alpha", blk)
            if alpha_range is not None:
                nla = -np.log(g.uniform(alpha_range[0], alpha_range[1], (r1 - r0, Hv)))
            else:
                nla = g.uniform(nla_range[0], nla_range[1], (r1 - r0, Hv))
            a[r0:r1] = _inv_softplus_of_neg_log_alpha(nla).astype(np.float32)
        acts["a"] = f32_to_bf16_bits(a) if bf16 else a
    return acts


def make_case(name: str, seed: int | None = None, T: int | None = None,
              n_seqs: int | None = None, nla_range: tuple | None = None) -> Case:
    """Build one named workload.  ``T`` / ``n_seqs`` shrink a workload for quick runs;
    ``nla_range`` replaces the -log alpha range of ``prefill_256k``."""
    if name == "tiny":
        s = 0 if seed is None else seed
        Hk, Hv, d, K = 2, 6, 32, 4
        T = 64 if T is None else T
        w = _weights(s, Hk, Hv, d, d, K, gates="alpha")
        acts = _acts(s, T, Hk, Hv, d, d, bf16=False, gates="alpha", alpha_range=(0.9, 0.999))
        cu = np.array([0, T], np.int32)
        return Case(name, Hk, Hv, d, d, K, 16, False, cu, w, acts,
                    np.zeros((1, 2 * Hk * d + Hv * d, K - 1), np.float32),
                    np.zeros((1, Hv, d, d), np.float32))
    Hk, Hv, d, K = 16, 48, 128, 4
    C = 2 * Hk * d + Hv * d
    if name == "prefill_4k":
        s = 1 if seed is None else seed
        T = 4096 if T is None else T
        w = _weights(s, Hk, Hv, d, d, K)
        acts = _acts(s, T, Hk, Hv, d, d, True, "model")
        cu = np.array([0, T], np.int32)
        return Case(name, Hk, Hv, d, d, K, 64, True, cu, w, acts,
                    np.zeros((1, C, K - 1), np.uint16), np.zeros((1, Hv, d, d), np.float32))
    if name == "varlen_8":
        s = 2 if seed is None else seed
        N = 8 if n_seqs is None else n_seqs
        lens = _rng(s, "lengths").integers(512, 16384, N, endpoint=True)
        if T is not None:   # shrink: scale lengths so that they sum to about T
            lens = np.maximum(1, (lens * (T / lens.sum())).astype(np.int64))
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        w = _weights(s, Hk, Hv, d, d, K)
        acts = _acts(s, int(cu[-1]), Hk, Hv, d, d, True, "model")
        return Case(name, Hk, Hv, d, d, K, 64, True, cu, w, acts,
                    np.zeros((N, C, K - 1), np.uint16), np.zeros((N, Hv, d, d), np.float32))
    if name == "decode_256":
        s = 3 if seed is None else seed
        N = 256 if n_seqs is None else n_seqs
        steps = 64 if T is None else T
        w = _weights(s, Hk, Hv, d, d, K)
        cu = np.arange(N + 1, dtype=np.int32)
        step_acts = [_acts(s, N, Hk, Hv, d, d, True, "model", prefix="step%d/" % i)
                     for i in range(steps)]
        rec = np.empty((N, Hv, d, d), np.float32)
        flat = rec.reshape(N * Hv, d * d)
        for blk, r0 in enumerate(range(0, N * Hv, ROW_BLOCK)):
            r1 = min(N * Hv, r0 + ROW_BLOCK)
            flat[r0:r1] = _rng(s, "rec_state", blk).standard_normal((r1 - r0, d * d),
                                                                     dtype=np.float32) * np.float32(0.02)
        conv = _normal_rows(s, "conv_state", N, C * (K - 1)).reshape(N, C, K - 1)
        return Case(name, Hk, Hv, d, d, K, 64, True, cu, w, step_acts[0], conv, rec,
                    steps=step_acts)
    if name == "prefill_256k":
        s = 4 if seed is None else seed
        T = 262144 if T is None else T
        w = _weights(s, Hk, Hv, d, d, K, gates="alpha")
        acts = _acts(s, T, Hk, Hv, d, d, True, "alpha", nla_range=nla_range or (1e-4, 0.1))
        cu = np.array([0, T], np.int32)
        return Case(name, Hk, Hv, d, d, K, 64, True, cu, w, acts,
                    np.zeros((1, C, K - 1), np.uint16), np.zeros((1, Hv, d, d), np.float32))
    raise KeyError(name)


CASES = ("tiny", "prefill_4k", "varlen_8", "decode_256", "prefill_256k")


@dataclass
class ProjCase:
    """Inputs of the mixer's two projections (bf16 bit patterns)."""
    hidden: np.ndarray      # [T, d_model]
    w_in: np.ndarray        # [2*Hk*dk + 2*Hv*dv + 2*Hv, d_model]
    w_out: np.ndarray       # [d_model, Hv*dv]
    o: np.ndarray           # [T, Hv*dv], a stand-in layer output for the out projection alone


def make_proj_case(T: int, d_model: int = 2560, Hk: int = 16, Hv: int = 48, dk: int = 128, dv: int = 128,
                   seed: int = 0) -> ProjCase:
    n_in = 2 * Hk * dk + 2 * Hv * dv + 2 * Hv
    return ProjCase(
        hidden=_normal_rows(seed, "proj.hidden", T, d_model),
        w_in=_normal_rows(seed, "proj.w_in", n_in, d_model, std=float(d_model) ** -0.5),
        w_out=_normal_rows(seed, "proj.w_out", d_model, Hv * dv, std=float(Hv * dv) ** -0.5),
        o=_normal_rows(seed, "proj.o", T, Hv * dv),
    )
