"""The C-ABI library loads and exports every symbol include/gdn.h declares, and its
host-side argument checks answer without touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

from hybrid_linear_attention_mixer_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, CUDA, TIMEOUT, WORKSPACE, SEQLENS, RANGE = range(8)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gdn.lib()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(gdn_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"gdn_prefill", "gdn_decode", "gdn_prefill_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(gdn.EXPORTS) <= set(names)


def test_default_config_is_the_published_shape(lib):
    c = gdn._CConfig()
    lib.gdn_config_default(ctypes.byref(c))
    assert (c.n_k_heads, c.n_v_heads, c.d_k, c.d_v, c.conv_kernel, c.chunk) == (16, 48, 128, 128, 4, 64)
    assert abs(c.norm_eps - 1e-6) < 1e-12 and abs(c.l2_eps - 1e-6) < 1e-12
    assert c.act_dtype == 0 and c.out_dtype == 0 and c.state_dtype == 1   # bf16 I/O, fp32 state


def test_workspace_size(lib):
    cfg = gdn.Config()
    T = 4096
    # fp16 q^, k^ [T, 16*128] and v^ [T, 48*128]; chunk offsets [N+1] and the check word,
    # int32 (256-byte rounded); per (chunk, value head) a 57 KiB intra-chunk record and a
    # [64][128] o tile of the output dtype, with at most ceil(T / 64) + N chunks
    # A call pipelined over chunk ranges (automatic for up to 2 sequences and T_total of 64
    # chunks or more; prefill_segments > 1 asks for it) adds each chain's fp32 state,
    # [N][48][128][128].
    conv = 2 * T * 2048 * 2 + T * 6144 * 2
    per_chunk = 48 * (58368 + 64 * 128 * 2)
    carry = 48 * 128 * 128 * 4
    assert gdn.workspace_size(cfg, T, 1) == conv + 256 + (T // 64 + 1) * per_chunk + carry
    # the split chain (asked for): the first half's end state, [P | S_loc], S0 in bf16, a second
    # set of o tiles and a zeroed 64-row v block
    split = 3 * carry + carry // 2 + (T // 64 + 1) * 48 * 64 * 128 * 2 + 64 * 48 * 128 * 2
    assert gdn.workspace_size(gdn.Config(prefill_segments=-1), T, 1) == conv + 256 + (T // 64 + 1) * per_chunk + split
    assert gdn.workspace_size(gdn.Config(prefill_segments=1), T, 1) == conv + 256 + (T // 64 + 1) * per_chunk
    assert gdn.workspace_size(cfg, T, 2) == conv + 256 + (T // 64 + 2) * per_chunk + 2 * carry
    assert gdn.workspace_size(cfg, T, 3) == conv + 256 + (T // 64 + 3) * per_chunk
    assert gdn.workspace_size(gdn.Config(prefill_segments=4), T, 3) == conv + 256 + (T // 64 + 3) * per_chunk + 3 * carry
    w = lambda T_, n: 2 * T_ * 2048 * 2 + T_ * 6144 * 2 + 256 + (-(-T_ // 64) + n) * per_chunk
    assert gdn.workspace_size(cfg, 4032, 2) == w(4032, 2)
    assert gdn.workspace_size(cfg, 4033, 2) == w(4033, 2) + 2 * carry
    f32 = gdn.Config(out_dtype=__import__("torch").float32)   # (no split chain with an fp32 output)
    assert gdn.workspace_size(f32, T, 1) == conv + 256 + (T // 64 + 1) * 48 * (58368 + 64 * 128 * 4) + carry
    assert gdn.workspace_size(cfg, T, 63) == conv + 512 + (T // 64 + 63) * per_chunk
    assert gdn.workspace_size(cfg, 0, 0) == 256
    assert gdn.workspace_size(gdn.Config(d_k=48), T, 1) == 0
    assert gdn.workspace_size(gdn.Config(prefill_segments=-2), T, 1) == 0
    assert gdn.workspace_size(gdn.Config(prefill_segments=33), T, 1) == 0


def test_prefill_segments_plan(lib):
    cfg = gdn.Config()
    SPLIT = -1
    # automatic: at most 8 ranges of at least 32 chunks for at most 96 chains (2 sequences of 48 heads)
    assert gdn.prefill_segments(cfg, 4096, 1) == 2
    assert gdn.prefill_segments(cfg, 4032, 1) == 1 and gdn.prefill_segments(cfg, 4033, 1) == 2
    assert gdn.prefill_segments(cfg, 4096, 2) == 2
    assert gdn.prefill_segments(cfg, 4096, 3) == 1
    assert gdn.prefill_segments(cfg, 4032, 2) == 1 and gdn.prefill_segments(cfg, 4033, 2) == 2
    assert gdn.prefill_segments(cfg, 16384, 1) == 8
    assert gdn.prefill_segments(cfg, 262144, 1) == 8
    assert gdn.prefill_segments(cfg, 0, 0) == 1
    # asked for: the split chain where it applies (one sequence, published head size, bf16 in and
    # out, fp32 state), else one range
    assert gdn.prefill_segments(gdn.Config(prefill_segments=SPLIT), 200, 1) == SPLIT
    assert gdn.prefill_segments(gdn.Config(prefill_segments=SPLIT), 64, 1) == 1
    assert gdn.prefill_segments(gdn.Config(prefill_segments=SPLIT), 4096, 2) == 1
    import torch
    assert gdn.prefill_segments(gdn.Config(prefill_segments=SPLIT, state_dtype=torch.bfloat16), 4096, 1) == 1
    assert gdn.prefill_segments(gdn.Config(prefill_segments=SPLIT, d_k=64, d_v=64), 4096, 1) == 1
    # asked for: ranges of ceil(chunks / n) chunks, never more ranges than chunks
    assert gdn.prefill_segments(gdn.Config(prefill_segments=7), 4096, 1) == 7
    assert gdn.prefill_segments(gdn.Config(prefill_segments=32), 4096, 5) == 32
    assert gdn.prefill_segments(gdn.Config(prefill_segments=3), 100, 1) == 2
    assert gdn.prefill_segments(gdn.Config(prefill_segments=1), 262144, 1) == 1
    assert gdn.prefill_segments(gdn.Config(prefill_segments=33), 4096, 1) == 0


def _call_prefill(lib, cfg, w=True, ptr=0x1000, T=16, n=1, ws_bytes=1 << 30, ws=0x100000):
    c = cfg.c()
    cw = gdn._CWeights(0x2000, 0x3000, 0x4000, 0x5000) if w else None
    P = ctypes.c_void_p
    ptrs = [P(ptr)] * 8
    return lib.gdn_prefill(ctypes.byref(c), ctypes.byref(cw) if cw else None, *ptrs, P(0x6000), n, T,
                           P(0x7000), P(ws), ws_bytes, None)


def test_argument_errors_are_synchronous_and_launch_nothing(lib):
    cfg = gdn.Config()
    assert _call_prefill(lib, cfg, w=False) == INVALID
    assert _call_prefill(lib, gdn.Config(d_k=48)) == UNSUPPORTED
    assert _call_prefill(lib, gdn.Config(n_k_heads=5)) == UNSUPPORTED
    assert _call_prefill(lib, gdn.Config(conv_kernel=3)) == UNSUPPORTED
    assert _call_prefill(lib, gdn.Config(chunk=32)) == UNSUPPORTED
    bad = gdn.Config().c()
    bad.state_dtype = 7
    assert lib.gdn_prefill_workspace_size(ctypes.byref(bad), 16, 1) == 0   # invalid config
    assert _call_prefill(lib, cfg, ptr=0x1001) == INVALID          # misaligned activation
    assert _call_prefill(lib, cfg, ws=0x100010) == INVALID         # workspace not 256-aligned
    assert _call_prefill(lib, cfg, ws_bytes=1000) == WORKSPACE
    assert _call_prefill(lib, cfg, T=0) == OK                      # nothing to do
    assert _call_prefill(lib, cfg, n=-1) == INVALID
    c = cfg.c()
    cw = gdn._CWeights(0x2000, 0x3000, 0x4000, 0x5000)
    P = ctypes.c_void_p
    assert lib.gdn_decode(ctypes.byref(c), ctypes.byref(cw), *[P(0)] * 8, 4, P(0x7000), None) == INVALID
    assert lib.gdn_decode(ctypes.byref(c), ctypes.byref(cw), *[P(0x1000)] * 8, 0, P(0x7000), None) == OK
    assert lib.gdn_decode(None, ctypes.byref(cw), *[P(0x1000)] * 8, 4, P(0x7000), None) == INVALID


def test_decode_multi_argument_errors(lib):
    c = gdn.Config().c()
    cw = gdn._CWeights(0x2000, 0x3000, 0x4000, 0x5000)
    P = ctypes.c_void_p
    call = lambda n, k, snap=0, ptr=0x1000: lib.gdn_decode_multi(
        ctypes.byref(c), ctypes.byref(cw), *[P(ptr)] * 8, n, k, P(0x7000), P(snap), None, None)
    assert call(4, gdn.DECODE_MULTI_MAX_TOKENS + 1) == UNSUPPORTED
    assert call(4, -1) == INVALID
    assert call(-1, 2) == INVALID
    assert call(4, 0) == OK and call(0, 3) == OK          # nothing to do
    assert call(4, 2, snap=0x8008) == INVALID             # misaligned snapshots
    assert call(4, 2, ptr=0) == INVALID                   # missing inputs


def test_linear_argument_errors(lib):
    P = ctypes.c_void_p

    def segs(*widths, ptr=0x10000):
        return (gdn._CSegment * len(widths))(*[gdn._CSegment(ptr, w) for w in widths])

    call = lambda M, N, K, sg, n=None, x=0x1000, w=0x2000: lib.gdn_linear(
        P(x), P(w), M, N, K, sg, len(sg) if n is None else n, None)
    assert call(-1, 64, 64, segs(64)) == INVALID
    assert call(4, 0, 64, segs(64)) == INVALID
    assert call(4, 64, 64, segs(8, 8, 8, 8, 8, 8, 8, 8, 8), n=9) == UNSUPPORTED
    assert call(4, 12, 64, segs(12)) == UNSUPPORTED       # N not a multiple of 8
    assert call(4, 64, 20, segs(64)) == UNSUPPORTED       # K not a multiple of 8
    assert call(0, 64, 64, segs(64)) == OK                # nothing to do
    assert call(4, 64, 64, segs(32, 16)) == INVALID       # widths do not add up to N
    assert call(4, 64, 64, segs(60, 4)) == INVALID        # width not a multiple of 8
    assert call(4, 64, 64, segs(64, ptr=0x10008)) == INVALID   # misaligned output
    assert call(4, 64, 64, segs(64), x=0x1004) == INVALID       # misaligned x
    assert call(4, 64, 64, segs(64), w=0) == INVALID
    c = gdn.Config(n_k_heads=2, n_v_heads=6, d_k=32, d_v=32).c()
    assert lib.gdn_in_proj(ctypes.byref(c), P(0x1000), P(0x2000), 4, 64, *[P(0x3000)] * 6, None) == UNSUPPORTED
    c = gdn.Config().c()
    assert lib.gdn_in_proj(ctypes.byref(c), P(0x1000), P(0x2000), 0, 2560, *[P(0x3000)] * 6, None) == OK
    assert lib.gdn_in_proj(ctypes.byref(c), P(0x1000), P(0x2000), 4, 2564, *[P(0x3000)] * 6, None) == UNSUPPORTED
    assert lib.gdn_out_proj(ctypes.byref(c), P(0x1000), P(0x2000), 0, 2560, P(0x3000), None) == OK
    assert lib.gdn_out_proj(ctypes.byref(c), P(0x1000), P(0x2000), -1, 2560, P(0x3000), None) == INVALID


def test_cp_argument_errors(lib):
    P = ctypes.c_void_p
    cw = gdn._CWeights(0x2000, 0x3000, 0x4000, 0x5000)
    c = gdn.Config().c()
    assert lib.gdn_cp_workspace_size(ctypes.byref(c), 4096) > gdn.workspace_size(gdn.Config(), 4096, 1)
    assert lib.gdn_cp_workspace_size(ctypes.byref(c), 0) == 0
    local = lambda cfg, T, ws=1 << 40, p=0x1000: lib.gdn_cp_local(
        ctypes.byref(cfg), ctypes.byref(cw), *[P(p)] * 5, P(0x6000), T, P(0x7000), P(0x100000), ws, None)
    assert local(c, 0) == INVALID
    assert local(c, 64, p=0) == INVALID
    assert local(c, 64, ws=1024) == WORKSPACE
    cb = gdn.Config(state_dtype=torch.bfloat16).c()
    assert local(cb, 64) == UNSUPPORTED                   # the maps need an fp32 state
    cd = gdn.Config(d_k=64, d_v=128).c()
    assert local(cd, 64) == UNSUPPORTED                   # P has the state's shape only when d_k == d_v
    fin = lambda n, r, ws=1 << 40: lib.gdn_cp_finish(
        ctypes.byref(c), ctypes.byref(cw), P(0x1000), P(0x2000), n, r, P(0x3000), 64, P(0x4000), P(0x5000),
        P(0x100000), ws, None)
    assert fin(2, 2) == INVALID and fin(2, -1) == INVALID and fin(0, 0) == INVALID
    assert fin(2, 1, ws=1024) == WORKSPACE


def test_prefill_host_argument_errors(lib):
    """gdn_prefill_host reads cu_seqlens on the host: bad offsets are refused before any launch."""
    P = ctypes.c_void_p
    cw = gdn._CWeights(0x2000, 0x3000, 0x4000, 0x5000)
    c = gdn.Config().c()
    size = lib.gdn_prefill_host_workspace_size(ctypes.byref(c), 4096, 2)
    assert size > gdn.workspace_size(gdn.Config(), 512, 2)

    def call(cu, T, ws=1 << 40):
        arr = (ctypes.c_int32 * len(cu))(*cu)
        return lib.gdn_prefill_host(ctypes.byref(c), ctypes.byref(cw), *[P(0x1000)] * 6, P(0x6000), P(0x7000),
                                    arr, len(cu) - 1, T, P(0x8000), P(0x100000), ws, None)
    assert call([1, 10, 20], 20) == INVALID          # does not start at 0
    assert call([0, 12, 10], 10) == INVALID          # decreasing
    assert call([0, 10, 20], 21) == INVALID          # does not end at T
    assert call([0, 10, 20], 20, ws=4096) == WORKSPACE
    assert call([0], 0) == OK                        # nothing to do


def test_status_strings(lib):
    names = {gdn.status_string(s) for s in range(8)}
    assert len(names) == 8 and "unknown status" not in names
    assert gdn.status_string(99) == "unknown status"


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "LIB_PATH", "/nonexistent/libgdn_b200.so")
    with pytest.raises(RuntimeError):
        gdn.lib()
