"""The Python binding's own checks (CPU only): shapes, dtypes and layouts are refused
before anything reaches the device, and the library's synchronous argument errors
come back as GdnError with their status.  A stand-in stream handle (0) lets calls
reach the library's checks on a machine without a GPU; every call here fails those
checks before any launch."""
import types

import pytest
import torch

from hybrid_linear_attention_mixer_b200 import build, gdn

NULL_STREAM = types.SimpleNamespace(cuda_stream=0)
INVALID, UNSUPPORTED = 1, 2


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return gdn.lib()


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_linear_shapes_and_segments():
    x, w = bf16(4, 16), bf16(24, 16)
    with pytest.raises(ValueError):
        gdn.linear(x, bf16(24, 8), stream=NULL_STREAM)                      # K differs
    with pytest.raises(ValueError):
        gdn.linear(x, w, outs=[bf16(4, 8)] * 9, stream=NULL_STREAM)          # too many segments
    with pytest.raises(ValueError):
        gdn.linear(x, w, outs=[bf16(5, 24)], stream=NULL_STREAM)             # rows differ
    with pytest.raises(TypeError):
        gdn.linear(x.float(), w, stream=NULL_STREAM)
    with pytest.raises(gdn.GdnError) as e:
        gdn.linear(x, w, outs=[bf16(4, 8), bf16(4, 8)], stream=NULL_STREAM)  # widths add to 16, not 24
    assert e.value.status == INVALID
    with pytest.raises(gdn.GdnError) as e:
        gdn.linear(x, bf16(20, 16), stream=NULL_STREAM)                      # N not a multiple of 8
    assert e.value.status == UNSUPPORTED


def test_projection_shapes():
    cfg = gdn.Config()
    with pytest.raises(ValueError):
        gdn.in_proj(cfg, bf16(4, 2560), bf16(16480, 2048), stream=NULL_STREAM)
    with pytest.raises(ValueError):
        gdn.in_proj(cfg, bf16(4, 2560), bf16(16479, 2560), stream=NULL_STREAM)
    bad_out = {n: bf16(4, 8) for n in "qkvzab"}
    with pytest.raises(ValueError):
        gdn.in_proj(cfg, bf16(4, 2560), bf16(16480, 2560), out=bad_out, stream=NULL_STREAM)
    with pytest.raises(ValueError):
        gdn.out_proj(cfg, bf16(4, 6144), bf16(2560, 4096), stream=NULL_STREAM)


def test_decode_multi_rows_must_split_into_tokens():
    cfg = gdn.Config()
    q = bf16(6, 16, 128)
    with pytest.raises(ValueError):
        gdn.decode_multi(cfg, {}, q, q, bf16(6, 48, 128), bf16(6, 48), bf16(6, 48), bf16(6, 48, 128),
                         bf16(1, 10240, 3), torch.zeros(1, 48, 128, 128), 4, stream=NULL_STREAM)


def test_prefill_host_checks_host_tensors():
    cfg = gdn.Config()
    T = 8
    host = {"q": bf16(T, 2048), "k": bf16(T, 2048), "v": bf16(T, 6144), "a": bf16(T, 48), "b": bf16(T, 48),
            "z": bf16(T, 6144), "cu_seqlens": torch.tensor([0, T], dtype=torch.int32), "out": bf16(T, 6144)}
    cs, rs = bf16(1, 10240, 3), torch.zeros(1, 48, 128, 128)
    with pytest.raises(TypeError):
        gdn.prefill_host(cfg, {}, dict(host, q=host["q"].float()), cs, rs, workspace=torch.empty(0),
                         stream=NULL_STREAM)
    with pytest.raises(TypeError):
        gdn.prefill_host(cfg, {}, dict(host, cu_seqlens=host["cu_seqlens"].long()), cs, rs,
                         workspace=torch.empty(0), stream=NULL_STREAM)
    with pytest.raises(ValueError):
        gdn.prefill_host(cfg, {}, dict(host, v=bf16(6144, T).t()), cs, rs, workspace=torch.empty(0),
                         stream=NULL_STREAM)


def test_context_parallel_dtypes():
    cfg = gdn.Config()
    T = 8
    q = bf16(T, 2048)
    with pytest.raises(TypeError):
        gdn.cp_local(cfg, {}, q, q, bf16(T, 6144), bf16(T, 48), bf16(T, 48), torch.zeros(10240, 3),
                     workspace=torch.empty(0), summary=torch.empty(0), stream=NULL_STREAM)
    with pytest.raises(TypeError):
        gdn.cp_finish(cfg, {}, bf16(T, 6144), torch.zeros(2, 2, 48, 128, 128, dtype=torch.float64), 0,
                      torch.zeros(48, 128, 128), torch.empty(0), stream=NULL_STREAM)
