"""Context-parallel prefill of one long sequence over the ranks of a process group.

Every rank holds one contiguous segment of the sequence (rank order = sequence
order) and calls :func:`prefill` with it.  The steps, and the only data the ranks
exchange (``torch.distributed`` all-gathers, NCCL between GPUs):

1. the segment lengths, so that every rank takes the same path;
2. the conv halo: each rank's last K-1 input rows (q | k | v channels), which the
   next rank's short conv reads before its first token;
3. ``gdn_cp_local`` on the segment -> (P, S_loc): the segment's affine state map
   S_end = S_0 . P + S_loc;
4. the summaries (2 x H_v x 128 x 128 fp32 per rank, 6 MiB at the published
   shape), all-gathered in rank order;
5. ``gdn_cp_finish``: fold the maps of the ranks before this one onto the
   sequence's initial state, then scan and norm the segment from that state.

The long context this serves is the 262,144 tokens of "Qwen3.8-Flash-Next"
(llm-atlas-9r2), "Key facts".  All arithmetic runs in the CUDA library; this
module only moves tensors between ranks.  ``ops`` lets the host logic run with
other implementations of the two phases (the CPU tests use the fp64 oracle).
"""
from __future__ import annotations

from types import SimpleNamespace

import torch
import torch.distributed as dist

from . import gdn

CUDA_OPS = SimpleNamespace(local=gdn.cp_local, finish=gdn.cp_finish)


def _all_gather(t: torch.Tensor, world: int, group) -> list:
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return parts


def prefill(cfg: gdn.Config, w: dict, q, k, v, a, b, z, conv_state, rec_state, group=None, ops=None):
    """Run on every rank with its segment: q, k [T_seg, H_k*d_k], v, z [T_seg, H_v*d_v],
    a, b [T_seg, H_v]; conv_state [C, K-1] and rec_state [H_v, d_v, d_k] are the states
    before the whole sequence (the same on every rank).

    Returns (out [T_seg, H_v*d_v], state after this segment [H_v, d_v, d_k], conv state
    after this segment [C, K-1]); on the last rank these are the sequence's final states.
    Every segment needs at least K-1 rows (ValueError on every rank otherwise)."""
    ops = ops or CUDA_OPS
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T = q.shape[0]
    K1 = conv_state.shape[-1]
    lens = _all_gather(torch.tensor([T], dtype=torch.int64, device=q.device), world, group)
    if min(int(x.item()) for x in lens) < K1:
        raise ValueError("every segment needs at least %d rows, got %s" % (K1, [int(x.item()) for x in lens]))
    # conv halo, in conv_state layout: [C, K-1], oldest row first
    tail = torch.cat([x.reshape(T, -1)[T - K1:] for x in (q, k, v)], dim=1).t().contiguous()
    tails = _all_gather(tail, world, group)
    cs = (conv_state if rank == 0 else tails[rank - 1]).clone()
    summary, ws = ops.local(cfg, w, q, k, v, a, b, cs)
    summaries = torch.stack(_all_gather(summary, world, group))
    out, state = ops.finish(cfg, w, z, summaries, rank, rec_state, ws)
    return out, state, cs
