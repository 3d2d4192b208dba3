"""Sequence-parallel prefill: one long sequence split into contiguous segments, one per rank.

The prefix state of eq. (4) ("OAL: 按 QK 离群贡献分组的正二次注意力核", section 核心公式) is a sum
over tokens, so the state a rank must start from is the sum of the segment states of the ranks
before it.  Each rank
  1. computes the state of its own segment alone (a prefill without outputs),
  2. all-gathers the segment states (the one exchange step: B*Hkv*2176*65 fp32 per rank,
     1.1 MB for one Qwen2.5-0.5B layer, independent of the sequence length),
  3. writes the sum of the earlier ranks' states into its state buffer (oal_state_prefix_sum)
     and continues its segment from there (oal_prefill_continue),
which yields its tokens' outputs and the prefix state after its segment (the last rank holds
the state of the whole sequence, ready for decode).

The backend performs the local operations (segment state, state access, combine, continue);
the default one is this library on the rank's GPU.  Ranks are torch.distributed ranks (NCCL on GPUs); `allgather` may be replaced
(e.g. to run the ranks of one process for testing).
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch


class LibraryBackend:
    """The three local steps on this library (bf16, chunk 128)."""

    def __init__(self, Hq: int):
        from . import oal
        self.oal = oal
        self.Hq = Hq

    def segment_state(self, k, v, group_id, L, G, eps):
        return self.oal.prefill_state(k, v, group_id, L, G, eps, self.Hq)

    def body(self, state, B, Hkv):
        return self.oal.state_body(state, B, self.Hq, Hkv)

    def set_tokens(self, state, tokens):
        self.oal.set_state_tokens(state, tokens)

    def combine(self, parts, n_parts, body):
        """body = parts[0] + ... + parts[n_parts - 1], in the library (fixed order)."""
        self.oal.state_prefix_sum(parts, n_parts, body)

    def continue_from(self, q, k, v, group_id, L, G, eps, state):
        return self.oal.prefill_continue(q, k, v, group_id, L, G, eps, state)


def _dist_allgather(group):
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> Sequence[torch.Tensor]:
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return parts
    return gather


def sequence_parallel_prefill(q, k, v, group_id, L, G, eps: float, *, rank: int, world: int,
                              tokens_before: int, backend=None,
                              allgather: Optional[Callable] = None, group=None):
    """Prefill of this rank's segment (q [B,Hq,Ts,64], k/v [B,Hkv,Ts,64]) of a sequence whose
    earlier segments (tokens_before tokens in all) live on ranks 0..rank-1.

    Returns (out [B,Hq,Ts,64] fp32, state): out holds yhat of this segment's tokens given the
    whole prefix, state the prefix state after this segment."""
    B, Hq = q.shape[0], q.shape[1]
    Hkv = k.shape[1]
    if backend is None:
        backend = LibraryBackend(Hq)
    if allgather is None:
        allgather = _dist_allgather(group)
    state = backend.segment_state(k, v, group_id, L, G, eps)
    body = backend.body(state, B, Hkv)
    parts = allgather(body.clone())
    if len(parts) != world:
        raise RuntimeError(f"all-gather returned {len(parts)} parts for {world} ranks")
    if isinstance(parts, (list, tuple)):
        parts = torch.stack(list(parts))  # one [world, n] buffer
    backend.combine(parts, rank, body)
    backend.set_tokens(state, tokens_before)
    out = backend.continue_from(q, k, v, group_id, L, G, eps, state)
    return out, state
