"""Running the gated path on several GPUs: one process per GPU, independent sequences.

The path has no exchange step between sequences (every sequence is scored, pruned and
attended on its own), so a batch spreads over GPUs by whole sequences with no data-path
collective. torch.distributed is used only for barriers and the max-over-ranks timing.
"""
from __future__ import annotations


def sequence_cost(n: int, q: int, k: int) -> float:
    """Relative device time of one sequence: the score pass is linear in N, the gated
    attention quadratic in the kept rows M = min(K, N - q) + q."""
    m = min(max(int(k), 0), int(n) - int(q)) + int(q)
    return float(n) + 0.0625 * float(m) * float(m)


def assign_sequences(seqlens, q_len, k, world: int) -> list:
    """Longest-processing-time assignment of whole sequences to `world` ranks.

    Returns one ascending list of sequence indices per rank. Deterministic: ties in cost
    go to the lower sequence index, ties in load to the lower rank.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(seqlens)), key=lambda b: (-sequence_cost(seqlens[b], q_len[b], k[b]), b))
    load = [0.0] * world
    out = [[] for _ in range(world)]
    for b in order:
        r = min(range(world), key=lambda i: (load[i], i))
        out[r].append(b)
        load[r] += sequence_cost(seqlens[b], q_len[b], k[b])
    return [sorted(x) for x in out]


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the default process group (the rank's own value when
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
