"""Top-K selection of one sequence whose context is split over several devices.

A long sequence's context is cut into contiguous blocks, one per rank. Each rank takes the
top-k of its own block as (score, global index) candidates; the ranks exchange the candidates
with one all-gather; every rank then merges them identically. Every token of the sequence's
top-k lies in some block's top-k, and the candidates are concatenated in block order, so
position order is index order and the merge's lower-position tie-break is the lower-index rule:
the result equals the single-device top-K (aitualizate.com TokenGate article, phase 2: the K
highest-scoring context tokens; the question tail is always kept).

The per-block and merge steps run in the library's kernels (tg_topk_candidates,
tg_topk_merge); torch.distributed only moves the candidates. The two steps can be replaced
(``candidates_fn``, ``merge_fn``) so that the exchange logic can run on CPU process groups.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple


def block_bounds(n_ctx: int, world: int, rank: int) -> Tuple[int, int]:
    """Context positions [lo, hi) of ``rank``'s block: contiguous, sizes differing by at most 1."""
    if world < 1 or not 0 <= rank < world or n_ctx < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and n_ctx >= 0")
    q, r = divmod(n_ctx, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def candidate_counts(n_ctx: int, world: int, k: int) -> List[int]:
    """Candidates each rank contributes: min(k, its block size)."""
    out = []
    for rank in range(world):
        lo, hi = block_bounds(n_ctx, world, rank)
        out.append(min(max(int(k), 0), hi - lo))
    return out


def merge_gathered(cand_score, cand_idx, counts: Sequence[int], stride: int, k: int, q_start: int, q: int,
                   merge_fn: Optional[Callable] = None):
    """Merge candidates gathered as ``len(counts)`` slots of ``stride`` entries, slot r holding
    ``counts[r]`` real candidates first: the real ones are compacted in slot order (device
    copies), then merged. Returns the kept indices (top-k context indices ascending, then the
    question tail q_start .. q_start + q - 1)."""
    import torch

    parts_s = [cand_score[r * stride: r * stride + c] for r, c in enumerate(counts) if c > 0]
    parts_i = [cand_idx[r * stride: r * stride + c] for r, c in enumerate(counts) if c > 0]
    if parts_s:
        s = torch.cat(parts_s)
        i = torch.cat(parts_i)
    else:
        s = cand_score[:0]
        i = cand_idx[:0]
    if merge_fn is None:
        import learned_token_pruning_02_b200 as tg

        return tg.tg_topk_merge(s, i, k, q_start, q)
    return merge_fn(s, i, k, q_start, q)


def split_select(score_block, rank: int, world: int, n_ctx: int, q: int, k: int, group=None,
                 candidates_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """Top-K of one sequence whose context scores are split over ``world`` ranks.

    score_block: this rank's scores for its block (``block_bounds``), a 1-D float32 tensor.
    The question tail is the q tokens after the context (indices n_ctx .. n_ctx + q - 1).
    Returns kept indices within the sequence, identical on every rank.
    """
    import torch
    import torch.distributed as dist

    lo, hi = block_bounds(n_ctx, world, rank)
    if score_block.numel() != hi - lo:
        raise ValueError(f"rank {rank} holds {score_block.numel()} scores, its block has {hi - lo}")
    counts = candidate_counts(n_ctx, world, k)
    stride = max(max(counts), 1)
    if candidates_fn is None:
        import learned_token_pruning_02_b200 as tg

        cs, ci = tg.tg_topk_candidates(score_block, k, base=lo)
    else:
        cs, ci = candidates_fn(score_block, k, lo)
    send_s = torch.zeros(stride, dtype=torch.float32, device=score_block.device)
    send_i = torch.zeros(stride, dtype=torch.int32, device=score_block.device)
    send_s[: counts[rank]] = cs
    send_i[: counts[rank]] = ci
    if world > 1:
        got_s = [torch.empty_like(send_s) for _ in range(world)]
        got_i = [torch.empty_like(send_i) for _ in range(world)]
        dist.all_gather(got_s, send_s, group=group)
        dist.all_gather(got_i, send_i, group=group)
        all_s, all_i = torch.cat(got_s), torch.cat(got_i)
    else:
        all_s, all_i = send_s, send_i
    return merge_gathered(all_s, all_i, counts, stride, k, n_ctx, q, merge_fn=merge_fn)
