"""Top-K of one sequence split over ranks: every rank takes its block's top-k as candidates,
the candidates are all-gathered, every rank merges them. The result must equal the top-K of
the whole sequence exactly (ties to the lower index, NaN below -inf, question tail kept).

CPU part: the exchange logic on gloo process groups (world 2 and 3), with the per-block and
merge steps done by the oracle's top-K. GPU part: the library's kernels for both steps, the
ranks emulated in one process (a gather is a concatenation), checked bit for bit against
tg_topk_select on the whole sequence and against the oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from learned_token_pruning_02_b200 import split

CASES = [  # (n_ctx, q, k, kind)
    (1000, 24, 100, "normal"),
    (1001, 0, 400, "ties"),      # blocks of 334 / 334 / 333 < k for world 3
    (999, 7, 999, "normal"),     # k = n_ctx: everything
    (1000, 5, 0, "normal"),      # only the question tail
    (777, 3, 50, "nan"),         # NaN and -inf and -0 among the scores
    (50, 2, 45, "nan"),          # k larger than the number of finite scores
]


def _scores(n, kind, seed):
    g = np.random.default_rng(seed)
    s = g.standard_normal(n).astype(np.float32)
    if kind == "ties":
        s = np.round(s * 2).astype(np.float32)
    elif kind == "nan":
        s[g.random(n) < 0.1] = np.nan
        s[g.random(n) < 0.05] = -np.inf
        s[g.random(n) < 0.05] = -0.0
    return s


def test_block_bounds_partition():
    for n in (0, 1, 7, 1000, 1001):
        for world in (1, 2, 3, 8):
            b = [split.block_bounds(n, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            assert max(h - l for l, h in b) - min(h - l for l, h in b) <= 1
    assert split.candidate_counts(1001, 3, 400) == [334, 334, 333]
    assert split.candidate_counts(1000, 4, 100) == [100] * 4


def _oracle_candidates(block, k, lo):
    from oracle import tg_oracle as orc

    n = block.numel()
    kept, _ = orc.topk_select(block.numpy(), [n], [0], [k])
    kept = np.asarray(kept, dtype=np.int64)
    return block[torch.from_numpy(kept)], torch.from_numpy((kept + lo).astype(np.int32))


def _oracle_merge(s, i, k, q_start, q):
    from oracle import tg_oracle as orc

    n = s.numel()
    pos, _ = orc.topk_select(s.numpy(), [n], [0], [k])
    ctx = i[torch.from_numpy(np.asarray(pos, dtype=np.int64))]
    return torch.cat([ctx, torch.arange(q_start, q_start + q, dtype=torch.int32)])


def _free_port():
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    p = sk.getsockname()[1]
    sk.close()
    return p


def _worker(rank, world, port, ret):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = []
        for ci, (n_ctx, q, k, kind) in enumerate(CASES):
            s = torch.from_numpy(_scores(n_ctx + q, kind, ci))
            lo, hi = split.block_bounds(n_ctx, world, rank)
            kept = split.split_select(s[lo:hi].clone(), rank, world, n_ctx, q, k,
                                      candidates_fn=_oracle_candidates, merge_fn=_oracle_merge)
            out.append(kept.tolist())
        gathered = [None] * world
        dist.all_gather_object(gathered, out)
        if rank == 0:
            ret["kept"] = gathered
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_split_select_equals_whole_sequence_gloo(world):
    from oracle import tg_oracle as orc

    ctx = mp.get_context("spawn")
    ret = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), ret), nprocs=world, join=True, start_method="spawn")
    for r in range(world):  # every rank holds the same result
        assert ret["kept"][r] == ret["kept"][0]
    for ci, (n_ctx, q, k, kind) in enumerate(CASES):
        s = _scores(n_ctx + q, kind, ci)
        ref, _ = orc.topk_select(s, [n_ctx + q], [q], [k])
        assert ret["kept"][0][ci] == [int(x) for x in ref], (world, ci)


@pytest.mark.gpu
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_split_select_kernels_equal_select_gpu(world):
    """Both steps on the GPU; the all-gather of the ranks is a concatenation here."""
    import learned_token_pruning_02_b200 as tg
    from oracle import tg_oracle as orc

    cases = CASES + [(131072 - 256, 256, 4096, "ties"), (200000, 64, 60000, "normal")]
    for ci, (n_ctx, q, k, kind) in enumerate(cases):
        s = _scores(n_ctx + q, kind, 100 + ci)
        sd = torch.from_numpy(s).cuda()
        counts = split.candidate_counts(n_ctx, world, k)
        stride = max(max(counts), 1)
        cs = torch.zeros(world * stride, device="cuda", dtype=torch.float32)
        cidx = torch.zeros(world * stride, device="cuda", dtype=torch.int32)
        st = torch.zeros(1, device="cuda", dtype=torch.int32)
        for r in range(world):
            lo, hi = split.block_bounds(n_ctx, world, r)
            if counts[r]:
                tg.tg_topk_candidates(sd[lo:hi], k, base=lo, cand_score=cs[r * stride: r * stride + counts[r]],
                                      cand_idx=cidx[r * stride: r * stride + counts[r]], dev_status=st)
        kept = split.merge_gathered(cs, cidx, counts, stride, k, n_ctx, q)
        whole, _ = tg.tg_topk_select(sd, (n_ctx + q,), (q,), (k,))
        torch.cuda.synchronize()
        assert torch.equal(kept, whole), (world, ci)
        ref, _ = orc.topk_select(s, [n_ctx + q], [q], [k])
        assert kept.cpu().numpy().tolist() == [int(x) for x in ref], (world, ci)
        if kind == "nan":
            assert st.item() & tg.TG_DEV_NAN_SCORE
