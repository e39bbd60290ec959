"""Multi-process (gloo, world size 2, CPU) checks of the multi-GPU host logic: sequences are
spread over ranks without any exchange, the per-rank results equal the whole-batch result,
and the timing reduction takes the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from learned_token_pruning_02_b200 import replicas


def test_assign_sequences_covers_each_sequence_once():
    seqlens, q, k = [16384, 12000, 8192, 3000, 500, 70000], [64, 200, 32, 128, 0, 256], [256] * 6
    for world in (1, 2, 3, 4, 8):
        parts = replicas.assign_sequences(seqlens, q, k, world)
        flat = sorted(b for p in parts for b in p)
        assert flat == list(range(len(seqlens)))
        assert parts == replicas.assign_sequences(seqlens, q, k, world)  # deterministic
    # the longest sequence sits alone when there are enough ranks
    parts = replicas.assign_sequences(seqlens, q, k, 4)
    assert [5] in parts


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, seqlens, q, k, ret):
    import torch.distributed as dist

    from oracle import tg_oracle as orc

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = replicas.assign_sequences(seqlens, q, k, world)[rank]
        g = np.random.default_rng(7)
        scores = [g.standard_normal(n).astype(np.float32) for n in seqlens]
        res = {}
        for b in mine:  # each rank runs its own sequences; no exchange of data
            kept, _ = orc.topk_select(scores[b], [seqlens[b]], [q[b]], [k[b]])
            res[b] = kept.tolist()
        gathered = [None] * world
        dist.all_gather_object(gathered, res)
        t = replicas.max_over_ranks(1.5 + rank)
        if rank == 0:
            ret["kept"] = {b: v for d in gathered for b, v in d.items()}
            ret["tmax"] = t
            ret["scores"] = [s.tolist() for s in scores]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_match_whole_batch():
    from oracle import tg_oracle as orc

    seqlens, q, k = [300, 1000, 77, 512, 4], [10, 64, 0, 512, 2], [50, 100, 77, 3, 9]
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    ret = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, seqlens, q, k, ret)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    scores = np.concatenate([np.array(s, dtype=np.float32) for s in ret["scores"]])
    kept_all, cu = orc.topk_select(scores, seqlens, q, k)
    starts = np.concatenate([[0], np.cumsum(seqlens)])
    for b in range(len(seqlens)):
        ref = kept_all[cu[b]:cu[b + 1]] - starts[b]
        assert ret["kept"][b] == ref.tolist()
    assert ret["tmax"] == 2.5
