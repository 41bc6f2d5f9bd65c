"""Multi-rank host logic on CPU (gloo, world size 2): the bench's job time is
the max over ranks of each rank's own CUDA-event time, and the KV-head
partition of one problem (bench.py --shard heads) covers every head exactly
once, with per-rank results that, concatenated, equal the whole problem's."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], "cpu")
    q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [11.0, 5.0]


def test_max_over_ranks_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], "cpu") == [1.5, 2.5]


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np
    import oracle as O
    from dynamic_block_sparse_qk_b200.shard import kv_head_range, q_head_range
    from synthetic import Workload, make_qkv
    w = Workload("shard", 1, 4, 2, 64, 1024, 64, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    kv = kv_head_range(w.h_kv, world, rank)
    qh = q_head_range(w.h_q, w.h_kv, world, rank)
    qs, ks, vs, _ = make_qkv(w, heads_kv=list(kv))        # this rank's slice only
    prm = O.CrispParams(block=w.block)
    res = O.crisp_prefill(O.bf16_to_f64(qs), O.bf16_to_f64(ks), O.bf16_to_f64(vs), prm)
    mine = {"rank": rank, "kv": list(kv), "q": list(qh),
            "pattern": [res["heads"][(0, i)]["pattern"] for i in range(len(qh))],
            "mask": [res["heads"][(0, i)]["mask"] for i in range(len(qh))],
            "o": [res["attn"][(0, i)][0] for i in range(len(qh))]}
    objs = [None] * world
    dist.all_gather_object(objs, mine)
    if rank == 0:
        q.put(objs)
    dist.barrier()
    dist.destroy_process_group()


def test_kv_head_shards_cover_every_head_and_match_the_whole_problem():
    import numpy as np
    import oracle as O
    from synthetic import Workload, make_qkv
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    parts = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = Workload("shard", 1, 4, 2, 64, 1024, 64, n_vertical=2, diffuse_frac=0.5, sink_logit=8.0)
    kv_all = sorted(h for part in parts for h in part["kv"])
    q_all = sorted(h for part in parts for h in part["q"])
    assert kv_all == list(range(w.h_kv)) and q_all == list(range(w.h_q))      # each head exactly once
    qf, kf, vf, _ = make_qkv(w)
    whole = O.crisp_prefill(O.bf16_to_f64(qf), O.bf16_to_f64(kf), O.bf16_to_f64(vf), O.CrispParams(block=w.block))
    for part in parts:
        for i, h in enumerate(part["q"]):
            assert part["pattern"][i] == whole["heads"][(0, h)]["pattern"]
            np.testing.assert_array_equal(part["mask"][i], whole["heads"][(0, h)]["mask"])
            np.testing.assert_array_equal(part["o"][i], whole["attn"][(0, h)][0])
    assert {part["pattern"][i] for part in parts for i in range(len(part["q"]))} == {O.VS, O.PE}


def test_kv_head_range_rejects_uneven_splits():
    import pytest
    from dynamic_block_sparse_qk_b200.shard import kv_head_range, q_head_range
    assert list(kv_head_range(8, 4, 3)) == [6, 7]
    assert list(q_head_range(32, 8, 4, 3)) == list(range(24, 32))
    with pytest.raises(ValueError):
        kv_head_range(8, 3, 0)
    with pytest.raises(ValueError):
        kv_head_range(8, 2, 2)
