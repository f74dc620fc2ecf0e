"""World-size-2 gloo runs (CPU) of the multi-rank plumbing bench.py uses:
per-rank seeds and inputs, the max-over-ranks time and the whole-job rate."""
import os
import socket

import torch
import torch.multiprocessing as mp

from gqa_softmax_attention_attn_b200 import multirank
from gqa_softmax_attention_attn_b200.inputs import prefill_inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    r, w, lr = multirank.env_rank()
    assert (r, w, lr) == (rank, world, rank)
    multirank.init("gloo", timeout_s=60)
    seed = multirank.rank_seed(1002, rank)
    t = prefill_inputs(1, 16, 16, 8, 2, 64, torch.bfloat16, 0.5, 1.0, seed=seed)
    # a fake per-rank device time: rank 1 is the slow one
    times = [10.0 + 5.0 * rank, 1.0 * rank]
    mx = multirank.max_over_ranks(times)
    multirank.barrier()
    out[rank] = (seed, float(t["q"].float().sum()), mx,
                 multirank.job_throughput(100.0, world, mx[0] * 1e-3))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    (s0, q0, mx0, v0), (s1, q1, mx1, v1) = out[0], out[1]
    assert s0 == 1002 and s1 != s0          # rank 0 runs the single-GPU batch, rank 1 its own
    assert q0 != q1                         # different inputs per rank
    assert mx0 == mx1 == [15.0, 1.0]        # every rank sees the slowest rank's times
    assert v0 == v1 == 100.0 * 2 / 15e-3    # whole-job units over the max time


def test_single_process_defaults():
    assert multirank.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert multirank.rank_seed(5, 0) == 5


def _dsink_worker(rank, world, port, out):
    # rank r holds batch element r of a B = 2 problem and its own backward
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import oracle

    multirank.init("gloo", timeout_s=60)
    t = prefill_inputs(2, 24, 24, 4, 2, 64, torch.float32, 1.0, 1.0, 1.0, seed=77, with_dout=True)
    sh = {k: (v[rank:rank + 1] if k in ("q", "k", "v", "dout") else v) for k, v in t.items()}
    _, _, _, ds = oracle.bwd(sh["q"], sh["k"], sh["v"], sh["sinks"], sh["dout"], 0, 0.125)
    local = torch.tensor(ds, dtype=torch.float64)
    total = multirank.allreduce_dsinks(local.clone())
    out[rank] = (local.tolist(), total.tolist())
    torch.distributed.destroy_process_group()


def test_dsinks_allreduce_over_batch_shards():
    import numpy as np

    import oracle

    world, port = 2, _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.start_processes(_dsink_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    t = prefill_inputs(2, 24, 24, 4, 2, 64, torch.float32, 1.0, 1.0, 1.0, seed=77, with_dout=True)
    _, _, _, full = oracle.bwd(t["q"], t["k"], t["v"], t["sinks"], t["dout"], 0, 0.125)
    (l0, s0), (l1, s1) = out[0], out[1]
    assert not np.allclose(l0, l1)                            # each rank saw only its shard
    assert s0 == s1                                           # every rank holds the same sum
    np.testing.assert_allclose(s0, full, rtol=1e-12, atol=1e-14)  # = dsinks of the whole batch

