"""The N > 1 path of the benchmark on CPU with world-size-2 gloo: independent
replicas (distinct seeded workloads per rank), max-over-ranks timing and the
whole-job weak-scaling value.  No collective touches the data path."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    from paged_kv_cache_409_b200 import workloads
    w_ws, w_rank, _ = bench.dist_setup(ws, backend="gloo")
    assert (w_ws, w_rank) == (ws, rank)
    local_ms = 1.0 + 0.5 * rank                  # rank 1 is the slower one
    slowest = bench.max_over_ranks(local_ms, ws, device="cpu")
    bench.barrier(ws)
    w = workloads.llama7b_decode_f16(num_seqs=3, seed=1002 + rank)
    out.put((rank, slowest, bench.weak_scaling_value(ws, 64, slowest), w.context_lens.tolist()))
    dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, s0, v0, lens0), (_, s1, v1, lens1) = res
    assert s0 == s1 == 1.5                       # both ranks see the slowest rank's time
    assert np.isclose(v0, 2 * 64 / 1.5e-3) and v0 == v1
    assert lens0 != lens1                        # each rank runs its own replica
