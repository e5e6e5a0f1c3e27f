"""Multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

Each rank gets its own batch (same shapes, different seed: weak scaling), the
only cross-rank step is a MAX of the device time, and the job throughput is all
ranks' rows over the slowest rank's time.
"""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    import bench
    from long_context_sparse_04_b200 import inputs as I
    base = I.CONFIGS["decode_128k_paged"].replace(ctx_lo=200, ctx_hi=400, n_seqs=2, h_idx=2,
                                                  d_idx=16, n_heads=2, d_c=8, d_r=8, topk=16)
    cfg = bench.rank_config(base, rank)
    inp = I.generate(cfg, threads=1)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    dist.barrier()
    q.put((rank, cfg.seed, int(inp["row_klen"].sum()), t,
           bench.throughput(world, len(inp["row_seq"]), 3, t)))
    dist.destroy_process_group()


def test_two_rank_weak_scaling_host_logic():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, k0, t0, v0), (r1, s1, k1, t1, v1) = res
    assert s0 != s1                    # each rank its own batch
    assert k0 != k1                    # and so its own context lengths
    assert t0 == t1 == 15.0            # max over ranks
    assert v0 == v1 == 2 * 4 * 3 / 0.015
