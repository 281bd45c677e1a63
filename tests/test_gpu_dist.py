"""The multi-GPU schedules with libpa's kernels: two ranks that share cuda:0.

Every kernel of the schedules runs (sequence-chunk packing, placement of received pieces,
partition attention at each chunk milestone, the ring's per-block attention, the merge);
the exchange goes through host memory over gloo (HostStagedExchange), so the two ranks'
kernels never wait on one another.  Results are checked against the fp64 oracle's full
attention on the same seeded inputs.  (The NCCL exchange of the same schedules needs one
GPU per rank.)
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as O
from tests.helpers import TOL

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed, shape):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(*shape, generator=g).to(torch.bfloat16) for _ in range(3)]


def _rank(rank, ws, port, kind, cfg, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=120))
    try:
        import sequence_partition_attn_b200 as pa
        from sequence_partition_attn_b200.dist import DeviceOps, GroupRing, HostStagedExchange, TorusUlysses
        torch.cuda.set_device(0)
        ctx = pa.Context(0)
        ops, ex = DeviceOps(ctx), HostStagedExchange()
        if kind == "torus":
            N, H, D, P, G, C = cfg
            full = _inputs(3, (N, H, D))
            tu = TorusUlysses(ops, ex, None, N, H, D, P, G, C, device="cuda:0")
            for x in tu.qkv:
                x.fill_(float("nan"))
            n_loc = N // ws
            shard = [x[rank * n_loc:(rank + 1) * n_loc].contiguous().cuda() for x in full]
            o, lse = tu.run(*shard)
        else:
            N_blk, H, D, P_blk = cfg
            full = _inputs(4, (1, H, N_blk * ws, D))
            ring = GroupRing(ops, ex, None, N_blk, H, D, P_blk, device="cuda:0")
            blk = [x[:, :, rank * N_blk:(rank + 1) * N_blk].contiguous().cuda() for x in full]
            o, lse = ring.run(*blk)
        ctx.sync_status()
        out.put((rank, o.float().cpu().numpy(), lse.cpu().numpy()))
        ctx.close()
    finally:
        dist.destroy_process_group()


def _run(kind, ws, cfg):
    port = _free_port()
    q = mp.get_context("spawn").Queue()
    pc = mp.start_processes(_rank, args=(ws, port, kind, cfg, q), nprocs=ws, join=False, start_method="spawn")
    res = [q.get(timeout=600) for _ in range(ws)]
    while not pc.join(timeout=60):
        pass
    return sorted(res, key=lambda r: r[0])


def _full_attention(q, k, v, scale):
    N = q.shape[1]
    o, l, _ = O.partition_states(q[None], k[None], v[None], np.array([0, N]), 1,
                                 np.ones((1, 1), dtype=np.uint8), scale)
    return o[0, 0], l[0, 0]


def test_torus_ulysses_two_ranks_on_one_gpu():
    # N = 2 ranks x 4 chunks x 2 partitions of 128 tokens; 4 heads, 2 per rank
    cfg = (2048, 4, 128, 16, 1, 4)
    N, H, D = cfg[:3]
    res = _run("torus", 2, cfg)
    full = [np.transpose(x.double().numpy(), (1, 0, 2)) for x in _inputs(3, (N, H, D))]
    ro, rl = _full_attention(*full, 1.0 / np.sqrt(D))
    H_loc = H // 2
    for rank, o, lse in res:
        hs = slice(rank * H_loc, (rank + 1) * H_loc)
        assert np.abs(o[0] - ro[hs]).max() <= TOL["bf16"]["o"]
        assert np.abs(lse[0] - rl[hs]).max() <= TOL["bf16"]["lse"]


def test_group_ring_two_ranks_on_one_gpu():
    cfg = (640, 2, 128, 3)       # 640-token blocks in 3 partitions (the last one short)
    N_blk, H, D, _ = cfg
    res = _run("ring", 2, cfg)
    full = [x[0].double().numpy() for x in _inputs(4, (1, H, N_blk * 2, D))]
    ro, rl = _full_attention(*full, 1.0 / np.sqrt(D))
    for rank, o, lse in res:
        rows = slice(rank * N_blk, (rank + 1) * N_blk)
        assert np.abs(o[0] - ro[:, rows]).max() <= TOL["bf16"]["o"]
        assert np.abs(lse[0] - rl[:, rows]).max() <= TOL["bf16"]["lse"]
