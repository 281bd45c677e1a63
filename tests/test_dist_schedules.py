"""The multi-GPU schedules (chunked Ulysses with attention on arrived chunks; ring inside a
group) on gloo ranks on the CPU.

The schedules' exchange steps run for real (torch.distributed over gloo, world sizes 2-4);
the kernel launches are replaced by host stand-ins built on the fp64 oracle, so these
tests check what the schedules decide -- which pieces go where, which (query group, KV
group) pairs each attention launch covers and when, which block each ring step holds --
and that the assembled result equals full attention.  The same schedules with libpa's
kernels on a GPU are in tests/test_gpu_dist.py.
"""
import collections
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _f64(t):
    return t.detach().to("cpu").double().numpy()


class HostOps:
    """Host stand-ins of DeviceOps (fp64 oracle), recording what each launch covers."""

    def __init__(self, scale):
        self.scale = scale
        self.pairs = collections.Counter()
        self.launches = []

    def pack(self, src, dst, stream=None):
        dst.copy_(torch.from_numpy(O.relayout_seq2head(src.numpy())))

    def place(self, piece, dst, tok0, stream=None):
        n = piece.shape[0]
        dst[:, tok0:tok0 + n, :] = torch.from_numpy(O.relayout_seq2head(piece.numpy()))

    def attend(self, q, k, v, part_off, G, fresh, o_part, lse_part, stream=None):
        P = len(part_off) - 1
        QG = -(-P // G)
        fr = np.ones((QG, QG), dtype=np.uint8) if fresh is None else np.asarray(fresh)
        for qg, kg in zip(*np.nonzero(fr)):
            self.pairs[(int(qg), int(kg))] += 1
        self.launches.append(fr.copy())
        o, l, sel = O.partition_states(_f64(q), _f64(k), _f64(v), part_off, G, fr, self.scale)
        for p in range(P):
            rows = np.nonzero(sel[p])[0]
            if len(rows):
                o_part[p, :, :, rows] = torch.from_numpy(o[p][:, :, rows]).to(o_part.dtype)
                lse_part[p, :, :, rows] = torch.from_numpy(l[p][:, :, rows]).to(lse_part.dtype)

    def merge(self, part_off, G, o_part, lse_part, o, lse, stream=None):
        ro, rl = O.merge_states(list(_f64(o_part)), list(_f64(lse_part)))
        o.copy_(torch.from_numpy(ro))
        lse.copy_(torch.from_numpy(rl))


def _full_attention(q, k, v, scale):
    """Oracle full attention per head: q, k, v [H, N, D] f64 -> (O [H, N, D], LSE [H, N])."""
    N = q.shape[1]
    o, l, _ = O.partition_states(q[None], k[None], v[None], np.array([0, N]), 1,
                                 np.ones((1, 1), dtype=np.uint8), scale)
    return o[0, 0], l[0, 0]


def _run_ranks(fn, ws, port, cfg, q):
    """Start ws spawned ranks, collect one result from each (before joining: a rank with a
    large result waits for it to be read), then join them."""
    pc = mp.start_processes(fn, args=(ws, port, cfg, q), nprocs=ws, join=False, start_method="spawn")
    res = [q.get(timeout=300) for _ in range(ws)]
    while not pc.join(timeout=60):
        pass
    return sorted(res, key=lambda r: r[0])


def _init(rank, ws, port):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    return dist


def _torus_rank(rank, ws, port, cfg, out):
    dist = _init(rank, ws, port)
    try:
        from sequence_partition_attn_b200.dist import NcclExchange, TorusUlysses
        N, H, D, P, G, C = cfg
        g = torch.Generator().manual_seed(5)
        full = [torch.randn(N, H, D, generator=g) for _ in range(3)]       # seq-major
        scale = 1.0 / np.sqrt(D)
        ops = HostOps(scale)
        # NcclExchange's calls on CPU tensors run over the gloo group
        tu = TorusUlysses(ops, NcclExchange(), None, N, H, D, P, G, C, dtype=torch.float32, device="cpu")
        for x in tu.qkv:
            x.fill_(float("nan"))          # a read of a piece before it arrives shows as NaN
        n_loc = N // ws
        shard = [x[rank * n_loc:(rank + 1) * n_loc].contiguous() for x in full]
        o, lse = tu.run(*shard)
        # gather every rank's heads
        og = [torch.empty_like(o) for _ in range(ws)]
        lg = [torch.empty_like(lse) for _ in range(ws)]
        dist.all_gather(og, o)
        dist.all_gather(lg, lse)
        out.put((rank, torch.cat(og, dim=1)[0].numpy(), torch.cat(lg, dim=1)[0].numpy(),
                 dict(ops.pairs), [m.tolist() for m in ops.launches], tu.milestones,
                 [x.numpy() for x in full]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,cfg", [
    (2, (128, 4, 16, 16, 1, 4)),     # 4 chunks, 2 partitions (= 2 groups) per piece
    (2, (96, 2, 8, 12, 2, 3)),       # 3 chunks (milestones 1, 2, 3), groups of 2
    (4, (128, 4, 8, 16, 2, 2)),      # 4 ranks, one head each
])
def test_torus_ulysses_schedule_on_gloo_ranks(ws, cfg):
    N, H, D, P, G, C = cfg
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    res = _run_ranks(_torus_rank, ws, port, cfg, q)
    full = res[0][6]
    hm = [np.transpose(x, (1, 0, 2)).astype(np.float64) for x in full]    # head-major [H, N, D]
    ro, rl = _full_attention(*hm, 1.0 / np.sqrt(D))
    QG = P // G
    for rank, o, lse, pairs, launches, milestones, _ in res:
        assert np.abs(o - ro).max() <= 1e-5 and np.abs(lse - rl).max() <= 1e-5
        # every (query group, KV group) pair computed exactly once, in the milestone launches
        assert len(pairs) == QG * QG and set(pairs.values()) == {1}
        assert len(launches) == len(milestones) and milestones[-1] == C


def _ring_rank(rank, ws, port, cfg, out):
    dist = _init(rank, ws, port)
    try:
        from sequence_partition_attn_b200.dist import GroupRing, HostStagedExchange
        N_blk, H, D, P_blk = cfg
        g = torch.Generator().manual_seed(9)
        N = N_blk * ws
        full = [torch.randn(1, H, N, D, generator=g) for _ in range(3)]   # head-major
        scale = 1.0 / np.sqrt(D)
        ops = HostOps(scale)
        ring = GroupRing(ops, HostStagedExchange(), None, N_blk, H, D, P_blk, dtype=torch.float32,
                         device="cpu")
        blk = [x[:, :, rank * N_blk:(rank + 1) * N_blk].contiguous() for x in full]
        o, lse = ring.run(*blk)
        out.put((rank, o.numpy().copy(), lse.numpy().copy(), ring.lse_part.numpy().copy(),
                 [x.numpy() for x in full]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws,cfg", [(2, (40, 2, 16, 3)), (3, (24, 1, 8, 2)), (4, (16, 2, 8, 1))])
def test_group_ring_on_gloo_ranks(ws, cfg):
    N_blk, H, D, P_blk = cfg
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    res = _run_ranks(_ring_rank, ws, port, cfg, q)
    full = [x[0].astype(np.float64) for x in res[0][4]]                  # [H, N, D]
    scale = 1.0 / np.sqrt(D)
    ro, rl = _full_attention(*full, scale)
    N = N_blk * ws
    S = -(-N_blk // P_blk)
    for rank, o, lse, lse_part, _ in res:
        rows = slice(rank * N_blk, (rank + 1) * N_blk)
        assert np.abs(o[0] - ro[:, rows]).max() <= 1e-5
        assert np.abs(lse[0] - rl[:, rows]).max() <= 1e-5
        # state of the block of rank s, partition p: keys [s*N_blk + p*S, ...) in token order
        for s in range(ws):
            for p in range(P_blk):
                k0, k1 = s * N_blk + min(p * S, N_blk), s * N_blk + min((p + 1) * S, N_blk)
                q = full[0][:, rows]
                sc = np.einsum("hnd,hmd->hnm", q, full[1][:, k0:k1]) * scale
                mx = sc.max(-1, keepdims=True)
                want = (mx[..., 0] + np.log(np.exp(sc - mx).sum(-1)))
                assert np.abs(lse_part[s * P_blk + p, 0] - want).max() <= 1e-5


def test_torus_chunk_masks_cover_every_pair_once():
    from sequence_partition_attn_b200.dist import chunk_milestones, torus_chunk_masks
    for W, C, gpp in [(2, 4, 1), (4, 2, 2), (8, 16, 1), (3, 5, 2)]:
        ms = chunk_milestones(C)
        masks = torus_chunk_masks(W, C, gpp, ms)
        np.testing.assert_array_equal(np.sum(masks, axis=0), 1)
        arrival = (np.arange(W * C * gpp) // gpp) % C
        for m, mask in zip(ms, masks):
            qg, kg = np.nonzero(mask)
            assert (arrival[qg] < m).all() and (arrival[kg] < m).all()


def test_torus_rejects_uneven_splits():
    from sequence_partition_attn_b200.dist import TorusUlysses

    class G:      # a stand-in group handle is never reached: the checks come first
        pass
    import torch.distributed as dist
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=30))
    try:
        with pytest.raises(ValueError):
            TorusUlysses(None, None, None, 100, 4, 8, 10, 1, 3, device="cpu")    # 100 tokens, 3 chunks
        with pytest.raises(ValueError):
            TorusUlysses(None, None, None, 96, 4, 8, 12, 5, 2, device="cpu")     # 6 partitions per piece, G=5
    finally:
        dist.destroy_process_group()
