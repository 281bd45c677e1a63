"""Schedules across the GPUs of one node, built on libpa's kernels and torch.distributed.

Two schedules of the pages' multi-GPU designs, each rank running libpa's kernels on its own
GPU and NCCL moving the data (over NVLink / NVSwitch):

* ``TorusUlysses`` -- sequence-parallel attention with the Ulysses all-to-all cut into
  sequence chunks, attention starting on the chunks that have arrived while later chunks
  are still in flight (SwiftFusion web summary, Methodology 2, "Torus Attention": chunking,
  pipelining, overlap).  Each rank starts with a sequence shard of Q, K, V for every head
  and ends with the attention states of every token for its share of the heads.
* ``GroupRing`` -- the attention state of a group computed by a ring over its g ranks: the
  KV blocks circulate, each rank computes the states of its own queries against the block
  it holds while the next block is in transfer, and the g blocks' states are merged into
  the group state (DiTango web summary, Methodology 2, "Group-wise state computation":
  g - 1 KV transfers overlapped with the attention, yielding a composed group state).

Every peer block is received into this GPU's own memory before a kernel reads it; no
kernel reads another GPU's memory.

The kernel launches go through an ``ops`` object (``DeviceOps``: libpa's calls on one
context).  The exchange goes through an ``exchange`` object: ``NcclExchange`` moves device
tensors with NCCL; ``HostStagedExchange`` moves them through host memory with whatever
process group it is given (gloo), which lets ranks that share one GPU exercise the whole
schedule.  Tests substitute host implementations of ``ops`` to check the schedules on CPU
ranks; the library itself has no CPU path.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import (Context, pa_merge_states, pa_partition_attn, pa_relayout_seq2head,
               pa_relayout_seq2head_at)


# ------------------------------------------------------------------ kernel launches
class DeviceOps:
    """The libpa calls the schedules launch, on one context."""

    def __init__(self, ctx: Context):
        self.ctx = ctx

    def pack(self, src, dst, stream=None):
        """dst[w, n, :] = src[n, w, :]: a sequence chunk [n, W, E] regrouped by destination
        rank (the relayout with ranks in place of heads)."""
        pa_relayout_seq2head(self.ctx, src, dst, stream=stream)

    def place(self, piece, dst, tok0, stream=None):
        """dst[h, tok0 + n, :] = piece[n, h, :] (a received piece into the head-major tensor)."""
        pa_relayout_seq2head_at(self.ctx, piece, dst, tok0, stream=stream)

    def attend(self, q, k, v, part_off, G, fresh, o_part, lse_part, stream=None):
        pa_partition_attn(self.ctx, q, k, v, part_off, G, fresh, o_part, lse_part, stream=stream)

    def merge(self, part_off, G, o_part, lse_part, o, lse, stream=None):
        pa_merge_states(self.ctx, part_off, G, None, o_part, lse_part, None, None, o, lse,
                        stream=stream)


# ------------------------------------------------------------------ data movement
class NcclExchange:
    """all-to-all and ring steps on device tensors through NCCL (the process group's
    backend must be nccl).  Calls are issued on the current stream's device; completion is
    awaited on the stream the caller names."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, out, inp, stream=None):
        with torch.cuda.stream(stream) if stream is not None else _nullcontext():
            return dist.all_to_all_single(out, inp, group=self.group, async_op=True)

    def ring(self, send, recv, nxt, prv, stream=None):
        ops = [dist.P2POp(dist.isend, t, nxt, group=self.group) for t in send] + \
              [dist.P2POp(dist.irecv, t, prv, group=self.group) for t in recv]
        with torch.cuda.stream(stream) if stream is not None else _nullcontext():
            return dist.batch_isend_irecv(ops)

    @staticmethod
    def wait(work, stream=None):
        """Make `stream` (default: the current one) wait for the transfer (no host block)."""
        works = work if isinstance(work, list) else [work]
        with torch.cuda.stream(stream) if stream is not None else _nullcontext():
            for w in works:
                w.wait()


class HostStagedExchange:
    """The same steps through host memory over any process group (gloo): device tensors
    are copied to the host, exchanged, and copied back.  Synchronous; meant for ranks that
    share one GPU, whose kernels never wait on one another (the host exchange orders
    them)."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, out, inp, stream=None):
        h_in = inp.detach().to("cpu")
        h_out = torch.empty_like(h_in)
        dist.all_to_all_single(h_out, h_in, group=self.group)
        out.copy_(h_out)
        return None

    def ring(self, send, recv, nxt, prv, stream=None):
        h_send = [t.detach().to("cpu") for t in send]
        h_recv = [torch.empty_like(t, device="cpu") for t in recv]
        ops = [dist.P2POp(dist.isend, t, nxt, group=self.group) for t in h_send] + \
              [dist.P2POp(dist.irecv, t, prv, group=self.group) for t in h_recv]
        for w in dist.batch_isend_irecv(ops):
            w.wait()
        for d, h in zip(recv, h_recv):
            d.copy_(h)
        return None

    @staticmethod
    def wait(work, stream=None):
        return None


class _nullcontext:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def _rank_info(group):
    return dist.get_rank(group), dist.get_world_size(group)


# ------------------------------------------------------------------ Torus / Ulysses
def torus_chunk_masks(W: int, C: int, groups_per_piece: int, milestones):
    """Masks (uint8[QG, QG], 1 = compute) of the attention launches of the chunked
    all-to-all.  Group g (token order) belongs to piece (rank s, chunk c) with
    g // groups_per_piece = s * C + c, so it has arrived once chunks [0, c] have.  The
    launch after chunks [0, m) computes every pair whose later-arriving group came with a
    chunk in [previous milestone, m); together the launches cover every pair once."""
    QG = W * C * groups_per_piece
    arrival = (np.arange(QG) // groups_per_piece) % C
    last = np.maximum(arrival[:, None], arrival[None, :])
    masks, prev = [], 0
    for m in milestones:
        masks.append(((last >= prev) & (last < m)).astype(np.uint8))
        prev = m
    return masks


def chunk_milestones(n_chunks: int):
    """Chunk counts after which attention launches: 1, 2, 4, ... and n_chunks."""
    out, m = [], 1
    while m < n_chunks:
        out.append(m)
        m *= 2
    out.append(n_chunks)
    return out


class TorusUlysses:
    """Chunked Ulysses attention over the ranks of `group` (SwiftFusion web summary,
    Methodology 2, "Torus Attention").

    Every rank holds tokens [r * N_loc, (r + 1) * N_loc) of Q, K, V for all H heads,
    sequence-major [N_loc, H, D] (B = 1), and obtains, for heads
    [r * H_loc, (r + 1) * H_loc), the per-partition states and the merged (O, LSE) of every
    token.  The all-to-all runs in ``n_chunks`` steps: step c sends sub-chunk c of every
    rank's shard (tokens r * N_loc + c * n_c ... + n_c) to the rank owning each head slice.
    A received piece is placed into the head-major tensors, and attention launches at
    the milestones 1, 2, 4, ... n_chunks over the (query group, KV group) pairs whose
    pieces have both arrived, while later chunks are in flight.

    Partitions split N evenly (S = N / P) with P a multiple of W * n_chunks, so that every
    piece holds whole partitions and groups of G.
    """

    def __init__(self, ops, exchange, group, N, H, D, P, G, n_chunks, dtype=torch.bfloat16,
                 device="cuda:0", milestones=None):
        self.ops, self.ex, self.group = ops, exchange, group
        self.rank, self.W = _rank_info(group)
        W = self.W
        if N % (W * n_chunks) or H % W or N % P or P % (W * n_chunks):
            raise ValueError(f"N={N}, H={H}, P={P} must split evenly over {W} ranks x {n_chunks} chunks")
        per_piece = P // (W * n_chunks)
        if per_piece % G:
            raise ValueError(f"a piece of {per_piece} partitions is not a whole number of groups of {G}")
        self.N, self.H, self.D, self.P, self.G, self.C = N, H, D, P, G, n_chunks
        self.N_loc, self.H_loc, self.n_c = N // W, H // W, N // (W * n_chunks)
        self.part_off = np.arange(P + 1, dtype=np.int32) * (N // P)
        self.QG = P // G
        self.milestones = chunk_milestones(n_chunks) if milestones is None else list(milestones)
        self.masks = torus_chunk_masks(W, n_chunks, per_piece // G, self.milestones)
        dev = torch.device(device)
        mk = lambda *s, dt=dtype: torch.empty(*s, dtype=dt, device=dev)     # noqa: E731
        self.qkv = [mk(1, self.H_loc, N, D) for _ in range(3)]               # head-major, my heads
        self.send = [[mk(W, self.n_c, self.H_loc * D) for _ in range(3)] for _ in range(2)]
        self.recv = [[mk(W, self.n_c, self.H_loc, D) for _ in range(3)] for _ in range(2)]
        self.o_part = mk(P, 1, self.H_loc, N, D)
        self.lse_part = mk(P, 1, self.H_loc, N, dt=torch.float32)
        self.o = mk(1, self.H_loc, N, D)
        self.lse = mk(1, self.H_loc, N, dt=torch.float32)
        self.cuda = dev.type == "cuda"
        if self.cuda:
            self.s_comm = torch.cuda.Stream(device=dev)
            self.s_attn = torch.cuda.Stream(device=dev)

    def run(self, q_loc, k_loc, v_loc):
        """q_loc, k_loc, v_loc: [N_loc, H, D] sequence shards of this rank.  Returns
        (o, lse): [1, H_loc, N, D], [1, H_loc, N] for this rank's heads; the partition
        states stay in self.o_part / self.lse_part."""
        W, C, n_c, E = self.W, self.C, self.n_c, self.H_loc * self.D
        cur = torch.cuda.current_stream() if self.cuda else None
        comm, attn = (self.s_comm, self.s_attn) if self.cuda else (None, None)
        if self.cuda:
            comm.wait_stream(cur)
            attn.wait_stream(cur)
        arrived = []
        m_i = 0
        for c in range(C):
            b = c % 2
            if self.cuda and c >= 2:
                comm.wait_event(arrived[c - 2])           # buffers of chunk c-2 placed
            with _stream(comm):
                for x, src in enumerate((q_loc, k_loc, v_loc)):
                    chunk = src[c * n_c:(c + 1) * n_c].reshape(n_c, W, E)
                    self.ops.pack(chunk, self.send[b][x], stream=comm)
                works = [self.ex.all_to_all(self.recv[b][x].view(W, -1), self.send[b][x].view(W, -1),
                                            stream=comm) for x in range(3)]
                for w in works:
                    if w is not None:
                        self.ex.wait(w, stream=comm)
                for x in range(3):
                    for s in range(W):
                        tok0 = s * self.N_loc + c * n_c
                        self.ops.place(self.recv[b][x][s], self.qkv[x][0], tok0, stream=comm)
                if self.cuda:
                    ev = torch.cuda.Event()
                    ev.record(comm)
                    arrived.append(ev)
                else:
                    arrived.append(None)
            # attention over the pairs whose pieces have both arrived, at each milestone
            while m_i < len(self.milestones) and self.milestones[m_i] == c + 1:
                if self.cuda:
                    attn.wait_event(arrived[c])
                with _stream(attn):
                    self.ops.attend(*self.qkv, self.part_off, self.G, self.masks[m_i],
                                    self.o_part, self.lse_part, stream=attn)
                m_i += 1
        with _stream(attn):
            self.ops.merge(self.part_off, self.P, self.o_part, self.lse_part, self.o, self.lse,
                           stream=attn)
        if self.cuda:
            cur.wait_stream(attn)
            cur.wait_stream(comm)
        return self.o, self.lse


# ------------------------------------------------------------------ ring inside a group
class GroupRing:
    """Ring-composed attention inside the group of ranks `group` (DiTango web summary,
    Methodology 2, "Group-wise state computation").

    Rank r holds the query block and the KV block of tokens [r * N_blk, (r + 1) * N_blk)
    (head-major [1, H, N_blk, D]), each KV block split into P_blk partitions.  At step s it
    computes the states of its queries against the KV block of rank (r - s) mod g while
    that block moves on to rank r + 1 and the next one arrives from rank r - 1 (g - 1
    transfers, each overlapped with a step's attention); the g * P_blk states, ordered by
    token, are then merged into the group state (O, LSE) of its queries.
    """

    def __init__(self, ops, exchange, group, N_blk, H, D, P_blk, dtype=torch.bfloat16,
                 device="cuda:0"):
        self.ops, self.ex, self.group = ops, exchange, group
        self.rank, self.g = _rank_info(group)
        if P_blk < 1 or N_blk < 1:
            raise ValueError("empty block")
        self.N_blk, self.H, self.D, self.P_blk = N_blk, H, D, P_blk
        S = -(-N_blk // P_blk)
        self.blk_off = np.array([min(p * S, N_blk) for p in range(P_blk + 1)], dtype=np.int32)
        # the merge treats the g * P_blk states as partitions of one query group
        P = self.g * P_blk
        self.merge_off = np.array([min(i * N_blk // P, N_blk) for i in range(P + 1)], dtype=np.int32)
        self.merge_off[-1] = N_blk
        dev = torch.device(device)
        mk = lambda *s, dt=dtype: torch.empty(*s, dtype=dt, device=dev)     # noqa: E731
        self.kv = [[mk(1, H, N_blk, D), mk(1, H, N_blk, D)] for _ in range(2)]
        self.o_part = mk(P, 1, H, N_blk, D)
        self.lse_part = mk(P, 1, H, N_blk, dt=torch.float32)
        self.o = mk(1, H, N_blk, D)
        self.lse = mk(1, H, N_blk, dt=torch.float32)
        self.cuda = dev.type == "cuda"
        if self.cuda:
            self.s_comm = torch.cuda.Stream(device=dev)

    def run(self, q, k, v):
        """q, k, v: this rank's blocks [1, H, N_blk, D].  Returns (o, lse) of its queries
        over the whole group's keys; per-block states stay in self.o_part / self.lse_part
        (block of rank s at partitions [s * P_blk, (s + 1) * P_blk))."""
        g, r, Pb = self.g, self.rank, self.P_blk
        nxt, prv = (r + 1) % g, (r - 1) % g
        nxt_g = dist.get_global_rank(self.group, nxt) if self.group is not None else nxt
        prv_g = dist.get_global_rank(self.group, prv) if self.group is not None else prv
        cur = torch.cuda.current_stream() if self.cuda else None
        comm = self.s_comm if self.cuda else None
        blk = [k, v]
        done = None                            # event: attention on the previous block issued
        for s in range(g):
            src = (r - s) % g
            work = None
            if s < g - 1:
                dst_buf = self.kv[s % 2]
                if self.cuda:
                    comm.wait_stream(cur)      # the block to send is complete; recv buffer free
                work = self.ex.ring(blk, dst_buf, nxt_g, prv_g, stream=comm)
            self.ops.attend(q, blk[0], blk[1], self.blk_off, Pb, None,
                            self.o_part[src * Pb:(src + 1) * Pb], self.lse_part[src * Pb:(src + 1) * Pb],
                            stream=cur)
            if s < g - 1:
                if work is not None:
                    self.ex.wait(work, stream=cur)   # the next block has arrived
                blk = self.kv[s % 2]
        self.ops.merge(self.merge_off, g * Pb, self.o_part, self.lse_part, self.o, self.lse, stream=cur)
        return self.o, self.lse


def _stream(s):
    return torch.cuda.stream(s) if s is not None else _nullcontext()
