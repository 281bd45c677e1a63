"""Device-resident attention step with selective state reuse, built on the libpa calls.

A step takes Q, K, V of one denoising step already in HBM, computes the attention states of
the fresh (query group, KV group) pairs, and merges them with the cached states of the
other pairs into (O, LSE) plus the partition importance w (DiTango web summary,
Methodology 1-2).  ``Trajectory`` adds the host side of the selection: all pairs fresh at
anchor steps (importance stored, cache refreshed); otherwise either pairs whose stored
importance falls below a threshold reuse the anchor's states, or (online prediction) the
own groups are computed first, their drift from the anchor measured, and pairs whose
predicted error (importance times drift) stays below a bound reuse the anchor's states.

Only orchestration lives here; every arithmetic step runs in libpa's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (Context, pa_merge_states, pa_partition_attn, pa_relayout_seq2head,
               pa_state_drift, predict_fresh, select_fresh)


def attn_flops(part_off, G: int, fresh, B: int, H: int, D: int) -> float:
    """Algorithmic flops of the fresh pairs: 4*D per (query row, valid key) of each pair
    (QK^T and PV, multiply-add = 2).  Padding, skipped pairs and exponentials excluded."""
    off = np.asarray(part_off, dtype=np.int64)
    P = len(off) - 1
    QG = -(-P // G)
    gb = np.array([off[min(g * G, P)] for g in range(QG + 1)])
    rows = np.diff(gb)
    total = 0
    for qg in range(QG):
        for kg in range(QG):
            if fresh is None or fresh[qg][kg]:
                total += int(rows[qg]) * int(rows[kg])
    return 4.0 * D * B * H * total


def merge_bytes(B, H, N, D, P, elem_bytes) -> float:
    """Algorithmic HBM bytes of the merge: per row P states of (D*elem + 4) read and one
    state written; the importance adds nothing (fused)."""
    row = D * elem_bytes + 4
    return float(B) * H * N * (P * row + row)


class AttentionStep:
    """Buffers and launches of one attention step at a fixed shape, partitioning and mask."""

    def __init__(self, ctx: Context, B, H, N, D, part_off, G, fresh, dtype=torch.bfloat16,
                 device="cuda:0"):
        self.ctx = ctx
        self.B, self.H, self.N, self.D, self.G = B, H, N, D, G
        self.part_off = np.asarray(part_off, dtype=np.int32)
        self.P = len(self.part_off) - 1
        self.QG = -(-self.P // G)
        self.fresh = None if fresh is None else np.asarray(fresh, dtype=np.uint8)
        dev = torch.device(device)
        P = self.P
        mk = lambda *s, dt=dtype: torch.empty(*s, dtype=dt, device=dev)   # noqa: E731
        self.q, self.k, self.v = mk(B, H, N, D), mk(B, H, N, D), mk(B, H, N, D)
        self.o_fresh, self.lse_fresh = mk(P, B, H, N, D), mk(P, B, H, N, dt=torch.float32)
        reuse = self.fresh is not None and not self.fresh.all()
        self.o_cached = mk(P, B, H, N, D) if reuse else None
        self.lse_cached = mk(P, B, H, N, dt=torch.float32) if reuse else None
        self.o, self.lse = mk(B, H, N, D), mk(B, H, N, dt=torch.float32)
        self.w = mk(self.QG, P, dt=torch.float32)
        self.flops = attn_flops(self.part_off, G, self.fresh, B, H, D)
        self.merge_bytes = merge_bytes(B, H, N, D, P, torch.empty(0, dtype=dtype).element_size())

    def fill_cache(self, k_prev, v_prev, stream=None):
        """States of every pair on (Q, K_prev, V_prev): the cache of an earlier step."""
        if self.o_cached is None:
            return
        pa_partition_attn(self.ctx, self.q, k_prev, v_prev, self.part_off, self.G, None,
                          self.o_cached, self.lse_cached, stream=stream)

    def attention(self, stream=None, q=None, k=None, v=None):
        """Fresh states from q, k, v (default: the step's own input buffers)."""
        pa_partition_attn(self.ctx, self.q if q is None else q, self.k if k is None else k,
                          self.v if v is None else v, self.part_off, self.G, self.fresh,
                          self.o_fresh, self.lse_fresh, stream=stream)

    def merge(self, stream=None, o=None, lse=None, w=None):
        """Merge into o, lse, w (default: the step's own output buffers)."""
        pa_merge_states(self.ctx, self.part_off, self.G, self.fresh, self.o_fresh, self.lse_fresh,
                        self.o_cached, self.lse_cached, self.o if o is None else o,
                        self.lse if lse is None else lse, self.w if w is None else w, stream=stream)

    def run(self, stream=None):
        self.attention(stream)
        self.merge(stream)


class StreamedSteps:
    """Steps fed from host memory with the copies of neighbouring steps overlapped with
    compute.  Inputs (Q, K, V) and outputs (O, LSE, w) are double-buffered on the device;
    host-to-device copies run on one stream, the step on a second, device-to-host copies
    on a third, so step i's inputs arrive while step i-1 computes and step i-1's outputs
    leave while step i computes.  Every step still moves its own inputs in and its own
    outputs out; the intermediate states stay in the step's buffers.
    """

    def __init__(self, step: AttentionStep):
        self.step = step
        two = lambda t: [torch.empty_like(t) for _ in range(2)]          # noqa: E731
        self.q, self.k, self.v = two(step.q), two(step.k), two(step.v)
        self.o, self.lse, self.w = two(step.o), two(step.lse), two(step.w)
        dev = step.q.device
        self.s_h2d = torch.cuda.Stream(device=dev)
        self.s_cmp = torch.cuda.Stream(device=dev)
        self.s_d2h = torch.cuda.Stream(device=dev)

    def run(self, host_inputs, host_outputs, after=None):
        """host_inputs[i] = (q, k, v) and host_outputs[i] = (o, lse, w): pinned host tensors
        of step i (an output triple may be reused across steps).  The copies of step 0 wait
        for stream `after` (default: the current stream).  Returns the event recorded when
        the last step's outputs have reached the host."""
        after = torch.cuda.current_stream() if after is None else after
        start = torch.cuda.Event()
        start.record(after)
        n = len(host_inputs)
        ev_in, ev_cmp, ev_out = [None] * n, [None] * n, [None] * n
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(self.s_h2d):
                self.s_h2d.wait_event(start)
                if i >= 2:
                    self.s_h2d.wait_event(ev_cmp[i - 2])     # step i-2 done with buffer b
                for d, h in zip((self.q[b], self.k[b], self.v[b]), host_inputs[i]):
                    d.copy_(h, non_blocking=True)
                ev_in[i] = torch.cuda.Event()
                ev_in[i].record(self.s_h2d)
            with torch.cuda.stream(self.s_cmp):
                self.s_cmp.wait_event(ev_in[i])
                if i >= 2:
                    self.s_cmp.wait_event(ev_out[i - 2])     # outputs of step i-2 have left
                self.step.attention(self.s_cmp, self.q[b], self.k[b], self.v[b])
                self.step.merge(self.s_cmp, self.o[b], self.lse[b], self.w[b])
                ev_cmp[i] = torch.cuda.Event()
                ev_cmp[i].record(self.s_cmp)
            with torch.cuda.stream(self.s_d2h):
                self.s_d2h.wait_event(ev_cmp[i])
                for h, d in zip(host_outputs[i], (self.o[b], self.lse[b], self.w[b])):
                    h.copy_(d, non_blocking=True)
                ev_out[i] = torch.cuda.Event()
                ev_out[i].record(self.s_d2h)
        return ev_out[-1]


class Trajectory:
    """Denoising trajectory with anchor steps and importance-driven reuse (host selection).

    At an anchor step every pair is fresh, the states become the cache and the importance
    w is stored (copied to the host: QG*P floats).  Between anchors the mask comes from
    one of two policies (DiTango web summary, Methodology 1):

    * ``"threshold"``: ``select_fresh(w_stored, G, threshold)`` -- recompute where the
      stored importance reaches the threshold.  No device-to-host transfer.
    * ``"predict"`` (online prediction): the own (query group, KV group) pairs -- always
      recomputed -- run first; ``pa_state_drift`` measures their states' change from the
      anchor's cached states; ``predict_fresh(w_stored, d2, r2, G, threshold)`` recomputes
      the pairs whose importance times that drift reaches the threshold (an error bound
      here).  The other selected pairs then run in a second attention launch.  Costs one
      2*QG*P-float device-to-host copy per step.

    Fresh pairs are recomputed from the current K, V and merged with the anchor's cached
    states.
    """

    def __init__(self, ctx, B, H, N, D, part_off, G, anchors, threshold, dtype=torch.bfloat16,
                 device="cuda:0", policy="threshold"):
        if policy not in ("threshold", "predict"):
            raise ValueError(f"unknown policy {policy!r}")
        self.ctx = ctx
        self.anchors = set(anchors)
        self.threshold = threshold
        self.policy = policy
        self.G = G
        self.part_off = np.asarray(part_off, dtype=np.int32)
        P = len(self.part_off) - 1
        self.P, self.QG = P, -(-P // G)
        dev = torch.device(device)
        self.cache_o = torch.empty(P, B, H, N, D, dtype=dtype, device=dev)
        self.cache_lse = torch.empty(P, B, H, N, dtype=torch.float32, device=dev)
        self.o_fresh = torch.empty_like(self.cache_o)
        self.lse_fresh = torch.empty_like(self.cache_lse)
        self.o = torch.empty(B, H, N, D, dtype=dtype, device=dev)
        self.lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
        self.w = torch.empty(self.QG, P, dtype=torch.float32, device=dev)
        self.d2 = torch.empty(self.QG, P, dtype=torch.float32, device=dev)
        self.r2 = torch.empty_like(self.d2)
        self.w_stored = None
        self.drift = None                   # (d2, r2) host copies of the last prediction

    def _mask(self, q, k, v, stream):
        if self.policy == "threshold":
            mask = select_fresh(self.w_stored, self.G, self.threshold)
            pa_partition_attn(self.ctx, q, k, v, self.part_off, self.G, mask, self.o_fresh,
                              self.lse_fresh, stream=stream)
            return mask
        own = np.eye(self.QG, dtype=np.uint8)
        pa_partition_attn(self.ctx, q, k, v, self.part_off, self.G, own, self.o_fresh,
                          self.lse_fresh, stream=stream)
        pa_state_drift(self.ctx, self.part_off, self.G, own, self.o_fresh, self.cache_o,
                       self.d2, self.r2, stream=stream)
        self.ctx.sync_status(stream)
        d2 = self.d2.cpu().numpy().astype(np.float64)
        r2 = self.r2.cpu().numpy().astype(np.float64)
        self.drift = (d2, r2)
        mask = predict_fresh(self.w_stored, d2, r2, self.G, self.threshold)
        rest = mask & ~own.astype(bool)
        if rest.any():
            pa_partition_attn(self.ctx, q, k, v, self.part_off, self.G, rest, self.o_fresh,
                              self.lse_fresh, stream=stream)
        return mask

    def step(self, s: int, q, k, v, stream=None) -> np.ndarray:
        """Run step s on device tensors q, k, v; returns the mask it used (uint8[QG, KG])."""
        if s in self.anchors or self.w_stored is None:
            mask = np.ones((self.QG, self.QG), dtype=np.uint8)
            pa_partition_attn(self.ctx, q, k, v, self.part_off, self.G, None, self.cache_o,
                              self.cache_lse, stream=stream)
            pa_merge_states(self.ctx, self.part_off, self.G, None, self.cache_o, self.cache_lse,
                            None, None, self.o, self.lse, self.w, stream=stream)
            # the merge runs on `stream`, which need not be torch's current stream: wait for
            # it (and check its bounded waits) before the host reads w
            self.ctx.sync_status(stream)
            self.w_stored = self.w.cpu().numpy().astype(np.float64)
            return mask
        mask = self._mask(q, k, v, stream)
        pa_merge_states(self.ctx, self.part_off, self.G, mask, self.o_fresh, self.lse_fresh,
                        self.cache_o, self.cache_lse, self.o, self.lse, self.w, stream=stream)
        return mask


def relayout_overlapped(ctx, src_qkv, dst_qkv, n_chunks, part_off, G, o_part, lse_part,
                        s_copy, s_attn, milestones=None):
    """Chunked seq-major -> head-major relayout of Q, K, V on one stream, overlapped with
    partition attention over the chunks already moved on another (SwiftFusion web summary,
    Methodology 2, Torus Attention).  All pairs fresh.

    Every chunk is relayed out on ``s_copy`` (3 launches) and recorded.  Attention runs in
    a few launches at the chunk counts in ``milestones`` (default 1, 2, 4, ... n_chunks):
    after chunks [0, m) have moved, it computes every (query chunk, KV chunk) pair whose
    later chunk lies in [previous milestone, m).  Geometric milestones keep the first
    attention launch early and the number of partially filled launches small.  Chunk
    boundaries must be group boundaries.  Returns the relayout events.
    """
    check_chunk_bounds(part_off, G, n_chunks)
    src_q, src_k, src_v = src_qkv
    q, k, v = dst_qkv
    P = len(part_off) - 1
    per = P // n_chunks
    QG = -(-P // G)
    gpc = per // G                          # groups per chunk
    if milestones is None:
        milestones = chunk_milestones(n_chunks)
    masks = milestone_masks(QG, gpc, milestones)
    events = []
    for c in range(n_chunks):
        with torch.cuda.stream(s_copy):
            for s, d in ((src_q, q), (src_k, k), (src_v, v)):
                pa_relayout_seq2head(ctx, s, d.view(d.shape[-3], d.shape[-2], d.shape[-1]),
                                     n_chunks=n_chunks, chunk=c, stream=s_copy)
            ev = torch.cuda.Event()
            ev.record(s_copy)
            events.append(ev)
    for m, mask in zip(milestones, masks):
        s_attn.wait_event(events[m - 1])
        pa_partition_attn(ctx, q, k, v, part_off, G, mask, o_part, lse_part, stream=s_attn)
    return events


def check_chunk_bounds(part_off, G: int, n_chunks: int) -> None:
    """Raise ValueError unless every relayout chunk ends on a group boundary.

    pa_relayout_seq2head cuts the sequence at multiples of ceil(N / n_chunks); attention
    after chunk c covers the partitions [0, c * P / n_chunks), i.e. the tokens
    [0, part_off[c * P / n_chunks]).  The two must coincide, or attention reads K/V rows
    that the other stream has not moved yet."""
    off = np.asarray(part_off, dtype=np.int64)
    P = len(off) - 1
    N = int(off[-1])
    if n_chunks < 1 or P % n_chunks:
        raise ValueError(f"P={P} partitions do not split into {n_chunks} chunks")
    per = P // n_chunks
    if per % G:
        raise ValueError(f"a chunk of {per} partitions is not a whole number of groups of {G}")
    step = -(-N // n_chunks)
    for c in range(n_chunks + 1):
        if int(off[c * per]) != min(c * step, N):
            raise ValueError(f"chunk {c} boundary: relayout at token {min(c * step, N)}, "
                             f"partitions at token {int(off[c * per])}")


def chunk_milestones(n_chunks):
    """Chunk counts after which attention launches: 1, 2, 4, ... and n_chunks."""
    milestones, m = [], 1
    while m < n_chunks:
        milestones.append(m)
        m *= 2
    milestones.append(n_chunks)
    return milestones


def milestone_masks(QG, gpc, milestones):
    """Reuse masks (uint8[QG, QG], 1 = compute) of the attention launches at `milestones`:
    after chunks [0, m) have moved, every (query group, KV group) pair whose later chunk
    lies in [previous milestone, m).  Together they select every pair exactly once."""
    masks, prev = [], 0
    for m in milestones:
        mask = np.zeros((QG, QG), dtype=np.uint8)
        lo, hi = prev * gpc, m * gpc
        mask[lo:hi, :hi] = 1                # new query chunks x every moved KV chunk
        mask[:lo, lo:hi] = 1                # earlier query chunks x new KV chunks
        masks.append(mask)
        prev = m
    return masks
