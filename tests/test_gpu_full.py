"""Full-size GPU parity: the 720p step in the launch configuration bench.py times, the
10-step denoising trajectory with anchor steps, and the Ulysses-layout workload with the
chunked relayout overlapped with attention.  Sampled outputs are compared with the fp64
oracle row by row; w at full size is the oracle's fp64 importance reduction over every row
of the states the merge took, checked as well through properties that hold at any size and
against the stand-alone importance call."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests.helpers import TOL, maxerr

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pa():
    from sequence_partition_attn_b200 import build
    build.build()
    import sequence_partition_attn_b200 as m
    return m


def _rows_720p(wl):
    # 512 random rows, the first two 128-row query tiles of the first query partition, the
    # last 256 rows (the ragged last partition) and a query-group boundary, on every head
    off = W.part_offsets(wl.N, wl.P)
    rng = np.random.default_rng(11)
    r = rng.choice(wl.N, size=512, replace=False)
    first = np.arange(0, 256)
    tail = np.arange(off[-1] - 256, off[-1])
    bound = np.arange(off[4] - 8, off[4] + 8)
    return np.unique(np.concatenate([r, first, tail, bound]))


def test_720p_step_full_size_sampled_rows(pa):
    from sequence_partition_attn_b200.step import AttentionStep
    wl = W.workload(2)
    fresh = W.reuse_mask(wl)
    off = W.part_offsets(wl.N, wl.P)
    host = W.make_qkv(wl)
    kc, vc = W.make_cached_kv(wl, host["k"], host["v"])
    ctx = pa.Context(0)
    step = AttentionStep(ctx, wl.B, wl.H, wl.N, wl.D, off, wl.G, fresh, device=DEV)
    step.q.copy_(host["q"])
    step.k.copy_(host["k"])
    step.v.copy_(host["v"])
    step.fill_cache(kc.to(DEV), vc.to(DEV))
    step.run()
    ctx.sync_status()
    rows = _rows_720p(wl)
    ri = torch.as_tensor(rows, device=DEV)
    g = dict(o=step.o.index_select(2, ri).float().cpu().numpy(),
             lse=step.lse.index_select(2, ri).cpu().numpy(),
             of=step.o_fresh.index_select(3, ri).float().cpu().numpy(),
             lf=step.lse_fresh.index_select(3, ri).cpu().numpy(),
             oc=step.o_cached.index_select(3, ri).float().cpu().numpy(),
             lc=step.lse_cached.index_select(3, ri).cpu().numpy())
    w = step.w.cpu().numpy().astype(np.float64)
    # w: properties at full size, and the stand-alone importance on the merged states
    gb = O.group_bounds(off, wl.G)
    qg_of_p = np.repeat(np.arange(wl.QG), wl.G)[:wl.P]
    chosen = torch.empty_like(step.lse_fresh)
    for qg in range(wl.QG):
        r0, r1 = int(gb[qg]), int(gb[qg + 1])
        for p in range(wl.P):
            src = step.lse_fresh if fresh[qg, qg_of_p[p]] else step.lse_cached
            chosen[p, :, :, r0:r1] = src[p, :, :, r0:r1]
    w2 = torch.empty_like(step.w)
    pa.pa_importance(ctx, off, wl.G, chosen, step.lse, w2)
    ctx.sync_status()
    assert np.all(w >= 0)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-3)
    assert maxerr(w, w2.cpu().numpy()) <= 1e-5
    # the full-size importance reduction (every row of every query group, all heads) done
    # by the oracle in fp64 on the states the merge took; those states are checked against
    # the oracle's own, computed from Q, K, V, on the sampled rows below
    chosen_h = chosen.cpu().numpy().astype(np.float64)
    lse_h = step.lse.cpu().numpy().astype(np.float64)
    del chosen
    rw = O.importance(chosen_h, lse_h, off, wl.G)
    del chosen_h, lse_h
    assert maxerr(w, rw) <= TOL["bf16"]["w"], maxerr(w, rw)
    del step
    torch.cuda.empty_cache()

    ones = np.ones_like(fresh)
    tol = TOL["bf16"]
    sel = np.stack([fresh[np.searchsorted(gb, rows, side="right") - 1, p // wl.G] != 0
                    for p in range(wl.P)])                       # [P, R]
    worst = dict(o=0.0, lse=0.0, of=0.0, lf=0.0, oc=0.0, lc=0.0)
    for h in range(wl.H):
        qf, kf, vf = (W.to_f64(host[n][:, h:h + 1]) for n in ("q", "k", "v"))
        kcf, vcf = W.to_f64(kc[:, h:h + 1]), W.to_f64(vc[:, h:h + 1])
        rof, rlf, _ = O.partition_states(qf, kf, vf, off, wl.G, fresh, wl.scale, rows=rows)
        roc, rlc, _ = O.partition_states(qf, kcf, vcf, off, wl.G, ones, wl.scale, rows=rows)
        ro, rl, _ = O.merge_with_reuse(rof, rlf, roc, rlc, off, wl.G, fresh, rows=rows)
        m5 = np.broadcast_to(sel[:, :, None], (wl.P, len(rows), wl.D))
        worst["of"] = max(worst["of"], maxerr(g["of"][:, 0, h], rof[:, 0, 0], m5))
        worst["lf"] = max(worst["lf"], maxerr(g["lf"][:, 0, h], rlf[:, 0, 0], sel))
        worst["oc"] = max(worst["oc"], maxerr(g["oc"][:, 0, h], roc[:, 0, 0]))
        worst["lc"] = max(worst["lc"], maxerr(g["lc"][:, 0, h], rlc[:, 0, 0]))
        worst["o"] = max(worst["o"], maxerr(g["o"][0, h], ro[0, 0]))
        worst["lse"] = max(worst["lse"], maxerr(g["lse"][0, h], rl[0, 0]))
    print("720p full size, sampled rows:", worst)
    for k in ("o", "of", "oc"):
        assert worst[k] <= tol["o"], worst
    for k in ("lse", "lf", "lc"):
        assert worst[k] <= tol["lse"], worst
    ctx.close()


def _run_trajectory(pa, wl, quality_heads=0, policy="threshold", margin=0.15, side_stream=False):
    from sequence_partition_attn_b200.step import Trajectory
    off = W.part_offsets(wl.N, wl.P)
    host = W.make_qkv(wl)
    q, k, v = host["q"], host["k"], host["v"]
    ctx = pa.Context(0)
    traj = Trajectory(ctx, wl.B, wl.H, wl.N, wl.D, off, wl.G, wl.anchors, wl.threshold, device=DEV,
                      policy=policy)
    own = np.eye(wl.QG, dtype=np.uint8)
    ref_w = None
    qd = q.to(DEV)
    qf = W.to_f64(q)
    ones = np.ones((wl.QG, wl.KG), dtype=np.uint8)
    ref_cache = None
    tol = TOL["bf16"]
    report = []
    for s in range(wl.steps):
        if s > 0:
            k, v = W.drift_kv(wl, k, v, s)
        kd, vd = k.to(DEV), v.to(DEV)
        if side_stream:
            # the step runs on a stream that is not torch's current one
            side = torch.cuda.Stream(device=DEV)
            side.wait_stream(torch.cuda.current_stream())
            mask = traj.step(s, qd, kd, vd, stream=side)
            ctx.sync_status(side)
        else:
            mask = traj.step(s, qd, kd, vd)                       # mask from the GPU's stored w
        ctx.sync_status()
        o = traj.o.float().cpu().numpy()
        lse = traj.lse.cpu().numpy()
        kf, vf = W.to_f64(k), W.to_f64(v)
        of, lf, _ = O.partition_states(qf, kf, vf, off, wl.G, mask, wl.scale)
        flips = None
        if s in wl.anchors:
            assert mask.all()
            ref_cache = (of, lf)
            ro, rl = O.merge_states(list(of), list(lf))
            rw = O.importance(lf, rl, off, wl.G)
            ref_w = rw
            assert maxerr(traj.w_stored, rw) <= tol["w"]
            # pairs the oracle's own w would select differently at the threshold
            flips = int((O.select_fresh(rw, wl.G, wl.threshold) !=
                         O.select_fresh(traj.w_stored, wl.G, wl.threshold)).sum())
        else:
            ro, rl, _ = O.merge_with_reuse(of, lf, ref_cache[0], ref_cache[1], off, wl.G, mask)
            if policy == "predict":
                # the oracle's own prediction from its own-group states, anchor cache and w;
                # pairs whose predicted error lies within `margin` of the bound may differ
                # (bf16 states on the GPU), every other pair must agree
                d2, r2 = O.state_drift(of, ref_cache[0], off, wl.G, own)
                rmask = O.predict_fresh(ref_w, d2, r2, wl.G, wl.threshold)
                drift = np.sqrt(np.diag(d2.reshape(wl.QG, wl.KG, wl.G).sum(2)) /
                                np.diag(r2.reshape(wl.QG, wl.KG, wl.G).sum(2)))
                pred = (ref_w * drift[:, None]).reshape(wl.QG, wl.KG, wl.G).max(2)
                firm = (np.abs(pred / wl.threshold - 1.0) > margin) | own.astype(bool)
                assert (mask[firm] == rmask[firm]).all(), (s, mask, rmask)
                flips = int((mask != rmask).sum())
        err_o, err_l = maxerr(o, ro), maxerr(lse, rl)
        assert err_o <= tol["o"] and err_l <= tol["lse"], (s, err_o, err_l)
        q_err = q_err_oracle = float("nan")
        if quality_heads:
            # quality numbers: the merged output (GPU, and the oracle's own reuse result on
            # the same mask and cache) against this step's fresh full attention
            hq = slice(0, quality_heads)
            fo, fl, _ = O.partition_states(qf[:, hq], kf[:, hq], vf[:, hq], off, wl.G, ones, wl.scale)
            full_o, _ = O.merge_states(list(fo), list(fl))
            q_err = float(np.abs(o[:, hq] - full_o).max())
            q_err_oracle = float(np.abs(ro[:, hq] - full_o).max())
        report.append((s, int(mask.sum()), err_o, err_l, q_err, q_err_oracle, flips))
    for r in report:
        print("step %d fresh pairs %2d |dO| %.2e |dLSE| %.2e vs fresh full attention: gpu %.3e oracle %.3e "
              "flips %s" % r)
    ctx.close()
    return report


def test_denoising_trajectory_as_specified(pa):
    # threshold 0.05: with these inputs every stored importance is >= ~0.09, so no pair is
    # reused and every step is a full recompute that must still match the oracle.
    wl = W.workload(3)
    report = _run_trajectory(pa, wl, quality_heads=4)
    assert all(r[1] == wl.QG * wl.KG for r in report)


def test_denoising_trajectory_with_reuse(pa):
    # same shape and drift, threshold 0.12 so that the importance-driven reuse path runs
    wl = W.small_variant(W.workload(3), grid=W.workload(3).grid, H=W.workload(3).H, threshold=0.12)
    report = _run_trajectory(pa, wl, quality_heads=4)
    assert report[0][1] == wl.QG * wl.KG and report[5][1] == wl.QG * wl.KG
    assert any(r[1] < wl.QG * wl.KG for r in report)           # reuse happened


def test_denoising_trajectory_on_a_side_stream(pa):
    # every launch of the trajectory on a stream other than torch's current one: the host
    # must still read the anchor's importance only after the merge that writes it
    base = W.workload(3)
    wl = W.small_variant(base, grid=base.grid, H=4, threshold=0.12)
    report = _run_trajectory(pa, wl, side_stream=True)
    assert any(r[1] < wl.QG * wl.KG for r in report)


def test_denoising_trajectory_online_prediction(pa):
    # same shape and drift; between anchors the mask comes from the online prediction
    # (own groups first, their drift from the anchor times the stored importance against
    # an error bound of 1e-3: with these inputs the oracle recomputes 8, 10, 29, 57 of the
    # 64 pairs on the four steps after each anchor -- own groups only on the first, more as
    # the drift grows)
    base = W.workload(3)
    wl = W.small_variant(base, grid=base.grid, H=base.H, threshold=1e-3)
    report = _run_trajectory(pa, wl, quality_heads=4, policy="predict")
    fresh = [r[1] for r in report]
    assert fresh[0] == wl.QG * wl.KG and fresh[5] == wl.QG * wl.KG
    assert fresh[1] == wl.QG and fresh[6] == wl.QG             # own groups only
    assert fresh[4] > fresh[2] and fresh[9] > fresh[7]          # more recomputed as drift grows
    assert fresh[4] < wl.QG * wl.KG


def test_ulysses_layout_full_size(pa):
    from sequence_partition_attn_b200.step import relayout_overlapped
    wl = W.workload(4)
    N, H, D, P = wl.N, wl.H, wl.D, wl.P
    host = W.make_qkv(wl)                                       # seq-major [N][H][D]
    off = W.part_offsets(N, P)
    ctx = pa.Context(0)
    srcs = [host[n].to(DEV) for n in ("q", "k", "v")]
    dsts = [torch.full((1, H, N, D), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    o_ov = torch.full((P, 1, H, N, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    l_ov = torch.full((P, 1, H, N), float("nan"), device=DEV)
    s_copy, s_attn = torch.cuda.Stream(), torch.cuda.Stream()
    cur = torch.cuda.current_stream()
    s_copy.wait_stream(cur)
    s_attn.wait_stream(cur)
    relayout_overlapped(ctx, srcs, dsts, wl.chunks, off, 1, o_ov, l_ov, s_copy, s_attn)
    cur.wait_stream(s_attn)
    cur.wait_stream(s_copy)
    ctx.sync_status()
    # relayout: bit-exact against the oracle's permutation
    for n, d in zip(("q", "k", "v"), dsts):
        ref = O.relayout_seq2head(host[n].view(torch.int16).numpy(), wl.chunks)
        assert np.array_equal(d[0].cpu().view(torch.int16).numpy(), ref), n
    # overlapped chunked attention == one unchunked launch, bit for bit
    o_seq = torch.empty_like(o_ov)
    l_seq = torch.empty_like(l_ov)
    pa.pa_partition_attn(ctx, dsts[0], dsts[1], dsts[2], off, 1, None, o_seq, l_seq)
    o = torch.empty(1, H, N, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(1, H, N, device=DEV)
    pa.pa_merge_states(ctx, off, 1, None, o_ov, l_ov, None, None, o, lse)
    ctx.sync_status()
    assert torch.equal(l_ov, l_seq) and torch.equal(o_ov.view(torch.int16), o_seq.view(torch.int16))
    del o_seq, l_seq, o_ov, l_ov
    # 512 random rows, the first and last 256 rows and a chunk boundary, on every head
    rows = np.unique(np.concatenate([np.random.default_rng(4).choice(N, 512, replace=False),
                                     np.arange(0, 256), np.arange(7200 - 4, 7200 + 4),
                                     np.arange(N - 256, N)]))
    ri = torch.as_tensor(rows, device=DEV)
    go = o.index_select(2, ri).float().cpu().numpy()
    gl = lse.index_select(2, ri).cpu().numpy()
    ones = np.ones((P, P), dtype=np.uint8)
    worst_o = worst_l = 0.0
    for h in range(H):
        x = {n: W.to_f64(host[n][:, h, :])[None, None] for n in ("q", "k", "v")}
        of, lf, _ = O.partition_states(x["q"], x["k"], x["v"], off, 1, ones, wl.scale, rows=rows)
        ro, rl = O.merge_states(list(of), list(lf))
        worst_o = max(worst_o, maxerr(go[0, h], ro[0, 0]))
        worst_l = max(worst_l, maxerr(gl[0, h], rl[0, 0]))
    print("Ulysses layout, sampled rows: |dO| %.3e |dLSE| %.3e" % (worst_o, worst_l))
    assert worst_o <= TOL["bf16"]["o"] and worst_l <= TOL["bf16"]["lse"]
    ctx.close()
