"""Shared test plumbing: run the CUDA path (through the C ABI binding) and the fp64 oracle
on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import workloads as W

# Tolerances (stated by the workloads: bf16 inputs with fp32 accumulation; fp32 inputs).
TOL = {"bf16": dict(o=2e-2, lse=1e-3, w=1e-3), "f32": dict(o=1e-4, lse=1e-4, w=1e-4)}


def gpu_states(pa, ctx, wl, q, k, v, off, G, fresh):
    """Device partition states for the fresh pairs (unselected entries stay NaN)."""
    P, B, H, N, D = len(off) - 1, q.shape[0], q.shape[1], q.shape[2], q.shape[3]
    o = torch.full((P, B, H, N, D), float("nan"), dtype=q.dtype, device=q.device)
    l = torch.full((P, B, H, N), float("nan"), dtype=torch.float32, device=q.device)
    pa.pa_partition_attn(ctx, q, k, v, off, G, fresh, o, l, scale=wl.scale)
    return o, l


def maxerr(a, b, mask=None):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if mask is not None:
        a, b = a[mask], b[mask]
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        d = np.where(both_inf, 0.0, np.abs(a - b))
    if d.size and np.isnan(d).any():
        return float("inf")                 # a NaN where a value is due fails every tolerance
    return float(d.max()) if d.size else 0.0


def run_reuse_case(pa, ctx, wl, fresh=None, rows=None):
    """Fresh states on (Q, K, V) for the mask, cached states on (Q, K_prev, V_prev) for
    every pair, merge with fused importance; the oracle does the same on the same inputs.

    Returns a dict of (gpu, oracle) arrays.  ``rows`` restricts the oracle (and the
    comparison) to those query rows; the oracle then runs head by head.
    """
    dev = torch.device("cuda:0")
    t = W.make_qkv(wl)
    off = W.part_offsets(wl.N, wl.P)
    if fresh is None:
        fresh = W.reuse_mask(wl)
    ones = np.ones_like(fresh)
    q, k, v = (t[n].to(dev) for n in ("q", "k", "v"))
    if wl.cache_sigma > 0:
        kc, vc = W.make_cached_kv(wl, t["k"], t["v"])
    else:
        kc, vc = t["k"], t["v"]
    of, lf = gpu_states(pa, ctx, wl, q, k, v, off, wl.G, fresh)
    oc, lc = gpu_states(pa, ctx, wl, q, kc.to(dev), vc.to(dev), off, wl.G, ones)
    B, H, N, D = q.shape
    o = torch.empty(B, H, N, D, dtype=q.dtype, device=dev)
    lse = torch.empty(B, H, N, device=dev)
    w = torch.empty(wl.QG, wl.P, device=dev)
    pa.pa_merge_states(ctx, off, wl.G, fresh, of, lf, oc, lc, o, lse, w)
    ctx.sync_status()
    g = dict(of=of, lf=lf, oc=oc, lc=lc, o=o, lse=lse, w=w)
    del q, k, v
    rows_np = np.arange(N) if rows is None else np.asarray(rows)
    gpu = {}
    for name in ("of", "oc", "o"):
        x = g[name]
        gpu[name] = x.index_select(-2, torch.as_tensor(rows_np, device=dev)).float().cpu().numpy()
    for name in ("lf", "lc", "lse"):
        gpu[name] = g[name].index_select(-1, torch.as_tensor(rows_np, device=dev)).cpu().numpy()
    gpu["w"] = w.cpu().numpy()
    del g, of, lf, oc, lc, o, lse
    torch.cuda.empty_cache()

    # Oracle, head by head (bounded memory at full sizes).
    P, R = wl.P, len(rows_np)
    oracle = dict(of=np.empty((P, B, H, R, D)), lf=np.empty((P, B, H, R)),
                  oc=np.empty((P, B, H, R, D)), lc=np.empty((P, B, H, R)),
                  o=np.empty((B, H, R, D)), lse=np.empty((B, H, R)), chosen=np.empty((P, B, H, R)))
    for b in range(B):
        for h in range(H):
            qf, kf, vf, kcf, vcf = (W.to_f64(x[b:b + 1, h:h + 1])
                                    for x in (t["q"], t["k"], t["v"], kc, vc))
            rof, rlf, _ = O.partition_states(qf, kf, vf, off, wl.G, fresh, wl.scale, rows=rows_np)
            roc, rlc, _ = O.partition_states(qf, kcf, vcf, off, wl.G, ones, wl.scale, rows=rows_np)
            ro, rl, ch = O.merge_with_reuse(rof, rlf, roc, rlc, off, wl.G, fresh, rows=rows_np)
            for n, x in (("of", rof), ("lf", rlf), ("oc", roc), ("lc", rlc), ("chosen", ch)):
                oracle[n][:, b, h] = x[:, 0, 0]
            oracle["o"][b, h] = ro[0, 0]
            oracle["lse"][b, h] = rl[0, 0]
    oracle["w"] = O.importance(oracle["chosen"], oracle["lse"], off, wl.G, rows=rows_np)
    qg_of_row = np.searchsorted(O.group_bounds(off, wl.G), rows_np, side="right") - 1
    sel_mask = np.stack([fresh[qg_of_row, p // wl.G] != 0 for p in range(wl.P)])   # [P, R]
    return gpu, oracle, sel_mask, off, fresh


def compare_states(gpu, oracle, sel_mask, tol):
    """Max errors of the fresh states (selected pairs), cached states, O, LSE."""
    P, B, H, R = oracle["lf"].shape
    m4 = np.broadcast_to(sel_mask[:, None, None, :], (P, B, H, R))
    m5 = np.broadcast_to(m4[..., None], oracle["of"].shape)
    errs = dict(
        of=maxerr(gpu["of"], oracle["of"], m5), lf=maxerr(gpu["lf"], oracle["lf"], m4),
        oc=maxerr(gpu["oc"], oracle["oc"]), lc=maxerr(gpu["lc"], oracle["lc"]),
        o=maxerr(gpu["o"], oracle["o"]), lse=maxerr(gpu["lse"], oracle["lse"]))
    # unselected fresh entries must be untouched (NaN sentinel)
    untouched = bool(np.all(np.isnan(gpu["lf"][~m4]))) if (~m4).any() else True
    return errs, untouched
