"""fp64 CPU oracle for partition attention with state merge, reuse and importance.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's ``smoke()`` entry and the
benchmark's CPU-baseline / reference arm may import this module.  It is independent of
the CUDA path: it shares no code, constant or helper with it and neither imports the
other.  Inputs come from the seeded generators in ``workloads``.

Everything is computed in float64 with NumPy; a matrix product (``@``), ``exp``, ``log``
and ``max`` are the only library steps.  There is no blocking, fusion or reordering
beyond the definitions below.

What is computed, and where the pages state it (DiTango web summary, Methodology,
"State Composition"; SwiftFusion web summary, Methodology 2 "Torus Attention"):

* partition_states -- the attention state (partial output, log-sum-exp) of each query row
  against one KV partition.  The pages state that such states compose; the exact form
  used is the standard one: for scores s_j = scale * q . k_j over the valid keys j of the
  partition, LSE_p = log sum_j exp(s_j) and O_p = sum_j exp(s_j - LSE_p) v_j.
* merge_states / merge_with_reuse -- the associative, commutative composition of states:
  LSE = log sum_p exp(LSE_p), O = sum_p exp(LSE_p - LSE) O_p, choosing per (query group,
  KV group) the freshly computed or the cached state (DiTango, Methodology 1: which
  partitions are recomputed and which reuse history is decided per group).
* importance -- partition importance w_p = exp(LSE_p - LSE), averaged over batch, heads
  and the valid rows of each query group (DiTango, Methodology 1, error modelling and
  anchor steps: importance is refreshed at anchors).
* select_fresh -- the reuse decision from stored importance: a KV group is recomputed when
  any of its partitions has stored importance >= threshold.
* compose_states / merge_with_composed_cache -- dynamic group compose (DiTango web summary,
  Methodology 2 "Dynamic Group Compose"): cached states of consecutive partitions merge
  into one coarser state with no recomputation, and a reused KV group then contributes
  its single composed state to the merge.
* state_drift / predict_fresh -- online error prediction between anchor steps (DiTango web
  summary, Methodology 1 "Online Prediction": changes of the local states, which are
  always computed, stand in for the drift of the reused remote ones).  state_drift sums,
  per (query group, partition) over the selected pairs, |O_new - O_ref|^2 and |O_ref|^2
  over batch, heads, rows and channels; predict_fresh recomputes a KV group when
  w[qg][p] * sqrt(d2_own / r2_own) >= eps for some partition p of it, where the own
  (diagonal) group's relative drift is the proxy.
* relayout_seq2head -- the sequence-major -> head-major permutation that the Ulysses
  all-to-all performs, here on one device (SwiftFusion, Methodology 2).

Conventions: a partition with no valid keys has LSE_p = -inf and O_p = 0; a row whose
states are all -inf merges to LSE = -inf, O = 0; importance of such a row is 0.

Every function is pinned by tests that do not re-use its code (closed forms, a library
attention routine, brute-force loops on tiny inputs, invariants and a hand-worked
fixture).  None is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "partition_states", "merge_states", "merge_with_reuse", "importance",
    "select_fresh", "relayout_seq2head", "group_bounds", "compose_states",
    "merge_with_composed_cache", "state_drift", "predict_fresh",
]


def group_bounds(part_off: np.ndarray, G: int) -> np.ndarray:
    """Token bounds of the G-partition groups: group g = partitions [gG, (g+1)G)."""
    P = len(part_off) - 1
    QG = -(-P // G)
    return np.array([int(part_off[min(g * G, P)]) for g in range(QG + 1)], dtype=np.int64)


def _row_groups(rows: np.ndarray, part_off: np.ndarray, G: int) -> np.ndarray:
    gb = group_bounds(part_off, G)
    return np.searchsorted(gb, rows, side="right") - 1


def partition_states(q, k, v, part_off, G, fresh, scale, rows=None):
    """Per-partition attention states for the selected (query group, KV group) pairs.

    q, k, v: float64 [B, H, N, D] (head-major).  part_off: int[P+1].  fresh: uint8
    [QG, KG] (1 = compute).  rows: query rows to produce (default: all N).

    Returns (o_part [P, B, H, R, D], lse_part [P, B, H, R], selected bool [P, R]).
    Entries of pairs that are not selected are NaN.
    """
    B, H, N, D = q.shape
    P = len(part_off) - 1
    rows = np.arange(N) if rows is None else np.asarray(rows)
    R = len(rows)
    qg_of_row = _row_groups(rows, part_off, G)
    o_part = np.full((P, B, H, R, D), np.nan)
    lse_part = np.full((P, B, H, R), np.nan)
    selected = np.zeros((P, R), dtype=bool)
    for p in range(P):
        kg = p // G
        sel = np.nonzero(fresh[qg_of_row, kg] != 0)[0]
        if len(sel) == 0:
            continue
        selected[p, sel] = True
        lo, hi = int(part_off[p]), int(part_off[p + 1])
        if hi <= lo:
            lse_part[p][:, :, sel] = -np.inf
            o_part[p][:, :, sel, :] = 0.0
            continue
        for b in range(B):
            for h in range(H):
                s = scale * (q[b, h, rows[sel], :] @ k[b, h, lo:hi, :].T)   # [r, n_p]
                m = s.max(axis=1, keepdims=True)
                lse = m + np.log(np.exp(s - m).sum(axis=1, keepdims=True))
                o = np.exp(s - lse) @ v[b, h, lo:hi, :]
                lse_part[p, b, h, sel] = lse[:, 0]
                o_part[p, b, h, sel, :] = o
    return o_part, lse_part, selected


def merge_states(o_list, lse_list):
    """Compose states: LSE = logsumexp_p LSE_p, O = sum_p exp(LSE_p - LSE) O_p.

    o_list: sequence of arrays [..., D]; lse_list: matching arrays [...].  Indices are
    taken in the given order.  Returns (O, LSE).
    """
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lse_list], axis=0)
    O = np.stack([np.asarray(x, dtype=np.float64) for x in o_list], axis=0)
    m = L.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    ssum = np.exp(L - m_safe[None]).sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, ssum, 1.0)), -np.inf)
    wts = np.where(finite[None], np.exp(L - np.where(finite, lse, 0.0)[None]), 0.0)
    o = (wts[..., None] * np.where(np.isfinite(L)[..., None], O, 0.0)).sum(axis=0)
    return o, lse


def merge_with_reuse(o_fresh, lse_fresh, o_cached, lse_cached, part_off, G, fresh, rows=None):
    """Merge per row the fresh or the cached state of every partition.

    State arrays are [P, B, H, R(, D)] over the rows ``rows`` (default all N).  The
    state of partition p for a row in query group qg is the fresh one when
    fresh[qg, p // G] else the cached one.

    Returns (O [B, H, R, D], LSE [B, H, R], chosen_lse [P, B, H, R]).
    """
    P = len(part_off) - 1
    R = lse_fresh.shape[-1]
    rows = np.arange(R) if rows is None else np.asarray(rows)
    qg_of_row = _row_groups(rows, part_off, G)
    o_sel, l_sel = [], []
    for p in range(P):
        use_fresh = (fresh[qg_of_row, p // G] != 0)                    # [R]
        l_sel.append(np.where(use_fresh[None, None, :], lse_fresh[p], lse_cached[p]))
        o_sel.append(np.where(use_fresh[None, None, :, None], o_fresh[p], o_cached[p]))
    O, L = merge_states(o_sel, l_sel)
    return O, L, np.stack(l_sel, axis=0)


def compose_states(o_part, lse_part, factor):
    """Merge the states of every `factor` consecutive partitions into one.

    o_part [P, ...rows, D], lse_part [P, ...rows] -> ([ceil(P/factor), ...], [...]); group c
    is the composition of partitions c*factor .. min((c+1)*factor, P) - 1.
    """
    P = lse_part.shape[0]
    C = -(-P // factor)
    outs = [merge_states(list(o_part[c * factor:(c + 1) * factor]),
                         list(lse_part[c * factor:(c + 1) * factor])) for c in range(C)]
    return np.stack([o for o, _ in outs]), np.stack([l for _, l in outs])


def merge_with_composed_cache(o_fresh, lse_fresh, o_comp, lse_comp, part_off, G, fresh, rows=None):
    """Merge per row: for KV group kg, the fresh per-partition states of its partitions when
    fresh[qg, kg], else its one composed cached state o_comp[kg], lse_comp[kg].

    o_fresh [P, B, H, R, D]; o_comp [KG, B, H, R, D].  Returns (O, LSE).
    """
    P = len(part_off) - 1
    KG = -(-P // G)
    R = lse_fresh.shape[-1]
    rows = np.arange(R) if rows is None else np.asarray(rows)
    qg_of_row = _row_groups(rows, part_off, G)
    o_sel, l_sel = [], []
    for kg in range(KG):
        use_fresh = (fresh[qg_of_row, kg] != 0)                       # [R]
        for p in range(kg * G, min((kg + 1) * G, P)):
            if p == kg * G:
                # the group's first slot carries the cached state where reused
                l_sel.append(np.where(use_fresh[None, None, :], lse_fresh[p], lse_comp[kg]))
                o_sel.append(np.where(use_fresh[None, None, :, None], o_fresh[p], o_comp[kg]))
            else:
                # further partitions only where fresh; reused rows take nothing (-inf)
                l_sel.append(np.where(use_fresh[None, None, :], lse_fresh[p], -np.inf))
                o_sel.append(np.where(use_fresh[None, None, :, None], o_fresh[p], 0.0))
    return merge_states(o_sel, l_sel)


def importance(lse_part, lse, part_off, G, rows=None):
    """w[qg, p] = mean over batch, heads and rows of qg of exp(LSE_p(row) - LSE(row)).

    lse_part: [P, B, H, R] (the states that were merged), lse: [B, H, R].  The mean runs
    over the rows given (default all N rows).
    """
    P = lse_part.shape[0]
    R = lse.shape[-1]
    rows = np.arange(R) if rows is None else np.asarray(rows)
    qg_of_row = _row_groups(rows, part_off, G)
    QG = len(group_bounds(part_off, G)) - 1
    fin = np.isfinite(lse)
    per_row = np.where(fin[None], np.exp(lse_part - np.where(fin, lse, 0.0)[None]), 0.0)
    w = np.zeros((QG, P))
    for g in range(QG):
        cols = np.nonzero(qg_of_row == g)[0]
        if len(cols):
            w[g] = per_row[:, :, :, cols].mean(axis=(1, 2, 3))
    return w


def select_fresh(w_stored, G, threshold):
    """uint8[QG, KG]: KV group kg is recomputed for query group qg when any partition p in
    kg has w_stored[qg, p] >= threshold; otherwise its cached states are reused."""
    QG, P = w_stored.shape
    KG = -(-P // G)
    m = np.zeros((QG, KG), dtype=np.uint8)
    for g in range(QG):
        for kg in range(KG):
            m[g, kg] = 1 if np.any(w_stored[g, kg * G:(kg + 1) * G] >= threshold) else 0
    return m


def state_drift(o_new, o_ref, part_off, G, sel):
    """(d2, r2), each [QG, P]: for every pair (query group qg, partition p) with
    sel[qg, p // G], the sums over batch, heads, rows of qg and channels of
    (o_new - o_ref)^2 and o_ref^2; 0 for other pairs.  o_new, o_ref: [P, B, H, N, D]."""
    P = len(part_off) - 1
    gb = group_bounds(part_off, G)
    QG = len(gb) - 1
    d2 = np.zeros((QG, P))
    r2 = np.zeros((QG, P))
    for qg in range(QG):
        r0, r1 = int(gb[qg]), int(gb[qg + 1])
        for p in range(P):
            if not sel[qg, p // G]:
                continue
            a = o_new[p][:, :, r0:r1, :].astype(np.float64)
            b = o_ref[p][:, :, r0:r1, :].astype(np.float64)
            d2[qg, p] = ((a - b) ** 2).sum()
            r2[qg, p] = (b ** 2).sum()
    return d2, r2


def predict_fresh(w_stored, d2, r2, G, eps):
    """uint8[QG, KG]: recompute KV group kg for query group qg when some partition p of kg
    has w_stored[qg, p] * drift[qg] >= eps, drift[qg] = sqrt(sum_p d2[qg, p] / sum_p r2[qg, p])
    over the partitions of the own group kg = qg (0 when nothing was measured).  The own
    group is always recomputed."""
    QG, P = w_stored.shape
    KG = -(-P // G)
    m = np.zeros((QG, KG), dtype=np.uint8)
    for qg in range(QG):
        own = slice(qg * G, min((qg + 1) * G, P))
        den = r2[qg, own].sum()
        drift = np.sqrt(d2[qg, own].sum() / den) if den > 0 else 0.0
        for kg in range(KG):
            pred = max(w_stored[qg, p] * drift for p in range(kg * G, min((kg + 1) * G, P)))
            m[qg, kg] = 1 if (kg == qg or pred >= eps) else 0
    return m


def relayout_seq2head(src, n_chunks=1):
    """[N, H, D] -> [H, N, D]: dst[h, n, :] = src[n, h, :], chunk by chunk along n."""
    N, H, D = src.shape
    dst = np.empty((H, N, D), dtype=src.dtype)
    step = -(-N // n_chunks)
    for c in range(n_chunks):
        lo, hi = c * step, min((c + 1) * step, N)
        for h in range(H):
            dst[h, lo:hi, :] = src[lo:hi, h, :]
    return dst
