"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics, not by the
oracle's own code.

* a library attention routine (torch scaled_dot_product_attention in float64) and
  scipy's logsumexp -- all-fresh merging must reach full softmax attention (DiTango
  web summary, Methodology 2 "State Composition": caching composable states loses
  nothing when every partition is fresh);
* closed forms: zero queries (uniform softmax, LSE_p = log n_p, w_p = n_p/N), identical
  keys, a single partition, an asymmetric reuse mask with constant values;
* invariants: merge order and merge-tree shape (associative and commutative
  composition), group-then-global composition (DiTango, Methodology 2 "Dynamic group
  compose"), all-ones mask = full recompute, unperturbed cache = fresh result,
  sum_p w_p = 1;
* brute force with pure-Python loops and math.exp on tiny inputs;
* a hand-worked fixture (tests/golden/hand_worked_states.json);
* the relayout against an index-encoding closed form (SwiftFusion web summary,
  Methodology 2 "Torus Attention": the chunked all-to-all moves data, nothing else);
* property-based: the merge against the direct softmax-weighted sum, group splits and
  the weights' sum on any states drawn by hypothesis, empty ones included.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st
from scipy.special import logsumexp

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_qkv(seed, B, H, N, D, scale_v=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    v = scale_v * rng.standard_normal((B, H, N, D))
    return q, k, v


def all_fresh(P, G=1):
    QG = -(-P // G)
    return np.ones((QG, QG), dtype=np.uint8)


# --------------------------------------------------------------------------- library pin
@pytest.mark.parametrize("N,P,D", [(50, 4, 16), (37, 5, 8), (64, 1, 32), (130, 7, 64)])
def test_all_fresh_merge_equals_library_attention(N, P, D):
    q, k, v = rand_qkv(N + P, 2, 3, N, D)
    off = W.part_offsets(N, P)
    scale = 1.0 / math.sqrt(D)
    op, lp, sel = O.partition_states(q, k, v, off, 1, all_fresh(P), scale)
    assert sel.all()
    o, lse = O.merge_states(list(op), list(lp))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    ref_lse = logsumexp(scale * np.einsum("bhid,bhjd->bhij", q, k), axis=-1)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_partition_state_equals_library_attention_on_its_keys():
    q, k, v = rand_qkv(3, 1, 2, 40, 16)
    off = W.part_offsets(40, 3)          # 14, 14, 12
    op, lp, _ = O.partition_states(q, k, v, off, 1, all_fresh(3), 0.25)
    for p in range(3):
        lo, hi = off[p], off[p + 1]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k[:, :, lo:hi]),
            torch.from_numpy(v[:, :, lo:hi]), scale=0.25).numpy()
        np.testing.assert_allclose(op[p], ref, atol=1e-12, rtol=0)
        ref_l = logsumexp(0.25 * np.einsum("bhid,bhjd->bhij", q, k[:, :, lo:hi]), axis=-1)
        np.testing.assert_allclose(lp[p], ref_l, atol=1e-12, rtol=0)


# --------------------------------------------------------------------------- closed forms
def test_zero_query_closed_form_with_ragged_tail():
    # 720p partitioning: S = 2363, the last partition holds 2347 valid tokens.
    wl = W.workload(2)
    off = W.part_offsets(wl.N, wl.P)
    assert off[-1] - off[-2] == 2347 and off[1] - off[0] == 2363
    # Zero queries on a reduced head count / dim, all keys, three query rows.
    rng = np.random.default_rng(5)
    D = 8
    k = rng.standard_normal((1, 1, wl.N, D))
    v = rng.standard_normal((1, 1, wl.N, D))
    q = np.zeros((1, 1, wl.N, D))
    rows = np.array([0, 40000, wl.N - 1])
    fresh = all_fresh(wl.P, wl.G)
    op, lp, _ = O.partition_states(q, k, v, off, wl.G, fresh, 1 / math.sqrt(D), rows=rows)
    n_p = np.diff(off).astype(np.float64)
    for p in range(wl.P):
        np.testing.assert_allclose(lp[p, 0, 0], np.log(n_p[p]), rtol=0, atol=1e-12)
        mean_v = v[0, 0, off[p]:off[p + 1]].mean(axis=0)
        np.testing.assert_allclose(op[p, 0, 0], np.broadcast_to(mean_v, (3, D)), atol=1e-12)
    assert abs(lp[-1, 0, 0, 0] - math.log(2347)) < 1e-12
    o, lse = O.merge_states(list(op), list(lp))
    np.testing.assert_allclose(lse, math.log(wl.N), atol=1e-12)
    w = O.importance(lp, lse, off, wl.G, rows=rows)
    # zero queries: w_p = n_p / N for every query group that has rows
    for g in np.unique(np.searchsorted(O.group_bounds(off, wl.G), rows, side="right") - 1):
        np.testing.assert_allclose(w[g], n_p / wl.N, atol=1e-12)


def test_identical_keys_give_uniform_softmax():
    rng = np.random.default_rng(8)
    N, D = 20, 4
    q = rng.standard_normal((1, 1, N, D))
    kk = rng.standard_normal(D)
    k = np.broadcast_to(kk, (1, 1, N, D)).copy()
    v = rng.standard_normal((1, 1, N, D))
    off = W.part_offsets(N, 3)                 # 7, 7, 6
    op, lp, _ = O.partition_states(q, k, v, off, 1, all_fresh(3), 0.5)
    for p in range(3):
        lo, hi = off[p], off[p + 1]
        s = 0.5 * q[0, 0] @ kk
        np.testing.assert_allclose(lp[p, 0, 0], s + math.log(hi - lo), atol=1e-12)
        np.testing.assert_allclose(op[p, 0, 0], np.broadcast_to(v[0, 0, lo:hi].mean(0), (N, D)),
                                   atol=1e-12)


def test_single_partition_state_is_the_merged_state_and_w_is_one():
    q, k, v = rand_qkv(11, 1, 2, 33, 8)
    off = W.part_offsets(33, 1)
    op, lp, _ = O.partition_states(q, k, v, off, 1, all_fresh(1), 0.3)
    o, lse = O.merge_states(list(op), list(lp))
    np.testing.assert_array_equal(lse, lp[0])
    np.testing.assert_allclose(o, op[0], atol=1e-15)
    w = O.importance(lp, lse, off, 1)
    np.testing.assert_allclose(w, [[1.0]], atol=1e-15)


def test_asymmetric_mask_orientation_closed_form():
    # Zero queries, fresh V constant a, cached V constant c: a row of query group g merges
    # sum_p (n_p/N) * (a if fresh[g, kg(p)] else c).  A transposed mask or a swapped
    # fresh/cached choice fails.
    N, D, P, G = 23, 4, 6, 2                  # S = 4: partitions 4,4,4,4,4,3
    off = W.part_offsets(N, P)
    q = np.zeros((1, 1, N, D))
    k = np.random.default_rng(1).standard_normal((1, 1, N, D))
    a, c = 1.0, -2.0
    v_fresh = np.full((1, 1, N, D), a)
    v_cached = np.full((1, 1, N, D), c)
    fresh = np.array([[1, 0, 0], [1, 1, 0], [0, 0, 1]], dtype=np.uint8)
    ones = all_fresh(P, G)
    of, lf, _ = O.partition_states(q, k, v_fresh, off, G, ones, 0.5)
    oc, lc, _ = O.partition_states(q, k, v_cached, off, G, ones, 0.5)
    o, lse, chosen = O.merge_with_reuse(of, lf, oc, lc, off, G, fresh)
    n_p = np.diff(off)
    gb = O.group_bounds(off, G)
    for row in range(N):
        g = np.searchsorted(gb, row, side="right") - 1
        expect = sum(n_p[p] / N * (a if fresh[g, p // G] else c) for p in range(P))
        np.testing.assert_allclose(o[0, 0, row], expect, atol=1e-12)
    np.testing.assert_allclose(lse, math.log(N), atol=1e-12)


# --------------------------------------------------------------------------- invariants
def _random_states(seed, P, R=5, D=3):
    rng = np.random.default_rng(seed)
    lse = rng.normal(scale=3.0, size=(P, R))
    o = rng.standard_normal((P, R, D))
    return o, lse


def test_merge_is_order_invariant():
    o, l = _random_states(0, 6)
    ref_o, ref_l = O.merge_states(list(o), list(l))
    rng = np.random.default_rng(1)
    for _ in range(20):
        perm = rng.permutation(6)
        mo, ml = O.merge_states([o[i] for i in perm], [l[i] for i in perm])
        np.testing.assert_allclose(mo, ref_o, atol=1e-12)
        np.testing.assert_allclose(ml, ref_l, atol=1e-12)


def test_merge_is_tree_shape_invariant():
    o, l = _random_states(2, 7)
    ref_o, ref_l = O.merge_states(list(o), list(l))
    rng = np.random.default_rng(3)
    for _ in range(20):
        items = [(o[i], l[i]) for i in rng.permutation(7)]
        while len(items) > 1:              # random binary tree of pairwise merges
            i = int(rng.integers(0, len(items) - 1))
            a, b = items[i], items[i + 1]
            items[i:i + 2] = [O.merge_states([a[0], b[0]], [a[1], b[1]])]
        np.testing.assert_allclose(items[0][0], ref_o, atol=1e-12)
        np.testing.assert_allclose(items[0][1], ref_l, atol=1e-12)


def test_group_then_global_equals_flat():
    o, l = _random_states(4, 8)
    ref_o, ref_l = O.merge_states(list(o), list(l))
    groups = [O.merge_states(list(o[g:g + 4]), list(l[g:g + 4])) for g in (0, 4)]
    mo, ml = O.merge_states([g[0] for g in groups], [g[1] for g in groups])
    np.testing.assert_allclose(mo, ref_o, atol=1e-12)
    np.testing.assert_allclose(ml, ref_l, atol=1e-12)


def test_minus_inf_states_contribute_nothing():
    o, l = _random_states(5, 3)
    l2 = np.concatenate([l, np.full((1, l.shape[1]), -np.inf)])
    o2 = np.concatenate([o, np.full((1,) + o.shape[1:], 7.0)])
    a = O.merge_states(list(o), list(l))
    b = O.merge_states(list(o2), list(l2))
    np.testing.assert_allclose(b[0], a[0], atol=1e-15)
    np.testing.assert_allclose(b[1], a[1], atol=1e-15)
    z = O.merge_states([o[0]], [np.full(l.shape[1], -np.inf)])
    assert np.all(z[1] == -np.inf) and np.all(z[0] == 0)


def test_all_ones_mask_ignores_the_cache():
    q, k, v = rand_qkv(6, 1, 2, 30, 8)
    off = W.part_offsets(30, 4)
    of, lf, _ = O.partition_states(q, k, v, off, 2, all_fresh(4, 2), 0.35)
    oc = np.full_like(of, np.nan)
    lc = np.full_like(lf, np.nan)
    o, lse, _ = O.merge_with_reuse(of, lf, oc, lc, off, 2, all_fresh(4, 2))
    ro, rl = O.merge_states(list(of), list(lf))
    assert np.isfinite(o).all()
    np.testing.assert_array_equal(o, ro)
    np.testing.assert_array_equal(lse, rl)


def test_unperturbed_cache_gives_the_fresh_result():
    q, k, v = rand_qkv(7, 1, 2, 41, 8)
    off = W.part_offsets(41, 5)
    ones = all_fresh(5)
    of, lf, _ = O.partition_states(q, k, v, off, 1, ones, 0.35)
    fresh = np.eye(5, dtype=np.uint8)
    oc, lc, _ = O.partition_states(q, k.copy(), v.copy(), off, 1, ones, 0.35)
    o, lse, _ = O.merge_with_reuse(of, lf, oc, lc, off, 1, fresh)
    ro, rl = O.merge_states(list(of), list(lf))
    np.testing.assert_allclose(o, ro, atol=1e-14)
    np.testing.assert_allclose(lse, rl, atol=1e-14)


def test_importance_rows_sum_to_one():
    q, k, v = rand_qkv(9, 2, 3, 57, 8)
    off = W.part_offsets(57, 6)
    of, lf, _ = O.partition_states(q, k, v, off, 2, all_fresh(6, 2), 0.35)
    o, lse = O.merge_states(list(of), list(lf))
    w = O.importance(lf, lse, off, 2)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-12)
    assert (w >= 0).all()


def test_select_fresh_threshold():
    w = np.array([[0.5, 0.04, 0.05, 0.0], [0.01, 0.02, 0.9, 0.049999]])
    np.testing.assert_array_equal(O.select_fresh(w, 1, 0.05), [[1, 0, 1, 0], [0, 0, 1, 0]])
    np.testing.assert_array_equal(O.select_fresh(w, 2, 0.05), [[1, 1], [0, 1]])


# --------------------------------------------------------------------------- brute force
def _brute(q, k, v, off, G, fresh, scale, kc, vc):
    """Pure-Python loops with math.exp; independent restatement for tiny inputs."""
    B, H, N, D = q.shape
    P = len(off) - 1
    QG = -(-P // G)
    gb = [off[min(g * G, P)] for g in range(QG + 1)]
    res_o = np.zeros((B, H, N, D))
    res_l = np.zeros((B, H, N))
    w = np.zeros((QG, P))
    cnt = np.zeros(QG)
    for b, h, i in itertools.product(range(B), range(H), range(N)):
        g = max(j for j in range(QG) if gb[j] <= i)
        states = []
        for p in range(P):
            kk, vv = (k, v) if fresh[g][p // G] else (kc, vc)
            scores = [scale * sum(q[b, h, i, d] * kk[b, h, j, d] for d in range(D))
                      for j in range(off[p], off[p + 1])]
            tot = sum(math.exp(s) for s in scores)
            if not scores:                      # empty partition: LSE -inf, O = 0
                states.append((-math.inf, [0.0] * D))
                continue
            lp = math.log(tot)
            op = [sum(math.exp(s) / tot * vv[b, h, j, d]
                      for s, j in zip(scores, range(off[p], off[p + 1]))) for d in range(D)]
            states.append((lp, op))
        big = sum(math.exp(lp) for lp, _ in states)
        res_l[b, h, i] = math.log(big)
        for d in range(D):
            res_o[b, h, i, d] = sum(math.exp(lp) / big * op[d] for lp, op in states)
        for p, (lp, _) in enumerate(states):
            w[g, p] += math.exp(lp) / big
        cnt[g] += 1
    return res_o, res_l, w / np.maximum(cnt, 1)[:, None]   # a group with no rows: w = 0


@pytest.mark.parametrize("N,P,G", [(2, 1, 1), (3, 2, 1), (9, 3, 1), (16, 5, 2), (13, 4, 2)])
def test_brute_force_tiny(N, P, G):
    rng = np.random.default_rng(N * 10 + P)
    B, H, D = 1, 2, 3
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    v = rng.standard_normal((B, H, N, D))
    kc = k + 0.1 * rng.standard_normal(k.shape)
    vc = v + 0.1 * rng.standard_normal(v.shape)
    off = W.part_offsets(N, P)
    QG = -(-P // G)
    fresh = (rng.random((QG, QG)) < 0.5).astype(np.uint8)
    scale = 0.7
    ones = all_fresh(P, G)
    of, lf, _ = O.partition_states(q, k, v, off, G, ones, scale)
    oc, lc, _ = O.partition_states(q, kc, vc, off, G, ones, scale)
    o, lse, chosen = O.merge_with_reuse(of, lf, oc, lc, off, G, fresh)
    w = O.importance(chosen, lse, off, G)
    bo, bl, bw = _brute(q, k, v, list(off), G, fresh, scale, kc, vc)
    np.testing.assert_allclose(o, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)
    np.testing.assert_allclose(w, bw, atol=1e-12)


def test_two_key_hand_expansion():
    # N = 2, one partition: LSE = log(e^{s0} + e^{s1}), O = softmax-weighted v.
    q = np.array([[[[0.3, -1.2]]]]).repeat(2, axis=2)
    k = np.array([[[[1.0, 0.5], [-0.4, 2.0]]]])
    v = np.array([[[[1.0, 2.0], [3.0, -1.0]]]])
    s0 = 0.5 * (0.3 * 1.0 + -1.2 * 0.5)
    s1 = 0.5 * (0.3 * -0.4 + -1.2 * 2.0)
    op, lp, _ = O.partition_states(q, k, v, np.array([0, 2]), 1, all_fresh(1), 0.5)
    e0, e1 = math.exp(s0), math.exp(s1)
    assert abs(lp[0, 0, 0, 0] - math.log(e0 + e1)) < 1e-14
    np.testing.assert_allclose(op[0, 0, 0, 0], [(e0 * 1 + e1 * 3) / (e0 + e1),
                                                (e0 * 2 - e1 * 1) / (e0 + e1)], atol=1e-14)


# --------------------------------------------------------------------------- golden fixture
def _val(s):
    s = s.strip()
    neg = s.startswith("-")
    body = s[1:] if neg else s
    if body.startswith("2*ln(") and body.endswith(")"):
        x = 2 * math.log(float(Fraction(body[5:-1])))
    elif body.startswith("ln(") and body.endswith(")"):
        x = math.log(float(Fraction(body[3:-1])))
    else:
        x = float(Fraction(body))
    return -x if neg else x


def _arr(x):
    if isinstance(x, str):
        return _val(x)
    return np.array([_arr(e) for e in x], dtype=np.float64)


def test_hand_worked_fixture():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_states.json")))
    q, k, v = (_arr(g[n])[None, None] for n in ("q", "k", "v"))
    kp, vp = (_arr(g[n])[None, None] for n in ("k_prev", "v_prev"))
    off = np.array(g["part_off"])
    scale = _val(g["scale"])
    ones = np.array(g["fresh_all"], dtype=np.uint8)
    of, lf, _ = O.partition_states(q, k, v, off, 1, ones, scale)
    np.testing.assert_allclose(lf[:, 0, 0], _arr(g["expected_lse_part"]), atol=1e-13)
    np.testing.assert_allclose(of[:, 0, 0], _arr(g["expected_o_part"]), atol=1e-13)
    o, lse, chosen = O.merge_with_reuse(of, lf, of, lf, off, 1, ones)
    np.testing.assert_allclose(lse[0, 0], _arr(g["expected_lse"]), atol=1e-13)
    np.testing.assert_allclose(o[0, 0], _arr(g["expected_o"]), atol=1e-13)
    np.testing.assert_allclose(O.importance(chosen, lse, off, 1), _arr(g["expected_w"]),
                               atol=1e-13)
    oc, lc, _ = O.partition_states(q, kp, vp, off, 1, ones, scale)
    reuse = np.array(g["fresh_reuse"], dtype=np.uint8)
    o2, l2, _ = O.merge_with_reuse(of, lf, oc, lc, off, 1, reuse)
    np.testing.assert_allclose(o2[0, 0], _arr(g["expected_o_reuse"]), atol=1e-13)
    np.testing.assert_allclose(l2[0, 0], _arr(g["expected_lse_reuse"]), atol=1e-13)


# --------------------------------------------------------------------------- relayout
@pytest.mark.parametrize("N,H,D,chunks", [(48, 3, 4, 1), (50, 5, 8, 16), (7, 2, 2, 3)])
def test_relayout_index_encoding(N, H, D, chunks):
    n, h, d = np.meshgrid(np.arange(N), np.arange(H), np.arange(D), indexing="ij")
    src = (n * 1_000_000 + h * 1_000 + d).astype(np.int64)
    dst = O.relayout_seq2head(src, chunks)
    assert dst.shape == (H, N, D)
    hh, nn, dd = np.meshgrid(np.arange(H), np.arange(N), np.arange(D), indexing="ij")
    np.testing.assert_array_equal(dst // 1_000_000, nn)
    np.testing.assert_array_equal((dst // 1_000) % 1_000, hh)
    np.testing.assert_array_equal(dst % 1_000, dd)


def test_relayout_round_trip_on_bf16_bits():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 16, size=(33, 4, 8), dtype=np.uint16)
    dst = O.relayout_seq2head(bits, 4)
    back = O.relayout_seq2head(dst, 1)     # [H, N, D] seen as [N', H', D] -> [N, H, D]
    np.testing.assert_array_equal(back, bits)


# --------------------------------------------------------------------------- generators
def test_positional_embedding_channels():
    pe = W.pe_3d((2, 3, 4), 64)            # d_a = 20 channels per axis, 4 zero channels
    coords = W.token_coords((2, 3, 4))
    assert pe.shape == (24, 64)
    np.testing.assert_allclose(pe[:, 0], np.sin(coords[:, 0]), atol=1e-6)      # t, om_0 = 1
    np.testing.assert_allclose(pe[:, 10], np.cos(coords[:, 0]), atol=1e-6)
    np.testing.assert_allclose(pe[:, 20], np.sin(coords[:, 1]), atol=1e-6)     # h
    np.testing.assert_allclose(pe[:, 40], np.sin(coords[:, 2]), atol=1e-6)     # w
    np.testing.assert_allclose(pe[:, 41], np.sin(coords[:, 2] * 10000 ** (-2 / 20)), atol=1e-6)
    assert np.all(pe[:, 60:] == 0)
    assert coords[13].tolist() == [1, 0, 1]          # t-major flattening


def test_workload_tables_match_the_configuration_text():
    wl2 = W.workload(2)
    assert (wl2.N, wl2.S, wl2.QG) == (75600, 2363, 8)
    m = W.reuse_mask(wl2)
    assert [list(np.nonzero(r)[0]) for r in m] == [[0, 1], [1, 2], [1, 2], [2, 3],
                                                  [4, 5], [5, 6], [5, 6], [6, 7]]
    m1 = W.reuse_mask(W.workload(1))
    assert m1.sum() == 22 and m1[0].tolist() == [1, 1, 0, 0, 0, 0, 0, 0]
    wl4 = W.workload(4)
    assert wl4.N == 115200 and wl4.N // wl4.chunks == 7200 and wl4.S == 1800


def test_spatial_locality_of_the_generated_inputs():
    # Generator sanity (not parity): with the positional term, a query partition's own
    # KV partition carries more importance than the farthest one.
    wl = W.small_variant(W.workload(1), grid=(1, 32, 32), H=2, D=64)
    t = W.make_qkv(wl)
    q, k, v = (W.to_f64(t[n]) for n in ("q", "k", "v"))
    off = W.part_offsets(wl.N, wl.P)
    op, lp, _ = O.partition_states(q, k, v, off, 1, all_fresh(wl.P), wl.scale)
    o, lse = O.merge_states(list(op), list(lp))
    w = O.importance(lp, lse, off, 1)
    for g in range(wl.P):
        far = 0 if g >= wl.P // 2 else wl.P - 1
        assert w[g, g] > w[g, far]


# --------------------------------------------------------------------------- group compose
def test_composed_cache_equals_per_partition_cache():
    # Dynamic group compose (DiTango, Methodology 2): composing cached states per group and
    # merging the composed ones gives the same result as merging the per-partition cache.
    q, k, v = rand_qkv(21, 1, 2, 70, 8)
    P, G = 6, 3
    off = W.part_offsets(70, P)
    ones = all_fresh(P, G)
    of, lf, _ = O.partition_states(q, k, v, off, G, ones, 0.35)
    rng = np.random.default_rng(22)
    kc, vc = k + 0.2 * rng.standard_normal(k.shape), v + 0.2 * rng.standard_normal(v.shape)
    oc, lc, _ = O.partition_states(q, kc, vc, off, G, ones, 0.35)
    fresh = np.array([[1, 0], [0, 1]], dtype=np.uint8)
    ref_o, ref_l, _ = O.merge_with_reuse(of, lf, oc, lc, off, G, fresh)
    co, cl = O.compose_states(oc, lc, G)
    assert co.shape[0] == 2
    o, l = O.merge_with_composed_cache(of, lf, co, cl, off, G, fresh)
    np.testing.assert_allclose(o, ref_o, atol=1e-12)
    np.testing.assert_allclose(l, ref_l, atol=1e-12)


def test_composed_state_is_attention_over_the_group():
    # a composed group state equals the state of one partition spanning the whole group
    q, k, v = rand_qkv(23, 1, 1, 40, 4)
    off = W.part_offsets(40, 4)                  # 10 keys each
    ones = all_fresh(4)
    op, lp, _ = O.partition_states(q, k, v, off, 1, ones, 0.5)
    co, cl = O.compose_states(op, lp, 2)
    wide, wl, _ = O.partition_states(q, k, v, np.array([0, 20, 40]), 1, all_fresh(2), 0.5)
    np.testing.assert_allclose(co, wide, atol=1e-12)
    np.testing.assert_allclose(cl, wl, atol=1e-12)


# --------------------------------------------------------------------------- online prediction
def test_state_drift_closed_forms():
    rng = np.random.default_rng(30)
    P, G, N, D = 4, 2, 20, 3
    off = W.part_offsets(N, P)                   # 5 rows per partition, 2 query groups
    ref = rng.standard_normal((P, 1, 2, N, D))
    sel = np.array([[1, 0], [1, 1]], dtype=np.uint8)
    d2, r2 = O.state_drift(ref, ref, off, G, sel)
    assert not d2.any()
    d2, r2 = O.state_drift(2 * ref, ref, off, G, sel)     # |2b - b|^2 = |b|^2
    np.testing.assert_allclose(d2, r2, rtol=1e-14)
    # brute force: query group 1 (rows 10..19), partition 1 (kv group 0, selected)
    expect = sum(float(ref[1, 0, h, i, c]) ** 2 for h in range(2) for i in range(10, 20) for c in range(D))
    assert abs(r2[1, 1] - expect) < 1e-10
    assert r2[0, 2] == 0 and r2[0, 3] == 0                # query group 0 x kv group 1 not selected


def test_predict_fresh_policy():
    w = np.array([[0.6, 0.3, 0.07, 0.03], [0.1, 0.1, 0.5, 0.3]])
    d2 = np.array([[4.0, 0.0, 0, 0], [0, 0, 1.0, 0.0]])
    r2 = np.array([[100.0, 0.0, 0, 0], [0, 0, 25.0, 75.0]])   # drift: 0.2 and 0.1
    m = O.predict_fresh(w, d2, r2, 2, eps=0.015)
    # qg 0: kv group 1 max w = 0.07 -> 0.014 < 0.015 -> reuse; qg 1: kv group 0 0.1*0.1=0.01 -> reuse
    np.testing.assert_array_equal(m, [[1, 0], [0, 1]])
    m = O.predict_fresh(w, d2, r2, 2, eps=0.01)
    np.testing.assert_array_equal(m, [[1, 1], [1, 1]])


# --------------------------------------------------------------------------- property-based


@settings(max_examples=60, deadline=None)
@given(P=st.integers(1, 9), R=st.integers(1, 6), seed=st.integers(0, 10_000),
       n_inf=st.integers(0, 3), split=st.integers(1, 8))
def test_merge_properties_hold_for_any_states(P, R, seed, n_inf, split):
    # any states, some of them empty (-inf): the merge equals the direct softmax-weighted
    # sum, any split into two groups merged separately and then together gives the same,
    # and the weights exp(LSE_p - LSE) of the non-empty states sum to one per row
    rng = np.random.default_rng(seed)
    lse = rng.normal(scale=4.0, size=(P, R))
    o = rng.standard_normal((P, R, 2))
    for p in rng.choice(P, size=min(n_inf, P - 1), replace=False):
        lse[p] = -np.inf
        o[p] = 0.0
    mo, ml = O.merge_states(list(o), list(lse))
    # direct definition, written out independently
    m = lse.max(axis=0)
    wts = np.exp(lse - m)
    ref_l = m + np.log(wts.sum(axis=0))
    ref_o = (wts[..., None] * o).sum(axis=0) / wts.sum(axis=0)[..., None]
    np.testing.assert_allclose(ml, ref_l, rtol=0, atol=1e-12)
    np.testing.assert_allclose(mo, ref_o, rtol=0, atol=1e-12)
    k = min(split, P)
    if 0 < k < P:
        a = O.merge_states(list(o[:k]), list(lse[:k]))
        b = O.merge_states(list(o[k:]), list(lse[k:]))
        go, gl = O.merge_states([a[0], b[0]], [a[1], b[1]])
        np.testing.assert_allclose(gl, ml, atol=1e-12)
        np.testing.assert_allclose(go, mo, atol=1e-12)
    np.testing.assert_allclose(np.exp(lse - ml).sum(axis=0), 1.0, atol=1e-12)
