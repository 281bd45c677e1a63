"""GPU parity: every libpa entry point, through the C ABI, against the fp64 oracle on the
same seeded inputs, at oracle-sized shapes that span several tiles and ragged tails."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests.helpers import TOL, compare_states, maxerr, run_reuse_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    from sequence_partition_attn_b200 import build
    build.build()
    import sequence_partition_attn_b200 as m
    return m


@pytest.fixture(scope="module")
def ctx(pa):
    c = pa.Context(0)
    yield c
    c.close()


DEV = "cuda:0"


# --------------------------------------------------------------------------- relayout
@pytest.mark.parametrize("N,H,D,dt,chunks", [(1000, 3, 128, torch.bfloat16, 16),
                                               (777, 5, 64, torch.float32, 3),
                                               (64, 1, 8, torch.bfloat16, 1),
                                               (7200 * 2, 24, 128, torch.bfloat16, 16),
                                               (333, 7, 96, torch.bfloat16, 5),     # 12 pieces per row
                                               (129, 3, 24, torch.bfloat16, 2),     # 3 pieces per row
                                               (50, 2, 40, torch.float32, 3),       # 10 pieces per row
                                               (40, 3, 2048, torch.float32, 4)])    # 512 pieces per row
def test_relayout_bit_exact(pa, ctx, N, H, D, dt, chunks):
    g = torch.Generator().manual_seed(N + H)
    src = torch.randn(N, H, D, generator=g).to(dt)
    bits = torch.int16 if dt == torch.bfloat16 else torch.int32
    ref = O.relayout_seq2head(src.view(bits).numpy(), chunks)
    s = src.to(DEV)
    dst = torch.full((H, N, D), float("nan"), dtype=dt, device=DEV)
    for c in range(chunks):                       # chunk by chunk
        pa.pa_relayout_seq2head(ctx, s, dst, n_chunks=chunks, chunk=c)
    ctx.sync_status()
    assert np.array_equal(dst.cpu().view(bits).numpy(), ref)
    dst2 = torch.zeros_like(dst)
    pa.pa_relayout_seq2head(ctx, s, dst2, n_chunks=chunks, chunk=-1)   # all at once
    ctx.sync_status()
    assert np.array_equal(dst2.cpu().view(bits).numpy(), ref)


@pytest.mark.parametrize("n_tok,H,D,dst_tokens,tok0,dt", [(300, 3, 128, 1000, 417, torch.bfloat16),
                                                         (64, 2, 64, 64, 0, torch.float32),
                                                         (7, 5, 8, 20, 13, torch.bfloat16),
                                                         (3600, 12, 128, 115200, 57600, torch.bfloat16)])
def test_relayout_at_places_a_piece_bit_exactly(pa, ctx, n_tok, H, D, dst_tokens, tok0, dt):
    g = torch.Generator().manual_seed(n_tok + tok0)
    src = torch.randn(n_tok, H, D, generator=g).to(dt)
    bits = torch.int16 if dt == torch.bfloat16 else torch.int32
    before = torch.randn(H, dst_tokens, D, generator=g).to(dt)
    want = before.view(bits).numpy().copy()
    want[:, tok0:tok0 + n_tok] = O.relayout_seq2head(src.view(bits).numpy())
    dst = before.to(DEV)
    pa.pa_relayout_seq2head_at(ctx, src.to(DEV), dst, tok0)
    ctx.sync_status()
    assert np.array_equal(dst.cpu().view(bits).numpy(), want)       # other rows untouched
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_relayout_seq2head_at(ctx, src.to(DEV), dst, dst_tokens - n_tok + 1)


def test_relayout_rejects_rows_above_16_kib(pa, ctx):
    src = torch.zeros(4, 1, 8192, dtype=torch.float32, device=DEV)
    with pytest.raises(pa.PAError, match="PA_EUNSUPPORTED"):
        pa.pa_relayout_seq2head(ctx, src, src.view(1, 4, 8192))


def test_relayout_single_chunk_touches_only_its_rows(pa, ctx):
    N, H, D = 1000, 2, 64
    src = torch.randn(N, H, D).to(torch.bfloat16).to(DEV)
    dst = torch.zeros(H, N, D, dtype=torch.bfloat16, device=DEV)
    pa.pa_relayout_seq2head(ctx, src, dst, n_chunks=4, chunk=2)    # rows [500, 750)
    ctx.sync_status()
    d = dst.cpu().float().numpy()
    s = src.cpu().float().numpy()
    assert np.array_equal(d[:, 500:750], s[500:750].transpose(1, 0, 2))
    assert not d[:, :500].any() and not d[:, 750:].any()


# --------------------------------------------------------------------------- merge / importance
def _gen_states(seed, P, B, H, N, D, dt, empty=()):
    rng = np.random.default_rng(seed)
    lse = rng.normal(loc=3.0, scale=2.5, size=(P, B, H, N)).astype(np.float32)
    o = rng.standard_normal((P, B, H, N, D)).astype(np.float32)
    for p in empty:
        lse[p] = -np.inf
        o[p] = 0.0
    o_t = torch.from_numpy(o).to(dt)
    return o_t, torch.from_numpy(lse)


@pytest.mark.parametrize("dt,D,N,P,G,B,H", [
    (torch.bfloat16, 128, 1000, 8, 1, 1, 3),
    (torch.bfloat16, 128, 2900, 32, 4, 1, 2),
    (torch.bfloat16, 64, 517, 5, 2, 2, 2),
    (torch.float32, 64, 1024, 4, 1, 1, 2),
    (torch.float32, 128, 300, 64, 8, 1, 1),
    (torch.bfloat16, 128, 640, 128, 16, 1, 1),
])
def test_merge_with_reuse_and_fused_importance(pa, ctx, dt, D, N, P, G, B, H):
    off = W.part_offsets(N, P)
    QG = -(-P // G)
    rng = np.random.default_rng(N + P)
    fresh = (rng.random((QG, QG)) < 0.4).astype(np.uint8)
    empty = [p for p in range(P) if off[p + 1] == off[p]]
    of, lf = _gen_states(1, P, B, H, N, D, dt, empty)
    oc, lc = _gen_states(2, P, B, H, N, D, dt, empty)
    o = torch.empty(B, H, N, D, dtype=dt, device=DEV)
    lse = torch.empty(B, H, N, device=DEV)
    w = torch.empty(QG, P, device=DEV)
    pa.pa_merge_states(ctx, off, G, fresh, of.to(DEV), lf.to(DEV), oc.to(DEV), lc.to(DEV), o, lse, w)
    ctx.sync_status()
    f64 = lambda x: x.double().numpy()   # noqa: E731
    ro, rl, ch = O.merge_with_reuse(f64(of), f64(lf), f64(oc), f64(lc), off, G, fresh)
    rw = O.importance(ch, rl, off, G)
    tol = TOL["bf16" if dt == torch.bfloat16 else "f32"]
    # stored states are exact inputs; the merge arithmetic is fp32 and O is rounded to dtype
    o_tol = tol["o"] if dt == torch.bfloat16 else 1e-5
    assert maxerr(o.float().cpu().numpy(), ro) <= o_tol
    assert maxerr(lse.cpu().numpy(), rl) <= 1e-5 + 1e-6 * np.abs(rl).max()
    assert maxerr(w.cpu().numpy(), rw) <= tol["w"]


def test_merge_all_fresh_without_cache(pa, ctx):
    N, P, D = 700, 4, 128
    off = W.part_offsets(N, P)
    of, lf = _gen_states(3, P, 1, 2, N, D, torch.bfloat16)
    o = torch.empty(1, 2, N, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(1, 2, N, device=DEV)
    pa.pa_merge_states(ctx, off, 1, None, of.to(DEV), lf.to(DEV), None, None, o, lse)
    ctx.sync_status()
    ro, rl = O.merge_states(list(of.double().numpy()), list(lf.double().numpy()))
    assert maxerr(o.float().cpu().numpy(), ro) <= TOL["bf16"]["o"]
    assert maxerr(lse.cpu().numpy(), rl) <= 1e-5


@pytest.mark.parametrize("N,P,G,B,H", [(1000, 8, 1, 1, 3), (2900, 32, 4, 2, 2), (16, 5, 2, 1, 1)])
def test_importance_standalone(pa, ctx, N, P, G, B, H):
    off = W.part_offsets(N, P)
    empty = [p for p in range(P) if off[p + 1] == off[p]]
    _, lp = _gen_states(4, P, B, H, N, 8, torch.float32, empty)
    _, l_all = O.merge_states([np.zeros(lp.shape[1:] + (1,))] * P, list(lp.double().numpy()))
    lse = torch.from_numpy(l_all.astype(np.float32))
    w = torch.empty(-(-P // G), P, device=DEV)
    pa.pa_importance(ctx, off, G, lp.to(DEV), lse.to(DEV), w)
    ctx.sync_status()
    rw = O.importance(lp.double().numpy(), lse.double().numpy(), off, G)
    assert maxerr(w.cpu().numpy(), rw) <= 1e-5
    np.testing.assert_allclose(w.cpu().numpy().sum(axis=1)[np.diff(O.group_bounds(off, G)) > 0], 1.0,
                               atol=1e-4)


# --------------------------------------------------------------------------- partition attention
def _check_case(pa, ctx, wl, fresh=None):
    gpu, ora, sel, off, fresh = run_reuse_case(pa, ctx, wl, fresh)
    tol = TOL[wl.dtype]
    errs, untouched = compare_states(gpu, ora, sel, tol)
    werr = maxerr(gpu["w"], ora["w"])
    assert untouched, "unselected pairs were written"
    assert errs["of"] <= tol["o"] and errs["oc"] <= tol["o"] and errs["o"] <= tol["o"], errs
    assert errs["lf"] <= tol["lse"] and errs["lc"] <= tol["lse"] and errs["lse"] <= tol["lse"], errs
    assert werr <= tol["w"], werr
    return errs, werr


def test_config0_fp32_full_recompute(pa, ctx):
    _check_case(pa, ctx, W.workload(0))


SMALL_BF16 = [
    dict(grid=(1, 20, 23), H=2, P=4, G=1),             # N=460: ragged partitions and tiles
    dict(grid=(1, 25, 40), H=2, P=7, G=2, mask="all"),  # N=1000, S=143
    dict(grid=(1, 10, 30), H=1, P=1, G=1, mask="all"),  # single partition
    dict(grid=(1, 10, 10), H=2, P=2, G=1),             # N=100 < one tile
    dict(grid=(2, 16, 16), H=2, P=4, G=1, D=64),       # D = 64
    dict(grid=(1, 16, 32), H=2, P=4, G=1, B=2),        # batch 2
    dict(grid=(1, 4, 4), H=1, P=5, G=1, mask="all"),   # N=16, S=4: partition 4 is empty
]


@pytest.mark.parametrize("kw", SMALL_BF16)
def test_bf16_small_cases(pa, ctx, kw):
    kw = dict(kw)
    wl = W.small_variant(W.workload(1), **kw)
    _check_case(pa, ctx, wl)


def test_bf16_maximum_partition_count(pa, ctx):
    # P = 128 (the largest table the ABI takes), G = 16, 8 groups of 16 partitions of ~16
    # keys: every partition is shorter than a key tile; a random group mask
    wl = W.small_variant(W.workload(1), grid=(1, 40, 50), H=1, P=128, G=16)
    fresh = (np.random.default_rng(17).random((wl.QG, wl.KG)) < 0.5).astype(np.uint8)
    np.fill_diagonal(fresh, 1)
    _check_case(pa, ctx, wl, fresh)


def _units(wl, fresh):
    """Work units of the bf16 launch: 256-row blocks of query groups with a fresh pair."""
    rb = W.group_row_bounds(W.part_offsets(wl.N, wl.P), wl.G)
    return wl.B * wl.H * sum(-(-(int(rb[g + 1]) - int(rb[g])) // 256)
                             for g in range(wl.QG) if fresh[g].any() and rb[g + 1] > rb[g])


def test_bf16_many_units_ragged(pa, ctx):
    # More work units (CTAs) than SMs, 200-key partitions (a shifted last tile each) and a
    # random mask.
    wl = W.small_variant(W.workload(1), grid=(1, 30, 40), H=40, P=6, G=1)
    fresh = (np.random.default_rng(5).random((wl.QG, wl.KG)) < 0.5).astype(np.uint8)
    np.fill_diagonal(fresh, 1)
    assert _units(wl, fresh) > 148
    _check_case(pa, ctx, wl, fresh)


def test_bf16_units_of_short_partitions(pa, ctx):
    # More units than SMs, each of partitions shorter than a tile (4 keys), an empty
    # partition, a query group whose only fresh partition is the empty one (a unit without
    # KV tiles: it only writes LSE = -inf, O = 0) and an idle query group; D = 64.
    wl = W.small_variant(W.workload(1), grid=(1, 4, 4), H=64, P=5, G=1, D=64)
    fresh = (np.random.default_rng(9).random((wl.QG, wl.KG)) < 0.6).astype(np.uint8)
    fresh[0] = 1
    fresh[3] = [0, 0, 0, 0, 1]
    fresh[1] = 0
    assert _units(wl, fresh) > 148
    _check_case(pa, ctx, wl, fresh)


def test_fp32_small_ragged_case(pa, ctx):
    wl = W.small_variant(W.workload(0), grid=(1, 13, 23), H=2, P=3, G=1, cache_sigma=0.05,
                         mask="neighbours", D=128)
    _check_case(pa, ctx, wl)


def test_config1_image_dit_with_reuse(pa, ctx):
    errs, werr = _check_case(pa, ctx, W.workload(1))
    print("config 1", errs, werr)


def test_720p_recipe_reduced_grid(pa, ctx):
    # the 720p workload's recipe (P=32, G=4, nearest-25% groups, sigma 0.03) on a 3-frame grid
    wl = W.small_variant(W.workload(2), grid=(3, 45, 80), H=2)
    assert wl.N == 10800 and wl.N % wl.P != 0
    errs, werr = _check_case(pa, ctx, wl)
    print("720p recipe, reduced", errs, werr)


# --------------------------------------------------------------------------- validation
def test_validation_errors(pa, ctx):
    q = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device=DEV)
    o = torch.zeros(2, 1, 1, 256, 128, dtype=torch.bfloat16, device=DEV)
    l = torch.zeros(2, 1, 1, 256, device=DEV)
    off = [0, 128, 256]
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_partition_attn(ctx, q, q, q, [0, 100, 200], 1, None, o, l)     # part_off[P] != N
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_partition_attn(ctx, q, q, q, [0, 200, 100, 256], 1, None, o, l)  # decreasing
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_partition_attn(ctx, q, q, q, off, 3, None, o, l)                 # G > P
    with pytest.raises(pa.PAError, match="PA_EUNSUPPORTED"):
        q96 = torch.zeros(1, 1, 256, 96, dtype=torch.bfloat16, device=DEV)
        pa.pa_partition_attn(ctx, q96, q96, q96, off, 1, None, o, l)
    with pytest.raises(pa.PAError, match="PA_EUNSUPPORTED"):
        qh = torch.zeros(1, 1, 256, 128, dtype=torch.float16, device=DEV)
        pa.pa_partition_attn(ctx, qh, qh, qh, off, 1, None, o, l)
    flat = torch.zeros(256 * 128 + 8, dtype=torch.bfloat16, device=DEV)
    mis = flat[1:1 + 256 * 128].view(1, 1, 256, 128)                        # 2-byte offset
    with pytest.raises(pa.PAError, match="PA_EALIGN"):
        pa.pa_partition_attn(ctx, mis, q, q, off, 1, None, o, l)
    ob = torch.zeros(1, 1, 256, 128, dtype=torch.bfloat16, device=DEV)
    lb = torch.zeros(1, 1, 256, device=DEV)
    with pytest.raises(pa.PAError, match="PA_EINVAL"):                      # reuse without a cache
        pa.pa_merge_states(ctx, off, 1, np.array([[1, 0], [0, 1]]), o, l, None, None, ob, lb)
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_relayout_seq2head(ctx, q[0, 0].view(256, 1, 128), q[0, 0].view(1, 256, 128), 4, 4)
    ctx.sync_status()


def test_empty_sequence_is_a_no_op(pa, ctx):
    q = torch.zeros(1, 1, 0, 128, dtype=torch.bfloat16, device=DEV)
    o = torch.zeros(1, 1, 1, 0, 128, dtype=torch.bfloat16, device=DEV)
    l = torch.zeros(1, 1, 1, 0, device=DEV)
    pa.pa_partition_attn(ctx, q, q, q, [0, 0], 1, None, o, l)
    ctx.sync_status()


@pytest.mark.parametrize("grid,P,p_sel", [((1, 25, 40), 4, 1),      # 250 keys: shifted last tile
                                          ((1, 32, 64), 128, 5),    # 16 keys: shorter than a tile
                                          ((1, 20, 23), 8, 7)])     # 54 keys, last partition
def test_partition_state_reads_no_other_partition(pa, ctx, grid, P, p_sel):
    # A partition's state must not depend on K/V rows of any other partition, even
    # non-finite ones: a partial last tile of a partition of >= 128 keys is loaded ending at
    # the partition end, and for a partition shorter than a tile the V rows past its end
    # are zeroed in shared memory before the PV product reads them.
    wl = W.small_variant(W.workload(1), grid=grid, H=2, P=P, G=1, mask="all")
    t = W.make_qkv(wl)
    off = W.part_offsets(wl.N, wl.P)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    fresh = np.zeros((P, P), dtype=np.uint8)
    fresh[:, p_sel] = 1                                          # every query group x one partition
    o1 = torch.zeros(P, 1, 2, wl.N, 128, dtype=torch.bfloat16, device=DEV)
    l1 = torch.zeros(P, 1, 2, wl.N, device=DEV)
    pa.pa_partition_attn(ctx, q, k, v, off, 1, fresh, o1, l1)
    k2, v2 = k.clone(), v.clone()
    for p in range(P):
        if p != p_sel:
            k2[:, :, off[p]:off[p + 1]] = float("nan")
            v2[:, :, off[p]:off[p + 1]] = float("inf")
    o2 = torch.zeros_like(o1)
    l2 = torch.zeros_like(l1)
    pa.pa_partition_attn(ctx, q, k2, v2, off, 1, fresh, o2, l2)
    ctx.sync_status()
    assert torch.isfinite(o2[p_sel].float()).all() and torch.isfinite(l2[p_sel]).all()
    assert torch.equal(o1[p_sel].view(torch.int16), o2[p_sel].view(torch.int16))
    assert torch.equal(l1[p_sel], l2[p_sel])
    # and the clean run matches the oracle on that partition
    qf, kf, vf = (W.to_f64(t[n]) for n in ("q", "k", "v"))
    ro, rl, _ = O.partition_states(qf, kf, vf, off, 1, fresh, wl.scale)
    assert maxerr(o1[p_sel].float().cpu().numpy(), ro[p_sel]) <= TOL["bf16"]["o"]
    assert maxerr(l1[p_sel].cpu().numpy(), rl[p_sel]) <= TOL["bf16"]["lse"]


# --------------------------------------------------------------------------- group compose
@pytest.mark.parametrize("dt,D,N,P,factor", [(torch.bfloat16, 128, 1500, 32, 4),
                                              (torch.float32, 64, 700, 7, 3),
                                              (torch.bfloat16, 64, 300, 5, 5)])
def test_compose_states(pa, ctx, dt, D, N, P, factor):
    off = W.part_offsets(N, P)
    empty = [p for p in range(P) if off[p + 1] == off[p]]
    o, l = _gen_states(7, P, 1, 2, N, D, dt, empty)
    C = -(-P // factor)
    og = torch.empty(C, 1, 2, N, D, dtype=dt, device=DEV)
    lg = torch.empty(C, 1, 2, N, device=DEV)
    pa.pa_compose_states(ctx, o.to(DEV), l.to(DEV), factor, og, lg)
    ctx.sync_status()
    ro, rl = O.compose_states(o.double().numpy(), l.double().numpy(), factor)
    tol = TOL["bf16" if dt == torch.bfloat16 else "f32"]
    assert maxerr(og.float().cpu().numpy(), ro) <= (tol["o"] if dt == torch.bfloat16 else 1e-5)
    assert maxerr(lg.cpu().numpy(), rl) <= 1e-5 + 1e-6 * np.abs(rl[np.isfinite(rl)]).max()


def test_compose_with_factor_one_is_the_identity(pa, ctx):
    # one partition per group: LSE = LSE_p + ln 1 and weight exp(0) = 1, so the composed
    # states are the partition states bit for bit (empty partition included)
    N, P = 333, 7
    off = W.part_offsets(N, P)
    o, l = _gen_states(9, P, 2, 2, N, 128, torch.bfloat16, empty=[3])
    og = torch.empty_like(o, device=DEV)
    lg = torch.empty_like(l, device=DEV)
    pa.pa_compose_states(ctx, o.to(DEV), l.to(DEV), 1, og, lg)
    ctx.sync_status()
    assert torch.equal(og.cpu().view(torch.int16), o.view(torch.int16))
    assert torch.equal(lg.cpu(), l)


def test_merge_with_composed_cache_against_oracle(pa, ctx):
    # seeded states (generated on the host) for both sides
    N, P, G, D, H = 2900, 32, 4, 128, 2
    off = W.part_offsets(N, P)
    KG = P // G
    fresh = (np.random.default_rng(3).random((KG, KG)) < 0.3).astype(np.uint8)
    of, lf = _gen_states(11, P, 1, H, N, D, torch.bfloat16)
    oc, lc = _gen_states(12, P, 1, H, N, D, torch.bfloat16)
    ocg = torch.empty(KG, 1, H, N, D, dtype=torch.bfloat16, device=DEV)
    lcg = torch.empty(KG, 1, H, N, device=DEV)
    pa.pa_compose_states(ctx, oc.to(DEV), lc.to(DEV), G, ocg, lcg)
    o = torch.empty(1, H, N, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(1, H, N, device=DEV)
    pa.pa_merge_states(ctx, off, G, fresh, of.to(DEV), lf.to(DEV), ocg, lcg, o, lse, cached_per_group=True)
    ctx.sync_status()
    f64 = lambda x: x.double().numpy()   # noqa: E731
    co, cl = O.compose_states(f64(oc), f64(lc), G)
    ro, rl = O.merge_with_composed_cache(f64(of), f64(lf), co, cl, off, G, fresh)
    # the composed cache is rounded to bf16 once more on the GPU side
    assert maxerr(o.float().cpu().numpy(), ro) <= TOL["bf16"]["o"]
    assert maxerr(lse.cpu().numpy(), rl) <= 1e-5 + 1e-6 * np.abs(rl).max()


def test_merge_with_composed_cache(pa, ctx):
    # 720p recipe on a reduced grid, states from the attention kernel: the composed-cache
    # merge agrees with the per-partition merge (associativity) and with the oracle.
    wl = W.small_variant(W.workload(2), grid=(3, 45, 80), H=2)
    t = W.make_qkv(wl)
    kc, vc = W.make_cached_kv(wl, t["k"], t["v"])
    off = W.part_offsets(wl.N, wl.P)
    fresh = W.reuse_mask(wl)
    q, k, v = (t[n].to(DEV) for n in ("q", "k", "v"))
    P, B, H, N, D = wl.P, wl.B, wl.H, wl.N, wl.D
    of = torch.zeros(P, B, H, N, D, dtype=torch.bfloat16, device=DEV)
    lf = torch.zeros(P, B, H, N, device=DEV)
    oc, lc = torch.zeros_like(of), torch.zeros_like(lf)
    pa.pa_partition_attn(ctx, q, k, v, off, wl.G, fresh, of, lf)
    pa.pa_partition_attn(ctx, q, kc.to(DEV), vc.to(DEV), off, wl.G, None, oc, lc)
    ocg = torch.empty(wl.KG, B, H, N, D, dtype=torch.bfloat16, device=DEV)
    lcg = torch.empty(wl.KG, B, H, N, device=DEV)
    pa.pa_compose_states(ctx, oc, lc, wl.G, ocg, lcg)
    o1 = torch.empty(B, H, N, D, dtype=torch.bfloat16, device=DEV)
    l1 = torch.empty(B, H, N, device=DEV)
    pa.pa_merge_states(ctx, off, wl.G, fresh, of, lf, ocg, lcg, o1, l1, cached_per_group=True)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    pa.pa_merge_states(ctx, off, wl.G, fresh, of, lf, oc, lc, o2, l2)
    ctx.sync_status()
    assert maxerr(o1.float().cpu().numpy(), o2.float().cpu().numpy()) <= TOL["bf16"]["o"]
    assert maxerr(l1.cpu().numpy(), l2.cpu().numpy()) <= 1e-5
    # and against the oracle from Q, K, V on sampled rows (every group boundary included):
    # fresh and cached states, composition of the cache per KV group, merge
    gb = W.group_row_bounds(off, wl.G)
    rng = np.random.default_rng(21)
    rows = np.unique(np.concatenate([rng.choice(N, 160, replace=False), gb[1:-1], gb[1:-1] - 1,
                                     np.arange(N - 8, N)]))
    ones = np.ones_like(fresh)
    qf, kf, vf = (W.to_f64(t[n]) for n in ("q", "k", "v"))
    rof, rlf, _ = O.partition_states(qf, kf, vf, off, wl.G, fresh, wl.scale, rows=rows)
    roc, rlc, _ = O.partition_states(qf, W.to_f64(kc), W.to_f64(vc), off, wl.G, ones, wl.scale, rows=rows)
    rco, rcl = O.compose_states(roc, rlc, wl.G)
    ro, rl = O.merge_with_composed_cache(rof, rlf, rco, rcl, off, wl.G, fresh, rows=rows)
    ri = torch.as_tensor(rows, device=DEV)
    assert maxerr(o1.index_select(2, ri).float().cpu().numpy(), ro) <= TOL["bf16"]["o"]
    assert maxerr(l1.index_select(2, ri).cpu().numpy(), rl) <= TOL["bf16"]["lse"]
    w = torch.empty(wl.QG, P, device=DEV)
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_merge_states(ctx, off, wl.G, fresh, of, lf, ocg, lcg, o1, l1, w, cached_per_group=True)


# --------------------------------------------------------------------------- state drift
@pytest.mark.parametrize("dt,D,N,P,G,B,H,sel_kind", [
    (torch.bfloat16, 128, 2900, 32, 4, 1, 2, "random"),
    (torch.float32, 64, 517, 5, 2, 2, 2, "all"),
    (torch.bfloat16, 64, 16, 5, 1, 1, 3, "own"),        # an empty partition, 4-row groups
    (torch.bfloat16, 128, 4096, 8, 1, 1, 4, "own"),     # trajectory shape, fewer heads
])
def test_state_drift_against_oracle(pa, ctx, dt, D, N, P, G, B, H, sel_kind):
    off = W.part_offsets(N, P)
    QG = -(-P // G)
    empty = [p for p in range(P) if off[p + 1] == off[p]]
    o_new, _ = _gen_states(21, P, B, H, N, D, dt, empty)
    o_ref, _ = _gen_states(22, P, B, H, N, D, dt, empty)
    if sel_kind == "random":
        sel = (np.random.default_rng(5).random((QG, QG)) < 0.4).astype(np.uint8)
        np.fill_diagonal(sel, 1)
    elif sel_kind == "own":
        sel = np.eye(QG, dtype=np.uint8)
    else:
        sel = np.ones((QG, QG), dtype=np.uint8)
    o_new_d = o_new.to(DEV)
    # states of unselected pairs may hold anything: poison every row outside the selection
    gb = W.group_row_bounds(off, G)
    for qg in range(QG):
        for p in range(P):
            if not sel[qg, p // G]:
                o_new_d[p, :, :, gb[qg]:gb[qg + 1]] = float("nan")
    d2 = torch.full((QG, P), -1.0, device=DEV)
    r2 = torch.full((QG, P), -1.0, device=DEV)
    pa.pa_state_drift(ctx, off, G, None if sel_kind == "all" else sel, o_new_d, o_ref.to(DEV), d2, r2)
    ctx.sync_status()
    rd, rr = O.state_drift(o_new.double().numpy(), o_ref.double().numpy(), off, G, sel)
    gd, gr = d2.cpu().numpy().astype(np.float64), r2.cpu().numpy().astype(np.float64)
    assert np.isfinite(gd).all() and np.isfinite(gr).all()
    assert np.abs(gd - rd).max() <= 1e-5 * max(rd.max(), 1.0)
    assert np.abs(gr - rr).max() <= 1e-5 * max(rr.max(), 1.0)
    assert (gd[rd == 0] == 0).all() and (gr[rr == 0] == 0).all()


def test_state_drift_empty_sequence_and_errors(pa, ctx):
    P, G = 4, 2
    off = np.zeros(P + 1, dtype=np.int32)
    o = torch.empty(P, 1, 1, 0, 64, dtype=torch.bfloat16, device=DEV)
    d2 = torch.full((2, P), 7.0, device=DEV)
    r2 = torch.full((2, P), 7.0, device=DEV)
    pa.pa_state_drift(ctx, off, G, None, o, o, d2, r2)
    ctx.sync_status()
    assert (d2.cpu() == 0).all() and (r2.cpu() == 0).all()
    o = torch.zeros(P, 1, 1, 64, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(pa.PAError, match="PA_EUNSUPPORTED"):
        pa.pa_state_drift(ctx, W.part_offsets(64, P), G, None, o, o, d2, r2)
    o = torch.zeros(P, 1, 1, 64, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_state_drift(ctx, W.part_offsets(63, P), G, None, o, o, d2, r2)


# --------------------------------------------------------------------------- streamed steps
def test_streamed_steps_match_serial_steps(pa, ctx):
    # three steps fed from host memory with overlapped copies give exactly the outputs of
    # the same steps run one after another
    from sequence_partition_attn_b200.step import AttentionStep, StreamedSteps
    wl = W.small_variant(W.workload(2), grid=(3, 45, 80), H=2)
    t = W.make_qkv(wl)
    kc, vc = W.make_cached_kv(wl, t["k"], t["v"])
    off = W.part_offsets(wl.N, wl.P)
    step = AttentionStep(ctx, wl.B, wl.H, wl.N, wl.D, off, wl.G, W.reuse_mask(wl), device=DEV)
    step.q.copy_(t["q"].to(DEV))
    step.fill_cache(kc.to(DEV), vc.to(DEV))
    inputs = []
    k, v = t["k"], t["v"]
    for s in range(3):
        if s:
            k, v = W.drift_kv(wl, k, v, s)
        inputs.append(tuple(x.pin_memory() for x in (t["q"], k, v)))
    outs = [(torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory(),
             torch.empty(step.lse.shape).pin_memory(), torch.empty(step.w.shape).pin_memory())
            for _ in range(3)]
    streamed = StreamedSteps(step)
    done = streamed.run(inputs, outs)
    done.synchronize()
    ctx.sync_status()
    for s in range(3):
        for d, h in zip((step.q, step.k, step.v), inputs[s]):
            d.copy_(h.to(DEV))
        step.run()
        ctx.sync_status()
        assert torch.equal(outs[s][0].view(torch.int16), step.o.cpu().view(torch.int16)), s
        assert torch.equal(outs[s][1], step.lse.cpu()) and torch.equal(outs[s][2], step.w.cpu()), s


# --------------------------------------------------------------------------- bounded waits
def test_bounded_wait_gives_up_reports_and_recovers(pa, ctx):
    # a wait on a barrier nothing completes gives up after 50 ms, the status word says
    # PA_ETIMEOUT once, and the context keeps working afterwards
    import time
    t0 = time.time()
    pa.pa_selftest_wait(ctx, 0.05)
    with pytest.raises(pa.PAError, match="PA_ETIMEOUT"):
        ctx.sync_status()
    assert time.time() - t0 < 10.0
    ctx.sync_status()                     # read and cleared
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        pa.pa_selftest_wait(ctx, 3.0)     # limits above 2 s are refused
    wl = W.small_variant(W.workload(1), grid=(1, 20, 23), H=1, P=4, mask="all")
    _check_case(pa, ctx, wl)


def test_debug_mode_reports_at_the_call(pa, monkeypatch):
    # PA_DEBUG at context creation: every call synchronises and returns the status itself
    monkeypatch.setenv("PA_DEBUG", "1")
    c = pa.Context(0)
    try:
        with pytest.raises(pa.PAError, match="PA_ETIMEOUT"):
            pa.pa_selftest_wait(c, 0.02)
        src = torch.randn(64, 2, 64, device=DEV).to(torch.bfloat16)
        dst = torch.empty(2, 64, 64, dtype=torch.bfloat16, device=DEV)
        pa.pa_relayout_seq2head(c, src, dst)             # an ordinary call passes through
        assert torch.equal(dst.cpu(), src.cpu().transpose(0, 1))
    finally:
        c.close()


def test_host_deadline_leaves_the_stream_running_and_the_context_usable(pa, ctx):
    # pa_wait_status gives up on the host after its deadline while a kernel still waits
    # (its own device-side limit is longer); nothing is cancelled: a later wait sees the
    # kernel finish and the device-side give-up it recorded, and the context keeps working
    import time
    pa.pa_selftest_wait(ctx, 1.0)
    t0 = time.time()
    with pytest.raises(pa.PAError, match="PA_ETIMEOUT.*host deadline"):
        ctx.sync_status(timeout=0.05)
    assert time.time() - t0 < 0.9
    with pytest.raises(pa.PAError, match="PA_ETIMEOUT.*device-side wait"):
        ctx.sync_status(timeout=30.0)
    ctx.sync_status(timeout=1.0)          # cleared; an idle stream passes at once
    with pytest.raises(pa.PAError, match="PA_EINVAL"):
        ctx.sync_status(timeout=-1.0)
    wl = W.small_variant(W.workload(1), grid=(1, 20, 23), H=1, P=4, mask="all")
    _check_case(pa, ctx, wl)


def test_injected_allocation_failure_is_reported_and_recoverable(pa, monkeypatch):
    # host-side injection (PA_INJECT_ENOMEM): the allocation fails as under memory
    # pressure, the call returns PA_ENOMEM having launched nothing, and the context works
    # again once memory is available
    monkeypatch.setenv("PA_INJECT_ENOMEM", "init")
    with pytest.raises(pa.PAError, match="PA_ENOMEM"):
        pa.Context(0)
    monkeypatch.setenv("PA_INJECT_ENOMEM", "workspace")
    c = pa.Context(0)
    try:
        N, P, G, D, H = 1000, 8, 2, 128, 2
        off = W.part_offsets(N, P)
        fresh = np.ones((4, 4), dtype=np.uint8)
        of, lf = _gen_states(31, P, 1, H, N, D, torch.bfloat16)
        of, lf = of.to(DEV), lf.to(DEV)
        o = torch.empty(1, H, N, D, dtype=torch.bfloat16, device=DEV)
        lse = torch.full((1, H, N), float("nan"), device=DEV)
        w = torch.full((4, P), float("nan"), device=DEV)
        with pytest.raises(pa.PAError, match="PA_ENOMEM"):
            pa.pa_merge_states(c, off, G, fresh, of, lf, None, None, o, lse, w)
        with pytest.raises(pa.PAError, match="PA_ENOMEM"):
            pa.pa_importance(c, off, G, lf, lse, w)
        c.sync_status()
        assert torch.isnan(lse).all() and torch.isnan(w).all()       # nothing launched
        pa.pa_merge_states(c, off, G, fresh, of, lf, None, None, o, lse)   # no workspace needed
        monkeypatch.delenv("PA_INJECT_ENOMEM")
        pa.pa_merge_states(c, off, G, fresh, of, lf, None, None, o, lse, w)
        c.sync_status()
        ro, rl = O.merge_states(list(of.double().cpu().numpy()), list(lf.double().cpu().numpy()))
        rw = O.importance(lf.double().cpu().numpy(), rl, off, G)
        assert maxerr(o.float().cpu().numpy(), ro) <= TOL["bf16"]["o"]
        assert maxerr(lse.cpu().numpy(), rl) <= TOL["bf16"]["lse"]
        assert maxerr(w.cpu().numpy(), rw) <= TOL["bf16"]["w"]
    finally:
        c.close()
