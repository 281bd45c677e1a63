"""pa_merge_states_noalloc: the merge for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: processes whose free HBM is held by another allocator
(a framework's caching pool), or loops that must not stall on the device-wide
synchronisation that cudaMalloc / cudaFree of a growing workspace brings.  This entry point
takes no context and uses libpa's fixed file-scope scratch array instead.  Its results
must match pa_merge_states and the fp64 oracle, call after call (the scratch keeps the
previous call's contents, so two calls in a row are checked).

Kept in a file of its own, collected last.
"""
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


def _states(seed, P, B, H, N, D, dt):
    """Seeded states generated on the host; returns the device tensors and their exact
    fp64 values (after rounding to dt) for the oracle."""
    rng = np.random.default_rng(seed)
    lse = torch.from_numpy(rng.normal(3.0, 2.5, size=(P, B, H, N)).astype(np.float32))
    o = torch.from_numpy(rng.standard_normal((P, B, H, N, D)).astype(np.float32)).to(dt)
    return o.to(DEV), lse.to(DEV), o.double().numpy(), lse.double().numpy()


@pytest.mark.parametrize("dt,D,N,P,G,H", [(torch.bfloat16, 128, 2900, 32, 4, 2),
                                          (torch.float32, 64, 1000, 8, 1, 3)])
def test_noalloc_merge_matches_the_allocating_merge_twice(pa, dt, D, N, P, G, H):
    B = 1
    off = W.part_offsets(N, P)
    QG = -(-P // G)
    fresh = (np.random.default_rng(N).random((QG, QG)) < 0.4).astype(np.uint8)
    of, lf, of64, lf64 = _states(1, P, B, H, N, D, dt)
    oc, lc, oc64, lc64 = _states(2, P, B, H, N, D, dt)
    ro, rl, chosen = O.merge_with_reuse(of64, lf64, oc64, lc64, off, G, fresh)
    rw = O.importance(chosen, rl, off, G)
    ctx = pa.Context(0)
    o_ref = torch.empty(B, H, N, D, dtype=dt, device=DEV)
    l_ref = torch.empty(B, H, N, device=DEV)
    w_ref = torch.empty(QG, P, device=DEV)
    pa.pa_merge_states(ctx, off, G, fresh, of, lf, oc, lc, o_ref, l_ref, w_ref)
    ctx.sync_status()
    tol = TOL["bf16" if dt == torch.bfloat16 else "f32"]
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        l = torch.full_like(l_ref, float("nan"))
        w = torch.full_like(w_ref, float("nan"))
        pa.pa_merge_states_noalloc(off, G, fresh, of, lf, oc, lc, o, l, w)
        torch.cuda.synchronize()
        on, ln, wn = o.float().cpu().numpy(), l.cpu().numpy(), w.cpu().numpy()
        # against the allocating entry point
        assert maxerr(on, o_ref.float().cpu().numpy()) <= tol["o"], call
        assert maxerr(ln, l_ref.cpu().numpy()) <= tol["lse"], call
        assert maxerr(wn, w_ref.cpu().numpy()) <= tol["w"], call
        # against the fp64 oracle on the same states
        assert maxerr(on, ro) <= tol["o"], call
        assert maxerr(ln, rl) <= tol["lse"], call
        assert maxerr(wn, rw) <= tol["w"], call
    ctx.close()


def test_noalloc_merge_without_importance(pa):
    N, P, D, H = 700, 4, 128, 2
    off = W.part_offsets(N, P)
    of, lf, of64, lf64 = _states(3, P, 1, H, N, D, torch.bfloat16)
    ro, rl = O.merge_states(list(of64), list(lf64))
    ctx = pa.Context(0)
    o_ref = torch.empty(1, H, N, D, dtype=torch.bfloat16, device=DEV)
    l_ref = torch.empty(1, H, N, device=DEV)
    pa.pa_merge_states(ctx, off, 1, None, of, lf, None, None, o_ref, l_ref)
    o = torch.empty_like(o_ref)
    l = torch.empty_like(l_ref)
    pa.pa_merge_states_noalloc(off, 1, None, of, lf, None, None, o, l)
    torch.cuda.synchronize()
    assert maxerr(o.float().cpu().numpy(), o_ref.float().cpu().numpy()) <= TOL["bf16"]["o"]
    assert maxerr(l.cpu().numpy(), l_ref.cpu().numpy()) <= TOL["bf16"]["lse"]
    assert maxerr(o.float().cpu().numpy(), ro) <= TOL["bf16"]["o"]
    assert maxerr(l.cpu().numpy(), rl) <= TOL["bf16"]["lse"]
    ctx.close()


def test_noalloc_merge_rejects_a_scratch_request_beyond_its_limit(pa):
    # P = 128 one-token partitions, 65 heads: 65 * 128 row blocks * 128 partitions
    # = 1,064,960 importance partials > the fixed 1,048,576.
    N, P, D, H = 128, 128, 64, 65
    off = W.part_offsets(N, P)
    of = torch.zeros(P, 1, H, N, D, dtype=torch.bfloat16, device=DEV)
    lf = torch.zeros(P, 1, H, N, device=DEV)
    o = torch.empty(1, H, N, D, dtype=torch.bfloat16, device=DEV)
    l = torch.empty(1, H, N, device=DEV)
    w = torch.empty(P, P, device=DEV)
    with pytest.raises(pa.PAError, match="PA_EINVAL.*exceeds"):
        pa.pa_merge_states_noalloc(off, 1, None, of, lf, None, None, o, l, w)
    # the same request without importance needs no scratch and runs
    pa.pa_merge_states_noalloc(off, 1, None, of, lf, None, None, o, l)
    torch.cuda.synchronize()
