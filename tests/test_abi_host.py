"""CPU tests of the C ABI library and the host-side logic (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import sequence_partition_attn_b200 as pa
from sequence_partition_attn_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(pa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_documented_entry_points():
    assert set(header_functions()) == set(pa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {pa.lib_path()}").read()
    for name in header_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_library_is_built_for_sm100a_only(lib):
    flags = " ".join(pa_build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1


def test_version_and_init_without_device(lib):
    assert lib.pa_version().decode().startswith("libpa")
    ctx = ctypes.c_void_p()
    rc = lib.pa_init(0, ctypes.byref(ctx))
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if not has_gpu:
        assert rc in (-1, -3, -5)           # no device: an error code, never a crash
        assert not ctx.value
        assert lib.pa_last_error(None)
    else:
        lib.pa_destroy(ctx)


def test_null_context_is_rejected(lib):
    assert lib.pa_partition_attn(None, None, None) == -1
    assert lib.pa_merge_states(None, None, None) == -1
    assert lib.pa_importance(None, 1, 1, 1, 1, 1, None, None, None, None, None) == -1
    assert lib.pa_relayout_seq2head(None, None, None, 1, 1, 8, 2, 1, -1, None) == -1
    assert lib.pa_compose_states(None, 1, 1, 1, 1, 64, 1, 1, None, None, None, None, None) == -1
    assert lib.pa_state_drift(None, 1, 1, 1, 1, 64, 1, 1, None, None, None, None, None, None, None) == -1
    assert lib.pa_selftest_wait(None, 0.01, None) == -1
    assert lib.pa_sync_status(None, None) == -1
    assert b"ctx" in lib.pa_last_error(None)
    lib.pa_destroy(None)                   # no-op


@pytest.mark.parametrize("seed", range(20))
def test_host_reuse_selection_matches_the_oracle(seed):
    rng = np.random.default_rng(seed)
    QG, P = rng.integers(1, 9), rng.integers(1, 33)
    G = int(rng.integers(1, P + 1))
    QG = -(-P // G)
    w = rng.dirichlet(np.ones(P), size=QG) * rng.uniform(0.2, 1.5)
    w[rng.random(w.shape) < 0.2] = 0.05                 # exact threshold hits
    np.testing.assert_array_equal(pa.select_fresh(w, G, 0.05), O.select_fresh(w, G, 0.05))


@pytest.mark.parametrize("seed", range(20))
def test_host_error_prediction_matches_the_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    P = int(rng.integers(1, 33))
    G = int(rng.integers(1, P + 1))
    QG = -(-P // G)
    w = rng.dirichlet(np.ones(P), size=QG)
    d2 = rng.uniform(0, 0.01, size=(QG, P)) * (rng.random((QG, P)) < 0.8)
    r2 = rng.uniform(0.5, 2.0, size=(QG, P))
    r2[rng.random(QG) < 0.2] = 0.0                      # groups with nothing measured
    eps = float(np.quantile(w, 0.5)) * 0.05
    np.testing.assert_array_equal(pa.predict_fresh(w, d2, r2, G, eps),
                                  O.predict_fresh(w, d2, r2, G, eps))


def test_host_prediction_extremes():
    rng = np.random.default_rng(7)
    P, G = 12, 3
    QG = P // G
    w = rng.dirichlet(np.ones(P), size=QG)
    d2 = rng.uniform(0.001, 0.01, size=(QG, P))
    r2 = rng.uniform(0.5, 2.0, size=(QG, P))
    # a zero bound recomputes everything; an unreachable one only the own groups
    assert pa.predict_fresh(w, d2, r2, G, 0.0).all()
    np.testing.assert_array_equal(pa.predict_fresh(w, d2, r2, G, np.inf), np.eye(QG, dtype=np.uint8))
    # no drift measured (all reference norms zero): only the own groups
    np.testing.assert_array_equal(pa.predict_fresh(w, d2, np.zeros_like(r2), G, 1e-9),
                                  np.eye(QG, dtype=np.uint8))
    # a threshold of zero selects every pair, an unreachable one none
    assert pa.select_fresh(w, G, 0.0).all()
    assert not pa.select_fresh(w, G, 2.0).any()


def test_binding_rejects_unsupported_dtypes():
    import torch
    with pytest.raises(pa.PAError, match="PA_EUNSUPPORTED"):
        pa._dtype_code(torch.empty(1, dtype=torch.float16))


def test_header_is_plain_c_and_links(tmp_path):
    # the C ABI compiles as C99 and links against the library; without a GPU the program
    # checks the device-free calls
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(pa.lib_path())
    exe = tmp_path / "c_abi_check"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                        os.path.join(root, "tests", "c_abi_check.c"), "-L", libdir, "-lpa",
                        f"-Wl,-rpath,{libdir}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)


@pytest.mark.parametrize("n_chunks,gpc", [(1, 4), (2, 1), (5, 2), (16, 4), (16, 1), (7, 3)])
def test_overlapped_relayout_launches_cover_every_pair_once(n_chunks, gpc):
    # the attention launches of the chunked relayout pipeline select every (query group,
    # KV group) pair exactly once, and only pairs whose chunks have both moved
    from sequence_partition_attn_b200.step import chunk_milestones, milestone_masks
    QG = n_chunks * gpc
    ms = chunk_milestones(n_chunks)
    assert ms[-1] == n_chunks and ms == sorted(set(ms))
    masks = milestone_masks(QG, gpc, ms)
    total = np.sum(masks, axis=0)
    np.testing.assert_array_equal(total, np.ones((QG, QG)))
    for m, mask in zip(ms, masks):
        qg, kg = np.nonzero(mask)
        assert (qg < m * gpc).all() and (kg < m * gpc).all()


@pytest.mark.parametrize("N,P,G,n_chunks,ok", [
    (115200, 64, 1, 16, True),      # the Ulysses layout workload: 7200-token chunks
    (100, 8, 1, 4, False),          # chunks end at 25/50/75, partitions at 26/52/78
    (96, 8, 2, 4, True),
    (96, 8, 4, 4, False),           # 2 partitions per chunk, groups of 4
    (96, 8, 1, 3, False),           # 8 partitions do not split into 3 chunks
    (75600, 32, 4, 8, False),       # the 720p partitioning (S = 2363) against 9450-token chunks
])
def test_overlapped_relayout_rejects_chunks_off_the_partition_bounds(N, P, G, n_chunks, ok):
    # the chunked pipeline starts attention on partitions whose K/V rows the relayout has
    # moved: chunk and partition boundaries must coincide, or it raises before any launch
    import workloads as W
    from sequence_partition_attn_b200.step import check_chunk_bounds, relayout_overlapped
    off = W.part_offsets(N, P)
    if ok:
        check_chunk_bounds(off, G, n_chunks)
    else:
        with pytest.raises(ValueError):
            check_chunk_bounds(off, G, n_chunks)
        with pytest.raises(ValueError):      # raised before the first CUDA call
            relayout_overlapped(None, (None,) * 3, (None,) * 3, n_chunks, off, G, None, None,
                                None, None)


def test_algorithmic_work_of_the_configurations():
    # flop and byte accounting behind every throughput figure, against the counts derived
    # by hand from the configuration text: 4*D per (query row, valid key) of each fresh
    # pair; merge bytes P*(D*b + 4) read + (D*b + 4) written per row
    import workloads as W
    from sequence_partition_attn_b200.step import attn_flops, merge_bytes
    expect = {0: (4 * 64 * 2 * 1024 * 1024, None),                        # all pairs fresh
              1: (4 * 128 * 24 * 512 * 512 * 22, 4096 * 24 * (8 * 260 + 260)),   # 22 of 64 pairs
              2: (29265744363520, 75600 * 40 * (32 * 260 + 260))}
    for i, (fl, mb) in expect.items():
        wl = W.workload(i)
        assert attn_flops(W.part_offsets(wl.N, wl.P), wl.G, W.reuse_mask(wl), wl.B, wl.H, wl.D) == fl
        if mb is not None:
            assert merge_bytes(wl.B, wl.H, wl.N, wl.D, wl.P, wl.elem_bytes) == mb
    # 720p: 8 query groups of 9452 / 9452 / ... rows with a 9436-row tail (2347 + 3 * 2363)
    wl = W.workload(2)
    rows = np.diff(W.group_row_bounds(W.part_offsets(wl.N, wl.P), wl.G))
    fresh = W.reuse_mask(wl)
    total = sum(int(rows[q]) * int(rows[k]) for q in range(8) for k in range(8) if fresh[q, k])
    assert 4 * 128 * 40 * total == 29265744363520


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    # no fallback: with libpa.so absent every call raises instead of computing elsewhere
    monkeypatch.setattr(pa, "_LIB", None)
    monkeypatch.setattr(pa, "lib_path", lambda: str(tmp_path / "libpa.so"))
    with pytest.raises(RuntimeError, match="missing"):
        pa.lib()
    with pytest.raises(RuntimeError, match="missing"):
        pa.Context(0)
