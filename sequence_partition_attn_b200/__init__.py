"""Python binding of libpa: partition attention with attention-state merge, selective reuse
and partition importance on one B200 (sm_100a).

Argument marshalling only -- every step of the path runs in libpa's CUDA kernels.  Tensors
are passed as device pointers (``tensor.data_ptr()``), partition offsets and reuse masks as
host arrays, and the stream is the current PyTorch CUDA stream unless one is given.  The
names follow the C ABI in ``include/pa.h``:

    pa_init / Context            pa_partition_attn    pa_merge_states
    pa_importance                pa_relayout_seq2head pa_sync_status / pa_wait_status
    pa_merge_states_noalloc      pa_compose_states    pa_state_drift

There is no fallback: if ``libpa.so`` is missing or the device is not sm_100 the calls
raise.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "PA_F32", "PA_BF16", "PAError", "Context", "lib", "lib_path",
    "pa_partition_attn", "pa_merge_states", "pa_importance", "pa_relayout_seq2head",
    "pa_merge_states_noalloc", "pa_compose_states", "pa_state_drift", "pa_selftest_wait", "EXPORTED",
    "pa_relayout_seq2head_at",
    "select_fresh",
    "predict_fresh",
]

PA_F32, PA_BF16 = 0, 1
PA_MAX_P = 128
_ERRORS = {-1: "PA_EINVAL", -2: "PA_EALIGN", -3: "PA_EUNSUPPORTED", -4: "PA_ENOMEM",
           -5: "PA_ECUDA", -6: "PA_ETIMEOUT"}
EXPORTED = ("pa_init", "pa_destroy", "pa_last_error", "pa_sync_status", "pa_wait_status", "pa_version",
            "pa_partition_attn", "pa_merge_states", "pa_importance", "pa_relayout_seq2head",
            "pa_merge_states_noalloc", "pa_compose_states", "pa_state_drift", "pa_selftest_wait",
            "pa_relayout_seq2head_at")

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "libpa.so")


class PAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{_ERRORS.get(code, code)}: {msg}")
        self.code = code


class _AttnDesc(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("N", ctypes.c_int), ("D", ctypes.c_int), ("scale", ctypes.c_float),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("P", ctypes.c_int), ("part_off", ctypes.c_void_p), ("G", ctypes.c_int),
                ("fresh", ctypes.c_void_p), ("o_part", ctypes.c_void_p),
                ("lse_part", ctypes.c_void_p)]


class _MergeDesc(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("N", ctypes.c_int), ("D", ctypes.c_int), ("P", ctypes.c_int),
                ("G", ctypes.c_int), ("part_off", ctypes.c_void_p),
                ("o_fresh", ctypes.c_void_p), ("lse_fresh", ctypes.c_void_p),
                ("o_cached", ctypes.c_void_p), ("lse_cached", ctypes.c_void_p),
                ("fresh", ctypes.c_void_p), ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("cached_per_group", ctypes.c_int)]


_LIB = None


def lib():
    """Load libpa.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m sequence_partition_attn_b200.build`")
        L = ctypes.CDLL(path)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        L.pa_init.argtypes = [ci, ctypes.POINTER(vp)]
        L.pa_destroy.argtypes = [vp]
        L.pa_destroy.restype = None
        L.pa_last_error.argtypes = [vp]
        L.pa_last_error.restype = ctypes.c_char_p
        L.pa_sync_status.argtypes = [vp, vp]
        L.pa_wait_status.argtypes = [vp, vp, ctypes.c_double]
        L.pa_version.restype = ctypes.c_char_p
        L.pa_partition_attn.argtypes = [vp, ctypes.POINTER(_AttnDesc), vp]
        L.pa_merge_states.argtypes = [vp, ctypes.POINTER(_MergeDesc), vp]
        L.pa_merge_states_noalloc.argtypes = [ctypes.POINTER(_MergeDesc), vp]
        L.pa_importance.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp]
        L.pa_compose_states.argtypes = [vp, ci, ci, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp]
        L.pa_relayout_seq2head.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, vp]
        L.pa_relayout_seq2head_at.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, vp]
        L.pa_state_drift.argtypes = [vp, ci, ci, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp, vp]
        L.pa_selftest_wait.argtypes = [vp, ctypes.c_double, vp]
        for f in ("pa_init", "pa_sync_status", "pa_wait_status", "pa_partition_attn", "pa_merge_states", "pa_merge_states_noalloc",
                  "pa_compose_states", "pa_state_drift", "pa_selftest_wait",
                  "pa_importance", "pa_relayout_seq2head", "pa_relayout_seq2head_at"):
            getattr(L, f).restype = ci
        _LIB = L
    return _LIB


def _check(ctx_ptr, rc):
    if rc != 0:
        msg = lib().pa_last_error(ctx_ptr)
        raise PAError(rc, msg.decode() if msg else "")


class Context:
    """A libpa context on one device (pa_init / pa_destroy)."""

    def __init__(self, device: int = 0):
        self._ptr = ctypes.c_void_p()
        _check(None, lib().pa_init(device, ctypes.byref(self._ptr)))
        self.device = device

    @property
    def ptr(self):
        return self._ptr

    def sync_status(self, stream=None, timeout=None):
        """pa_sync_status: synchronise the stream, raise if a device wait gave up.  With
        `timeout` (seconds), pa_wait_status: raise PAError (PA_ETIMEOUT) if the stream's
        work has not finished by then (nothing is cancelled)."""
        if timeout is None:
            _check(self._ptr, lib().pa_sync_status(self._ptr, _stream(stream)))
        else:
            _check(self._ptr, lib().pa_wait_status(self._ptr, _stream(stream), float(timeout)))

    def close(self):
        if self._ptr:
            lib().pa_destroy(self._ptr)
            self._ptr = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float32:
        return PA_F32
    raise PAError(-3, f"dtype {t.dtype} not supported")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _host_i32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _host_u8(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.uint8))


def pa_partition_attn(ctx: Context, q, k, v, part_off, G, fresh, o_part, lse_part,
                      scale=None, stream=None):
    """Per-partition attention states (O_p, LSE_p) for the fresh (query group, KV group)
    pairs.  q, k, v: [B, H, N, D] CUDA tensors (bf16 or f32); o_part [P, B, H, N, D];
    lse_part [P, B, H, N] f32; part_off int[P+1]; fresh uint8 [QG, KG] or None."""
    B, H, N, D = q.shape
    off = _host_i32(part_off)
    fr = _host_u8(fresh)
    d = _AttnDesc(_dtype_code(q), B, H, N, D,
                  float(scale if scale is not None else 1.0 / np.sqrt(D)),
                  q.data_ptr(), k.data_ptr(), v.data_ptr(), len(off) - 1,
                  off.ctypes.data, int(G), None if fr is None else fr.ctypes.data,
                  o_part.data_ptr(), lse_part.data_ptr())
    _check(ctx.ptr, lib().pa_partition_attn(ctx.ptr, ctypes.byref(d), _stream(stream)))


def pa_merge_states(ctx: Context, part_off, G, fresh, o_fresh, lse_fresh, o_cached, lse_cached,
                    o, lse, w=None, stream=None, cached_per_group=False):
    """Merge fresh / cached states per the mask; o [B, H, N, D], lse [B, H, N]; w [QG, P]
    (fused importance) optional.  cached_per_group: the cache holds one composed state per
    KV group ([KG, B, H, N, D], from pa_compose_states)."""
    P, B, H, N, D = o_fresh.shape
    off = _host_i32(part_off)
    fr = _host_u8(fresh)
    d = _MergeDesc(_dtype_code(o_fresh), B, H, N, D, P, int(G), off.ctypes.data,
                   o_fresh.data_ptr(), lse_fresh.data_ptr(),
                   None if o_cached is None else o_cached.data_ptr(),
                   None if lse_cached is None else lse_cached.data_ptr(),
                   None if fr is None else fr.ctypes.data, o.data_ptr(), lse.data_ptr(),
                   None if w is None else w.data_ptr(), 1 if cached_per_group else 0)
    _check(ctx.ptr, lib().pa_merge_states(ctx.ptr, ctypes.byref(d), _stream(stream)))


def pa_compose_states(ctx: Context, o_part, lse_part, factor, o_group, lse_group, stream=None):
    """Compose every `factor` consecutive partitions' states into one (no recomputation):
    o_part [P, B, H, N, D], lse_part [P, B, H, N] -> o_group [C, ...], lse_group [C, ...]."""
    P, B, H, N, D = o_part.shape
    _check(ctx.ptr, lib().pa_compose_states(ctx.ptr, _dtype_code(o_part), B, H, N, D, P, int(factor),
                                            o_part.data_ptr(), lse_part.data_ptr(),
                                            o_group.data_ptr(), lse_group.data_ptr(), _stream(stream)))


def pa_merge_states_noalloc(part_off, G, fresh, o_fresh, lse_fresh, o_cached, lse_cached, o, lse,
                            w=None, stream=None):
    """pa_merge_states without a context and without any device allocation: the fused
    importance uses libpa's fixed 4 MiB scratch array (for callers that must not call
    cudaMalloc).  Calls that overlap on the GPU share that scratch and must not be issued
    concurrently."""
    P, B, H, N, D = o_fresh.shape
    off = _host_i32(part_off)
    fr = _host_u8(fresh)
    d = _MergeDesc(_dtype_code(o_fresh), B, H, N, D, P, int(G), off.ctypes.data,
                   o_fresh.data_ptr(), lse_fresh.data_ptr(),
                   None if o_cached is None else o_cached.data_ptr(),
                   None if lse_cached is None else lse_cached.data_ptr(),
                   None if fr is None else fr.ctypes.data, o.data_ptr(), lse.data_ptr(),
                   None if w is None else w.data_ptr())
    _check(None, lib().pa_merge_states_noalloc(ctypes.byref(d), _stream(stream)))


def pa_importance(ctx: Context, part_off, G, lse_part, lse, w, stream=None):
    """w[qg, p] = mean over b, h, rows of qg of exp(lse_part - lse); w [QG, P] overwritten."""
    P, B, H, N = lse_part.shape
    off = _host_i32(part_off)
    _check(ctx.ptr, lib().pa_importance(ctx.ptr, B, H, N, P, int(G), off.ctypes.data,
                                        lse_part.data_ptr(), lse.data_ptr(), w.data_ptr(),
                                        _stream(stream)))


def pa_state_drift(ctx: Context, part_off, G, sel, o_new, o_ref, d2, r2, stream=None):
    """Per (query group, partition) sums of (o_new - o_ref)^2 and o_ref^2 over the pairs
    selected by sel (uint8 [QG, KG] or None = all): o_new, o_ref [P, B, H, N, D];
    d2, r2 [QG, P] f32, overwritten (0 for unselected pairs)."""
    P, B, H, N, D = o_new.shape
    off = _host_i32(part_off)
    sl = _host_u8(sel)
    _check(ctx.ptr, lib().pa_state_drift(ctx.ptr, _dtype_code(o_new), B, H, N, D, P, int(G),
                                         off.ctypes.data, None if sl is None else sl.ctypes.data,
                                         o_new.data_ptr(), o_ref.data_ptr(), d2.data_ptr(),
                                         r2.data_ptr(), _stream(stream)))


def pa_selftest_wait(ctx: Context, seconds=0.05, stream=None):
    """Launch the bounded-wait self-test: a wait that nothing completes gives up after
    `seconds`; the next ctx.sync_status() raises PAError with code PA_ETIMEOUT."""
    _check(ctx.ptr, lib().pa_selftest_wait(ctx.ptr, float(seconds), _stream(stream)))


def pa_relayout_seq2head(ctx: Context, src, dst, n_chunks=1, chunk=-1, stream=None):
    """dst[h, n, :] = src[n, h, :] for sequence chunk `chunk` of `n_chunks` (-1 = all)."""
    N, H, D = src.shape
    _check(ctx.ptr, lib().pa_relayout_seq2head(ctx.ptr, src.data_ptr(), dst.data_ptr(), N, H, D,
                                               src.element_size(), int(n_chunks), int(chunk),
                                               _stream(stream)))


def pa_relayout_seq2head_at(ctx: Context, src, dst, tok0, stream=None):
    """dst[h, tok0 + n, :] = src[n, h, :]: src [n_tok, H, D] placed at token tok0 of
    dst [H, N, D] (one piece of a chunked sequence-parallel all-to-all)."""
    n_tok, H, D = src.shape
    _check(ctx.ptr, lib().pa_relayout_seq2head_at(ctx.ptr, src.data_ptr(), dst.data_ptr(), n_tok, H, D,
                                                  src.element_size(), dst.shape[-2], int(tok0),
                                                  _stream(stream)))


def select_fresh(w_stored, G: int, threshold: float) -> np.ndarray:
    """Host reuse selection from stored importance: uint8[QG, KG], 1 where some partition of
    the KV group has stored importance at or above the threshold (recompute), else 0
    (reuse the cached states).  DiTango web summary, Methodology 1 (anchor-guided
    selection, group-wise decisions)."""
    w = np.asarray(w_stored, dtype=np.float64)
    QG, P = w.shape
    KG = -(-P // G)
    pad = np.full((QG, KG * G), -np.inf)
    pad[:, :P] = w
    return (pad.reshape(QG, KG, G).max(axis=2) >= threshold).astype(np.uint8)


def predict_fresh(w_stored, d2, r2, G: int, eps: float) -> np.ndarray:
    """Host reuse selection between anchors from predicted error (DiTango web summary,
    Methodology 1, "Error modelling" and "Online Prediction"): the error of reusing the
    states of partition p for query group qg grows with its stored importance times the
    drift of the states; the drift of the remote states is estimated by that of the own
    KV group's states, which are recomputed every step:
        drift[qg] = sqrt(sum_{p in own group} d2[qg, p] / sum_{p in own group} r2[qg, p]).
    Returns uint8[QG, KG]: 1 (recompute) where max_{p in kg} w_stored[qg, p] * drift[qg]
    reaches eps, and always on the diagonal (own group); d2, r2 as from pa_state_drift."""
    w = np.asarray(w_stored, dtype=np.float64)
    d2 = np.asarray(d2, dtype=np.float64)
    r2 = np.asarray(r2, dtype=np.float64)
    QG, P = w.shape
    KG = -(-P // G)
    own = (np.arange(P)[None, :] // G) == np.arange(QG)[:, None]
    num = np.where(own, d2, 0.0).sum(axis=1)
    den = np.where(own, r2, 0.0).sum(axis=1)
    drift = np.sqrt(np.divide(num, den, out=np.zeros_like(num), where=den > 0))
    pad = np.full((QG, KG * G), -np.inf)
    pad[:, :P] = w * drift[:, None]
    m = (pad.reshape(QG, KG, G).max(axis=2) >= eps).astype(np.uint8)
    m[np.arange(QG), np.arange(QG)] = 1
    return m
