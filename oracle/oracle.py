"""Python entry to the fp64 CPU oracle of the gated delta rule.

TEST INFRASTRUCTURE ONLY: used by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the library's compute path.

The arithmetic lives in ``gdn_oracle.c`` (token-by-token recurrence, first form
of the update in "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者", section 2.1
"Gated DeltaNet"); this module only converts arrays and calls it.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _library():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        fn = lib.gdn_oracle_forward
        fp = ctypes.c_void_p
        L = ctypes.c_long
        fn.argtypes = [fp, fp, fp, fp, fp, fp, fp, fp, L, L, L, L, L, L, L, L, ctypes.c_int]
        fn.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _f32(x):
    """Host fp32 copy of an array or CPU/GPU tensor (bf16 upcasts exactly)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def forward(q, k, v, alpha, beta, S0=None, h_range=None, nthreads=None):
    """fp64 token-by-token gated delta rule with read-out o_t = S_t^T q_t.

    q, k: [B, T, Hqk, dk]; v: [B, T, Hv, dv]; alpha, beta: [B, T, Hv];
    S0: [B, Hv, dk, dv] or None (zeros).  ``h_range`` = (h_begin, h_end)
    restricts the work to those V heads.  Returns (o, S_final) as float64
    arrays of shapes [B, T, nh, dv] and [B, nh, dk, dv], nh = h_end - h_begin.
    """
    q, k, v, alpha, beta, S0 = (_f32(a) for a in (q, k, v, alpha, beta, S0))
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T)
    assert alpha.shape == (B, T, Hv) and beta.shape == (B, T, Hv)
    if S0 is not None:
        assert S0.shape == (B, Hv, dk, dv)
    h0, h1 = (0, Hv) if h_range is None else h_range
    nh = h1 - h0
    o = np.zeros((B, T, nh, dv), dtype=np.float64)
    S_final = np.zeros((B, nh, dk, dv), dtype=np.float64)
    ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
    rc = _library().gdn_oracle_forward(
        ptr(q), ptr(k), ptr(v), ptr(alpha), ptr(beta), ptr(S0), ptr(o), ptr(S_final),
        B, T, Hqk, Hv, dk, dv, h0, h1, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_forward failed with code {rc}")
    return o, S_final


def decode_step(q, k, v, alpha, beta, S, nthreads=None):
    """One token of the recurrence for every (b, h): the same definition at T = 1.

    q, k: [B, Hqk, dk]; v: [B, Hv, dv]; alpha, beta: [B, Hv]; S: [B, Hv, dk, dv].
    Returns (o [B, Hv, dv], S_new [B, Hv, dk, dv]) in float64.
    """
    q, k, v, alpha, beta, S = (_f32(a) for a in (q, k, v, alpha, beta, S))
    o, S_new = forward(q[:, None], k[:, None], v[:, None], alpha[:, None], beta[:, None],
                       S, nthreads=nthreads)
    return o[:, 0], S_new
