"""ctypes binding of libgdn.so (see include/gdn.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, and their ``data_ptr()`` and the current CUDA stream are handed to
the C entry points.  All computation happens in the library's CUDA kernels.
PyTorch is used for device memory and streams.  If the shared library is
missing, every call raises ``GdnError``: there is no fallback.
"""
import contextlib
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = 0, 1, 2, 3, 4
GDN_F32, GDN_BF16 = 0, 1
_DTYPES = {torch.float32: GDN_F32, torch.bfloat16: GDN_BF16}
# gdn_prefill_kernel values
PREFILL_KERNELS = {"auto": 0, "simt": 1, "tc": 2}


class GdnError(RuntimeError):
    """A non-OK status from libgdn.so, or the library could not be loaded."""

    def __init__(self, msg, status=None):
        super().__init__(msg)
        self.status = status


_lib = None


class PipelineOptions(ctypes.Structure):
    """gdn_pipeline_options: chain_ctas (0 = automatic), wait_limit_cycles (0 = 2^32)."""
    _fields_ = [("chain_ctas", ctypes.c_int), ("wait_limit_cycles", ctypes.c_longlong)]


def library():
    """Loads libgdn.so once (no build step at run time; see ``build.py``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY_PATH):
            raise GdnError(f"libgdn.so not found at {LIBRARY_PATH}; build it with "
                           "`python -m linear_attention_recurrence_07_b200.build`")
        lib = ctypes.CDLL(LIBRARY_PATH)
        vp, fp, I = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
        lib.gdn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp,
                                      I, I, I, I, I, I, I, I, vp]
        lib.gdn_chunk_fwd.restype = I
        lib.gdn_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp,
                                        I, I, I, I, I, I, vp]
        lib.gdn_decode_step.restype = I
        lib.gdn_chunk_fwd_varlen.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp,
                                             I, I, I, I, I, I, I, I, vp]
        lib.gdn_chunk_fwd_varlen.restype = I
        lib.gdn_chunk_fwd_split_workspace.argtypes = [I, I, I, I, I, I]
        lib.gdn_chunk_fwd_split_workspace.restype = ctypes.c_size_t
        lib.gdn_chunk_fwd_split.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp,
                                            I, I, I, I, I, I, I, I, I, vp, ctypes.c_size_t, vp]
        lib.gdn_chunk_fwd_split.restype = I
        lib.gdn_chunk_fwd_split_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp,
                                                    I, I, I, I, I, I, I, I, I, vp]
        lib.gdn_chunk_fwd_split_noalloc.restype = I
        lib.gdn_decode_tokens.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, fp,
                                          I, I, I, I, I, I, I, vp]
        lib.gdn_decode_tokens.restype = I
        lib.gdn_decode_step_slots.argtypes = [vp, vp, vp, fp, fp, fp, vp, vp,
                                              I, I, I, I, I, I, I, vp]
        lib.gdn_decode_step_slots.restype = I
        lib.gdn_bwd_workspace.argtypes = [I, I, I, I, I]
        lib.gdn_bwd_workspace.restype = ctypes.c_size_t
        lib.gdn_bwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, fp, fp, fp, fp, fp, fp,
                                I, I, I, I, I, I, I, vp, ctypes.c_size_t, vp]
        lib.gdn_bwd.restype = I
        lib.gdn_bwd_chunk_workspace.argtypes = [I, I, I, I, I]
        lib.gdn_bwd_chunk_workspace.restype = ctypes.c_size_t
        lib.gdn_bwd_chunk.argtypes = lib.gdn_bwd.argtypes
        lib.gdn_bwd_chunk.restype = I
        lib.gdn_chunk_fwd_pipelined_workspace.argtypes = [I, I, I, I, I]
        lib.gdn_chunk_fwd_pipelined_workspace.restype = ctypes.c_size_t
        lib.gdn_chunk_fwd_pipelined.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp,
                                                I, I, I, I, I, I, I, I,
                                                ctypes.POINTER(PipelineOptions), vp, ctypes.c_size_t, vp]
        lib.gdn_chunk_fwd_pipelined.restype = I
        lib.gdn_device_status.argtypes = [vp]
        lib.gdn_device_status.restype = I
        lib.gdn_status_string.argtypes = [I]
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_last_cuda_error.argtypes = []
        lib.gdn_last_cuda_error.restype = I
        lib.gdn_version.argtypes = []
        lib.gdn_version.restype = I
        lib.gdn_set_prefill_kernel.argtypes = [I]
        lib.gdn_set_prefill_kernel.restype = I
        lib.gdn_get_prefill_kernel.argtypes = []
        lib.gdn_get_prefill_kernel.restype = I
        lib.gdn_prefill_kernel_for.argtypes = [I, I, I]
        lib.gdn_prefill_kernel_for.restype = I
        _lib = lib
    return _lib


def _call(dev, fn, *args):
    """Runs the C entry point with ``dev`` as the current CUDA device (the library
    looks up per-device state, such as static scratch, on the current device)."""
    with torch.cuda.device(dev):
        return fn(*args)


def _check(status, what):
    if status != GDN_OK:
        lib = library()
        name = lib.gdn_status_string(status).decode()
        extra = ""
        if status == GDN_ERR_CUDA:
            extra = f" (cudaError {lib.gdn_last_cuda_error()})"
        raise GdnError(f"{what} failed: {name}{extra}", status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _expect_cuda(q):
    if q.dtype not in _DTYPES:
        raise GdnError(f"unsupported dtype {q.dtype}")
    if q.device.type != "cuda":
        raise GdnError(f"tensors must be on a CUDA device, got {q.device}")


def _expect(t, name, shape, dtype, device):
    if t is None:
        raise GdnError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise GdnError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise GdnError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.device != device:
        raise GdnError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise GdnError(f"{name} must be contiguous")


def gdn_chunk_fwd(q, k, v, alpha, beta, S0, o, S_final, chunk=64, stream=None):
    """Prefill of T tokens (C entry point ``gdn_chunk_fwd``); writes o and S_final.

    q, k [B, T, Hqk, dk] and v, o [B, T, Hv, dv] (float32 or bfloat16, all the
    same); alpha, beta [B, T, Hv] float32; S0, S_final [B, Hv, dk, dv] float32
    or None.  Asynchronous on ``stream`` (default: the current stream)."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, T, Hv, dv), q.dtype),
                               ("o", o, (B, T, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, T, Hv), torch.float32),
                               ("beta", beta, (B, T, Hv), torch.float32)):
        _expect(t, name, shape, dt, dev)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None:
            _expect(t, name, (B, Hv, dk, dv), torch.float32, dev)
    _check(_call(dev, library().gdn_chunk_fwd, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                                   _ptr(o), _ptr(S_final), B, T, Hqk, Hv, dk, dv, chunk,
                                   _DTYPES[q.dtype], _stream_handle(stream, dev)),
           "gdn_chunk_fwd")


def gdn_decode_step(q, k, v, alpha, beta, S, o, S_new, stream=None):
    """One decode token (C entry point ``gdn_decode_step``); writes o and S_new
    (S_new may be S itself).  q, k [B, Hqk, dk]; v, o [B, Hv, dv]; alpha, beta
    [B, Hv] float32; S, S_new [B, Hv, dk, dv] float32."""
    B, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, Hv, dv), q.dtype),
                               ("o", o, (B, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, Hv), torch.float32),
                               ("beta", beta, (B, Hv), torch.float32),
                               ("S", S, (B, Hv, dk, dv), torch.float32),
                               ("S_new", S_new, (B, Hv, dk, dv), torch.float32)):
        _expect(t, name, shape, dt, dev)
    _check(_call(dev, library().gdn_decode_step, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S),
                                     _ptr(o), _ptr(S_new), B, Hqk, Hv, dk, dv,
                                     _DTYPES[q.dtype], _stream_handle(stream, dev)),
           "gdn_decode_step")


def set_prefill_kernel(name):
    """Selects the kernel of every later prefill call of this thread (C entry point
    ``gdn_set_prefill_kernel``, a per-thread setting): one of ``PREFILL_KERNELS``."""
    if name not in PREFILL_KERNELS:
        raise GdnError(f"unknown prefill kernel {name!r}; one of {sorted(PREFILL_KERNELS)}")
    _check(library().gdn_set_prefill_kernel(PREFILL_KERNELS[name]), "gdn_set_prefill_kernel")


def get_prefill_kernel():
    """The current prefill kernel choice, as a key of ``PREFILL_KERNELS``."""
    code = library().gdn_get_prefill_kernel()
    return {v: k for k, v in PREFILL_KERNELS.items()}[code]


def prefill_kernel_for(B, Hv, dtype):
    """The kernel a prefill of B sequences x Hv V heads in ``dtype`` (a torch dtype)
    runs under the current choice (C entry point ``gdn_prefill_kernel_for``)."""
    code = library().gdn_prefill_kernel_for(B, Hv, _DTYPES[dtype])
    if code < 0:
        raise GdnError(f"no prefill kernel takes B={B}, Hv={Hv}, {dtype} under the current choice",
                       GDN_ERR_UNSUPPORTED)
    return {v: k for k, v in PREFILL_KERNELS.items()}[code]


@contextlib.contextmanager
def prefill_kernel(name):
    """Context manager: ``name`` is the prefill kernel inside the block, the previous
    choice is restored after it."""
    prev = get_prefill_kernel()
    set_prefill_kernel(name)
    try:
        yield
    finally:
        set_prefill_kernel(prev)


def split_workspace_bytes(B, T, Hv, segments=0, dk=128, dv=128):
    """Device scratch bytes gdn_chunk_fwd_split needs (C entry point
    ``gdn_chunk_fwd_split_workspace``); 0 when no split happens."""
    return library().gdn_chunk_fwd_split_workspace(B, T, Hv, dk, dv, segments)


def gdn_chunk_fwd_split(q, k, v, alpha, beta, S0, o, S_final, segments=0, workspace=None,
                        chunk=64, stream=None):
    """Segment-parallel prefill (C entry point ``gdn_chunk_fwd_split``): the same
    arguments and results as gdn_chunk_fwd.  ``workspace`` is a uint8 CUDA tensor of
    at least split_workspace_bytes(...) bytes; None allocates one for this call."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, T, Hv, dv), q.dtype),
                               ("o", o, (B, T, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, T, Hv), torch.float32),
                               ("beta", beta, (B, T, Hv), torch.float32)):
        _expect(t, name, shape, dt, dev)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None:
            _expect(t, name, (B, Hv, dk, dv), torch.float32, dev)
    if workspace is None:
        need = split_workspace_bytes(B, T, Hv, segments, dk, dv)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    elif workspace.device != dev or workspace.dtype != torch.uint8:
        raise GdnError("workspace must be a uint8 tensor on the inputs' device")
    _check(_call(dev, library().gdn_chunk_fwd_split, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                         _ptr(S0), _ptr(o), _ptr(S_final), B, T, Hqk, Hv, dk, dv,
                                         chunk, segments, _DTYPES[q.dtype], _ptr(workspace),
                                         workspace.numel(), _stream_handle(stream, dev)),
           "gdn_chunk_fwd_split")


def bwd_workspace_bytes(B, T, Hv, dk=128, dv=128):
    """Device scratch bytes gdn_bwd needs (C entry point ``gdn_bwd_workspace``)."""
    return library().gdn_bwd_workspace(B, T, Hv, dk, dv)


def bwd_chunk_workspace_bytes(B, T, Hv, dk=128, dv=128):
    """Device scratch bytes gdn_bwd_chunk needs (C entry point ``gdn_bwd_chunk_workspace``)."""
    return library().gdn_bwd_chunk_workspace(B, T, Hv, dk, dv)


def _run_bwd(entry, ws_bytes, q, k, v, alpha, beta, S0, dO, dS_final, dq, dk, dv, dalpha, dbeta, dS0,
             workspace, stream):
    B, T, Hqk, dkk = q.shape
    Hv, dvv = v.shape[2], v.shape[3]
    dev = q.device
    _expect_cuda(q)
    f32 = torch.float32
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, T, Hv, dvv), q.dtype),
                               ("dO", dO, (B, T, Hv, dvv), q.dtype),
                               ("alpha", alpha, (B, T, Hv), f32), ("beta", beta, (B, T, Hv), f32),
                               ("dq", dq, q.shape, f32), ("dk", dk, q.shape, f32),
                               ("dv", dv, (B, T, Hv, dvv), f32), ("dalpha", dalpha, (B, T, Hv), f32),
                               ("dbeta", dbeta, (B, T, Hv), f32), ("dS0", dS0, (B, Hv, dkk, dvv), f32)):
        _expect(t, name, shape, dt, dev)
    for name, t in (("S0", S0), ("dS_final", dS_final)):
        if t is not None:
            _expect(t, name, (B, Hv, dkk, dvv), f32, dev)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes(B, T, Hv, dkk, dvv), 1), dtype=torch.uint8, device=dev)
    elif workspace.device != dev or workspace.dtype != torch.uint8:
        raise GdnError("workspace must be a uint8 tensor on the inputs' device")
    _check(_call(dev, getattr(library(), entry), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S0),
                 _ptr(dO), _ptr(dS_final), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dalpha), _ptr(dbeta),
                 _ptr(dS0), B, T, Hqk, Hv, dkk, dvv, _DTYPES[q.dtype], _ptr(workspace),
                 workspace.numel(), _stream_handle(stream, dev)),
           entry)


def gdn_bwd(q, k, v, alpha, beta, S0, dO, dS_final, dq, dk, dv, dalpha, dbeta, dS0,
            workspace=None, stream=None):
    """Gradients of sum <dO, o> + <dS_final, S_final> (C entry point ``gdn_bwd``).

    q, k, v, dO: the forward's dtype; alpha, beta, S0, dS_final fp32 (S0 and
    dS_final may be None).  Outputs (fp32, overwritten): dq, dk like q; dv like v;
    dalpha, dbeta like alpha; dS0 [B, Hv, dk, dv].  ``workspace``: uint8 CUDA
    tensor of at least bwd_workspace_bytes(...) bytes; None allocates one."""
    _run_bwd("gdn_bwd", bwd_workspace_bytes, q, k, v, alpha, beta, S0, dO, dS_final, dq, dk, dv,
             dalpha, dbeta, dS0, workspace, stream)


def gdn_bwd_chunk(q, k, v, alpha, beta, S0, dO, dS_final, dq, dk, dv, dalpha, dbeta, dS0,
                  workspace=None, stream=None):
    """The gradients of gdn_bwd in the chunkwise form on tensor cores (C entry point
    ``gdn_bwd_chunk``); bf16 q, k, v, dO, the same arguments; ``workspace`` of at
    least bwd_chunk_workspace_bytes(...) bytes, None allocates one."""
    _run_bwd("gdn_bwd_chunk", bwd_chunk_workspace_bytes, q, k, v, alpha, beta, S0, dO, dS_final, dq, dk,
             dv, dalpha, dbeta, dS0, workspace, stream)


def gdn_chunk_fwd_split_noalloc(q, k, v, alpha, beta, S0, o, S_final, segments=0, chunk=64,
                                stream=None):
    """gdn_chunk_fwd_split with the library's static scratch (C entry point
    ``gdn_chunk_fwd_split_noalloc``); the same arguments without a workspace."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, T, Hv, dv), q.dtype),
                               ("o", o, (B, T, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, T, Hv), torch.float32),
                               ("beta", beta, (B, T, Hv), torch.float32)):
        _expect(t, name, shape, dt, dev)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None:
            _expect(t, name, (B, Hv, dk, dv), torch.float32, dev)
    _check(_call(dev, library().gdn_chunk_fwd_split_noalloc, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                                 _ptr(S0), _ptr(o), _ptr(S_final), B, T, Hqk, Hv,
                                                 dk, dv, chunk, segments, _DTYPES[q.dtype],
                                                 _stream_handle(stream, dev)),
           "gdn_chunk_fwd_split_noalloc")


def gdn_chunk_fwd_varlen(q, k, v, alpha, beta, S0, o, S_final, cu_seqlens, chunk=64,
                         stream=None):
    """Prefill of N packed sequences (C entry point ``gdn_chunk_fwd_varlen``).  q, k
    [T_total, Hqk, dk] and v, o [T_total, Hv, dv] (float32 or bfloat16); alpha,
    beta [T_total, Hv] float32; cu_seqlens [N + 1] int32; S0, S_final
    [N, Hv, dk, dv] float32 or None."""
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    N = cu_seqlens.shape[0] - 1
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (T, Hv, dv), q.dtype),
                               ("o", o, (T, Hv, dv), q.dtype),
                               ("alpha", alpha, (T, Hv), torch.float32),
                               ("beta", beta, (T, Hv), torch.float32),
                               ("cu_seqlens", cu_seqlens, (N + 1,), torch.int32)):
        _expect(t, name, shape, dt, dev)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None:
            _expect(t, name, (N, Hv, dk, dv), torch.float32, dev)
    _check(_call(dev, library().gdn_chunk_fwd_varlen, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                          _ptr(S0), _ptr(o), _ptr(S_final), _ptr(cu_seqlens),
                                          N, T, Hqk, Hv, dk, dv, chunk, _DTYPES[q.dtype],
                                          _stream_handle(stream, dev)),
           "gdn_chunk_fwd_varlen")


def gdn_decode_tokens(q, k, v, alpha, beta, S, o, S_new, S_steps=None, stream=None):
    """n decode tokens per sequence (C entry point ``gdn_decode_tokens``); writes o,
    S_new (may be S itself) and, if given, S_steps.  q, k [B, n, Hqk, dk]; v, o
    [B, n, Hv, dv]; alpha, beta [B, n, Hv] float32; S, S_new [B, Hv, dk, dv]
    float32; S_steps [B, n, Hv, dk, dv] float32 or None."""
    B, n, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, n, Hv, dv), q.dtype),
                               ("o", o, (B, n, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, n, Hv), torch.float32),
                               ("beta", beta, (B, n, Hv), torch.float32),
                               ("S", S, (B, Hv, dk, dv), torch.float32),
                               ("S_new", S_new, (B, Hv, dk, dv), torch.float32)):
        _expect(t, name, shape, dt, dev)
    if S_steps is not None:
        _expect(S_steps, "S_steps", (B, n, Hv, dk, dv), torch.float32, dev)
    _check(_call(dev, library().gdn_decode_tokens, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(S),
                                       _ptr(o), _ptr(S_new), _ptr(S_steps), B, n, Hqk, Hv, dk, dv,
                                       _DTYPES[q.dtype], _stream_handle(stream, dev)),
           "gdn_decode_tokens")


def gdn_decode_step_slots(q, k, v, alpha, beta, state_pool, slots, o, stream=None):
    """One decode token per sequence with states in a pool (C entry point
    ``gdn_decode_step_slots``): state_pool[slots[b]] is updated in place.  q, k
    [B, Hqk, dk]; v, o [B, Hv, dv]; alpha, beta [B, Hv] float32; state_pool
    [n_slots, Hv, dk, dv] float32; slots [B] int32."""
    B, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    n_slots = state_pool.shape[0]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, Hv, dv), q.dtype),
                               ("o", o, (B, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, Hv), torch.float32),
                               ("beta", beta, (B, Hv), torch.float32),
                               ("state_pool", state_pool, (n_slots, Hv, dk, dv), torch.float32),
                               ("slots", slots, (B,), torch.int32)):
        _expect(t, name, shape, dt, dev)
    _check(_call(dev, library().gdn_decode_step_slots, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                           _ptr(state_pool), _ptr(slots), _ptr(o), B, n_slots,
                                           Hqk, Hv, dk, dv, _DTYPES[q.dtype],
                                           _stream_handle(stream, dev)),
           "gdn_decode_step_slots")


def pipelined_workspace_bytes(B, Hqk, Hv, dk=128, dv=128):
    """Device scratch bytes gdn_chunk_fwd_pipelined needs on the current device (C
    entry point ``gdn_chunk_fwd_pipelined_workspace``)."""
    return library().gdn_chunk_fwd_pipelined_workspace(B, Hqk, Hv, dk, dv)


def gdn_chunk_fwd_pipelined(q, k, v, alpha, beta, S0, o, S_final, chain_ctas=0,
                            wait_limit_cycles=0, workspace=None, chunk=64, stream=None):
    """Prefill with the chunks' WY preparation streamed from SMs of its own (C entry
    point ``gdn_chunk_fwd_pipelined``): the same arguments and results as
    gdn_chunk_fwd.  ``workspace`` is a uint8 CUDA tensor of at least
    pipelined_workspace_bytes(...) bytes; None allocates one for this call."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dev = q.device
    _expect_cuda(q)
    for name, t, shape, dt in (("k", k, q.shape, q.dtype), ("v", v, (B, T, Hv, dv), q.dtype),
                               ("o", o, (B, T, Hv, dv), q.dtype),
                               ("alpha", alpha, (B, T, Hv), torch.float32),
                               ("beta", beta, (B, T, Hv), torch.float32)):
        _expect(t, name, shape, dt, dev)
    for name, t in (("S0", S0), ("S_final", S_final)):
        if t is not None:
            _expect(t, name, (B, Hv, dk, dv), torch.float32, dev)
    if workspace is None:
        with torch.cuda.device(dev):
            need = pipelined_workspace_bytes(B, Hqk, Hv, dk, dv)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    elif workspace.device != dev or workspace.dtype != torch.uint8:
        raise GdnError("workspace must be a uint8 tensor on the inputs' device")
    opts = PipelineOptions(int(chain_ctas), int(wait_limit_cycles))
    _check(_call(dev, library().gdn_chunk_fwd_pipelined, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                 _ptr(beta), _ptr(S0), _ptr(o), _ptr(S_final), B, T, Hqk, Hv, dk, dv, chunk,
                 _DTYPES[q.dtype], ctypes.byref(opts), _ptr(workspace), workspace.numel(),
                 _stream_handle(stream, dev)),
           "gdn_chunk_fwd_pipelined")


def device_status(stream=None, device=None):
    """Waits for ``stream`` and returns (and clears) the library's device error
    state as a status name: "GDN_OK", or "GDN_ERR_TIMEOUT" if a bounded wait inside
    a kernel gave up (C entry point ``gdn_device_status``)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = _call(dev, library().gdn_device_status, _stream_handle(stream, dev))
    return library().gdn_status_string(code).decode()


def chunk_fwd(q, k, v, alpha, beta, S0=None, chunk=64, stream=None):
    """Allocating convenience wrapper: returns (o, S_final)."""
    B, T, Hqk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    o = torch.empty((B, T, Hv, dv), dtype=q.dtype, device=q.device)
    S_final = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    gdn_chunk_fwd(q, k, v, alpha, beta, S0, o, S_final, chunk=chunk, stream=stream)
    return o, S_final


def decode_step(q, k, v, alpha, beta, S, stream=None):
    """In-place decode convenience wrapper: updates S and returns o."""
    B, Hv, dv = v.shape
    o = torch.empty((B, Hv, dv), dtype=q.dtype, device=q.device)
    gdn_decode_step(q, k, v, alpha, beta, S, o, S, stream=stream)
    return o
