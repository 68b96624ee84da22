"""Host-side checks of libgdn.so that need no GPU: the library loads, exports every
entry point include/gdn.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from linear_attention_recurrence_07_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for header in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not header.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", header)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(gdn_\w+)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIBRARY_PATH):
        from linear_attention_recurrence_07_b200 import build
        build.build()
    return binding.library()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdn_chunk_fwd", "gdn_decode_step", "gdn_status_string", "gdn_last_cuda_error",
              "gdn_version", "gdn_set_prefill_kernel", "gdn_get_prefill_kernel",
              "gdn_prefill_kernel_for", "gdn_decode_tokens", "gdn_decode_step_slots",
              "gdn_chunk_fwd_varlen", "gdn_chunk_fwd_split", "gdn_chunk_fwd_split_workspace",
              "gdn_bwd", "gdn_bwd_workspace", "gdn_bwd_chunk", "gdn_bwd_chunk_workspace"):
        assert n in names, names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libgdn.so does not export {name}"


def test_status_strings_and_version(lib):
    assert lib.gdn_status_string(0) == b"GDN_OK"
    assert lib.gdn_status_string(1) == b"GDN_ERR_INVALID_ARG"
    assert lib.gdn_status_string(2) == b"GDN_ERR_UNSUPPORTED"
    assert lib.gdn_status_string(3) == b"GDN_ERR_CUDA"
    assert lib.gdn_version() >= 100
    assert lib.gdn_last_cuda_error() == 0


FAKE = ctypes.c_void_p(0x1000)        # aligned, never dereferenced: checks reject first
MISALIGNED = ctypes.c_void_p(0x1004)


def chunk(lib, B=1, T=64, Hqk=1, Hv=1, dk=128, dv=128, C=64, dtype=1, ptr=FAKE, o=FAKE):
    return lib.gdn_chunk_fwd(ptr, FAKE, FAKE, FAKE, FAKE, None, o, None,
                             B, T, Hqk, Hv, dk, dv, C, dtype, None)


def decode(lib, B=1, Hqk=1, Hv=1, dk=128, dv=128, dtype=1, ptr=FAKE):
    return lib.gdn_decode_step(ptr, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                               B, Hqk, Hv, dk, dv, dtype, None)


def test_chunk_argument_checks(lib):
    assert chunk(lib, B=-1) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, T=-5) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, Hqk=0) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, Hv=0) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, Hqk=2, Hv=3) == binding.GDN_ERR_UNSUPPORTED
    assert chunk(lib, dk=64) == binding.GDN_ERR_UNSUPPORTED
    assert chunk(lib, dv=256) == binding.GDN_ERR_UNSUPPORTED
    assert chunk(lib, C=32) == binding.GDN_ERR_UNSUPPORTED
    assert chunk(lib, dtype=7) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, ptr=None) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, o=None) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, ptr=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, o=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert chunk(lib, B=70000) == binding.GDN_ERR_UNSUPPORTED
    # B == 0 is a no-op that succeeds without touching the device
    assert chunk(lib, B=0) == binding.GDN_OK
    # T == 0 with no S_final has nothing to do
    assert chunk(lib, T=0) == binding.GDN_OK


def test_decode_argument_checks(lib):
    assert decode(lib, B=-1) == binding.GDN_ERR_INVALID_ARG
    assert decode(lib, Hqk=0) == binding.GDN_ERR_INVALID_ARG
    assert decode(lib, Hqk=16, Hv=40) == binding.GDN_ERR_UNSUPPORTED
    assert decode(lib, dk=96) == binding.GDN_ERR_UNSUPPORTED
    assert decode(lib, dtype=-1) == binding.GDN_ERR_INVALID_ARG
    assert decode(lib, ptr=None) == binding.GDN_ERR_INVALID_ARG
    assert decode(lib, ptr=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert decode(lib, B=0) == binding.GDN_OK


def test_binding_raises_on_bad_tensors():
    import torch
    q = torch.zeros(1, 4, 1, 128)
    with pytest.raises(binding.GdnError, match="CUDA device"):   # host tensors are refused
        binding.gdn_chunk_fwd(q, q, q, torch.zeros(1, 4, 1), torch.zeros(1, 4, 1), None, q, None)
    with pytest.raises(binding.GdnError, match="CUDA device"):
        binding.gdn_decode_step(q[:, 0], q[:, 0], q[:, 0], torch.zeros(1, 1), torch.zeros(1, 1),
                                torch.zeros(1, 1, 128, 128), q[:, 0], torch.zeros(1, 1, 128, 128))
    with pytest.raises(binding.GdnError, match="unsupported dtype"):
        binding.gdn_chunk_fwd(q.to(torch.float16), q.to(torch.float16), q.to(torch.float16),
                              torch.zeros(1, 4, 1), torch.zeros(1, 4, 1), None,
                              q.to(torch.float16), None)


def test_prefill_kernel_selection(lib):
    assert lib.gdn_get_prefill_kernel() == binding.PREFILL_KERNELS["auto"]
    for name, code in binding.PREFILL_KERNELS.items():
        with binding.prefill_kernel(name):
            assert lib.gdn_get_prefill_kernel() == code
            assert binding.get_prefill_kernel() == name
        assert binding.get_prefill_kernel() == "auto"
    assert lib.gdn_set_prefill_kernel(3) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_set_prefill_kernel(-1) == binding.GDN_ERR_INVALID_ARG
    assert binding.get_prefill_kernel() == "auto"
    with pytest.raises(binding.GdnError, match="unknown prefill kernel"):
        binding.set_prefill_kernel("wgmma")
    # the tensor-core kernels take bf16 only: fp32 with a forced TC kernel is refused
    # on the host, before any launch
    for name in ("tc",):
        with binding.prefill_kernel(name):
            assert chunk(lib, dtype=0) == binding.GDN_ERR_UNSUPPORTED
            assert chunk(lib, dtype=0, T=0) == binding.GDN_OK   # nothing to launch


def test_prefill_kernel_for_without_device_work(lib):
    import torch
    # fp32 never needs the device to decide
    assert binding.prefill_kernel_for(1, 48, torch.float32) == "simt"
    with binding.prefill_kernel("simt"):
        assert binding.prefill_kernel_for(4, 48, torch.bfloat16) == "simt"
    for name in ("tc",):
        with binding.prefill_kernel(name):
            with pytest.raises(binding.GdnError, match="no prefill kernel"):
                binding.prefill_kernel_for(1, 48, torch.float32)
    assert lib.gdn_prefill_kernel_for(-1, 48, 1) == -1
    assert lib.gdn_prefill_kernel_for(1, 0, 1) == -1
    assert lib.gdn_prefill_kernel_for(1, 48, 5) == -1


def test_decode_tokens_argument_checks(lib):
    def call(B=1, n=2, Hqk=1, Hv=1, dk=128, dv=128, dtype=1, ptr=FAKE, S_new=FAKE, steps=None):
        return lib.gdn_decode_tokens(ptr, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, S_new, steps,
                                     B, n, Hqk, Hv, dk, dv, dtype, None)
    assert call(n=0) == binding.GDN_ERR_INVALID_ARG
    assert call(n=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(n=65) == binding.GDN_ERR_UNSUPPORTED
    assert call(B=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(Hqk=2, Hv=3) == binding.GDN_ERR_UNSUPPORTED
    assert call(dk=64) == binding.GDN_ERR_UNSUPPORTED
    assert call(dtype=3) == binding.GDN_ERR_INVALID_ARG
    assert call(ptr=None) == binding.GDN_ERR_INVALID_ARG
    assert call(S_new=None) == binding.GDN_ERR_INVALID_ARG
    assert call(ptr=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert call(steps=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert call(B=0) == binding.GDN_OK


def test_decode_slots_argument_checks(lib):
    def call(B=1, n_slots=4, Hqk=1, Hv=1, dk=128, dv=128, dtype=1, pool=FAKE, slots=FAKE, ptr=FAKE):
        return lib.gdn_decode_step_slots(ptr, FAKE, FAKE, FAKE, FAKE, pool, slots, FAKE,
                                         B, n_slots, Hqk, Hv, dk, dv, dtype, None)
    assert call(n_slots=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(B=-2) == binding.GDN_ERR_INVALID_ARG
    assert call(slots=None) == binding.GDN_ERR_INVALID_ARG
    assert call(pool=None) == binding.GDN_ERR_INVALID_ARG
    assert call(slots=ctypes.c_void_p(0x1002)) == binding.GDN_ERR_INVALID_ARG
    assert call(pool=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert call(Hqk=4, Hv=6) == binding.GDN_ERR_UNSUPPORTED
    assert call(dtype=9) == binding.GDN_ERR_INVALID_ARG
    assert call(B=0) == binding.GDN_OK


def test_chunk_varlen_argument_checks(lib):
    def call(N=2, T=64, Hqk=1, Hv=1, dk=128, dv=128, C=64, dtype=1, cu=FAKE, ptr=FAKE):
        return lib.gdn_chunk_fwd_varlen(ptr, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, cu,
                                        N, T, Hqk, Hv, dk, dv, C, dtype, None)
    assert call(cu=None) == binding.GDN_ERR_INVALID_ARG
    assert call(cu=ctypes.c_void_p(0x1002)) == binding.GDN_ERR_INVALID_ARG
    assert call(N=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(T=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(N=70000) == binding.GDN_ERR_UNSUPPORTED
    assert call(C=16) == binding.GDN_ERR_UNSUPPORTED
    assert call(Hqk=2, Hv=3) == binding.GDN_ERR_UNSUPPORTED
    assert call(ptr=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert call(N=0) == binding.GDN_OK
    assert call(T=0) == binding.GDN_OK          # every sequence empty, no S_final: nothing to do


def test_split_workspace_sizes(lib):
    hs = 128 * 128
    # B=1, T=4096, 48 heads, 2 segments of 2048 tokens: D (2 segments), M (1), R (2048
    # rows), S_start (1), each rounded up to 1 KiB
    need = binding.split_workspace_bytes(1, 4096, 48, segments=2)
    assert need == 2 * 48 * hs * 4 + 48 * hs * 4 + 2048 * 48 * 128 * 2 + 48 * hs * 2
    # whole chunks per segment: 385 tokens (7 chunks) in 3 segments of 3 chunks
    need3 = binding.split_workspace_bytes(2, 385, 6, segments=3)
    D = 2 * 3 * 6 * hs * 4
    M = 2 * 2 * 6 * hs * 4
    R = 2 * (385 - 192) * 6 * 128 * 2
    align = lambda x: (x + 1023) // 1024 * 1024   # noqa: E731
    assert need3 == align(align(align(align(D) + M) + R) + M // 2)
    assert binding.split_workspace_bytes(1, 64, 48, segments=4) == 0     # one chunk: no split
    assert binding.split_workspace_bytes(1, 4096, 48, segments=1) == 0
    assert binding.split_workspace_bytes(1, 4096, 48, segments=17) == 0
    assert lib.gdn_chunk_fwd_split_workspace(1, 4096, 48, 64, 128, 2) == 0


def test_split_argument_checks(lib):
    def call(segments=2, ws=FAKE, nbytes=1 << 40, dtype=1, ptr=FAKE):
        return lib.gdn_chunk_fwd_split(ptr, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                                       1, 4096, 16, 48, 128, 128, 64, segments, dtype, ws, nbytes, None)
    assert call(segments=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(segments=17) == binding.GDN_ERR_INVALID_ARG


def test_bwd_workspace_sizes(lib):
    # checkpoints every 16 tokens plus a 16-state scratch, per (sequence, head),
    # each state 128 x 128 fp32
    assert binding.bwd_workspace_bytes(1, 4096, 48) == 48 * (256 + 16) * 128 * 128 * 4
    assert binding.bwd_workspace_bytes(2, 17, 6) == 2 * 6 * (2 + 16) * 128 * 128 * 4
    assert binding.bwd_workspace_bytes(1, 0, 48) == 0
    assert lib.gdn_bwd_workspace(1, 64, 48, 64, 128) == 0


def test_bwd_argument_checks(lib):
    def call(B=1, T=64, Hqk=1, Hv=1, dk=128, dv=128, dtype=1, ptr=FAKE, dS0=FAKE, ws=FAKE,
             nbytes=1 << 40, out=FAKE):
        return lib.gdn_bwd(ptr, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, out, FAKE, FAKE, FAKE,
                           FAKE, dS0, B, T, Hqk, Hv, dk, dv, dtype, ws, nbytes, None)
    assert call(B=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(T=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(dtype=3) == binding.GDN_ERR_INVALID_ARG
    assert call(Hqk=2, Hv=3) == binding.GDN_ERR_UNSUPPORTED
    assert call(dk=64) == binding.GDN_ERR_UNSUPPORTED
    assert call(B=70000) == binding.GDN_ERR_UNSUPPORTED
    assert call(ptr=None) == binding.GDN_ERR_INVALID_ARG
    assert call(out=None) == binding.GDN_ERR_INVALID_ARG
    assert call(dS0=None) == binding.GDN_ERR_INVALID_ARG
    assert call(ptr=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert call(ws=None) == binding.GDN_ERR_INVALID_ARG
    assert call(nbytes=1024) == binding.GDN_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(0x1010)) == binding.GDN_ERR_INVALID_ARG   # not 256-byte aligned
    assert call(B=0) == binding.GDN_OK


def test_bwd_chunk_workspace_sizes(lib):
    # per (sequence, V head, chunk of 64): W, U, dU (64 x 128 bf16), T, P (64 x 64
    # bf16), S, dS' (128 x 128 bf16), b, gamma, g (64 fp32 each) and two fp32 sums; each array
    # 256-byte aligned
    per = 3 * 64 * 128 * 2 + 2 * 64 * 64 * 2 + 2 * 128 * 128 * 2 + 3 * 64 * 4
    assert binding.bwd_chunk_workspace_bytes(1, 4096, 48) == 48 * 64 * (per + 8)
    assert binding.bwd_chunk_workspace_bytes(2, 17, 6) == 12 * per + 256
    assert binding.bwd_chunk_workspace_bytes(1, 0, 48) == 0
    assert lib.gdn_bwd_chunk_workspace(1, 64, 48, 64, 128) == 0


def test_bwd_chunk_argument_checks(lib):
    def call(B=1, T=64, Hqk=1, Hv=1, dk=128, dv=128, dtype=1, ptr=FAKE, dS0=FAKE, ws=FAKE,
             nbytes=1 << 40, out=FAKE):
        return lib.gdn_bwd_chunk(ptr, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, out, FAKE, FAKE, FAKE,
                                 FAKE, dS0, B, T, Hqk, Hv, dk, dv, dtype, ws, nbytes, None)
    assert call(B=-1) == binding.GDN_ERR_INVALID_ARG
    assert call(dtype=3) == binding.GDN_ERR_INVALID_ARG
    assert call(dtype=0) == binding.GDN_ERR_UNSUPPORTED    # fp32 inputs: gdn_bwd
    assert call(Hqk=2, Hv=3) == binding.GDN_ERR_UNSUPPORTED
    assert call(dv=64) == binding.GDN_ERR_UNSUPPORTED
    assert call(B=70000) == binding.GDN_ERR_UNSUPPORTED
    assert call(ptr=None) == binding.GDN_ERR_INVALID_ARG
    assert call(out=None) == binding.GDN_ERR_INVALID_ARG
    assert call(dS0=None) == binding.GDN_ERR_INVALID_ARG
    assert call(ptr=MISALIGNED) == binding.GDN_ERR_INVALID_ARG
    assert call(ws=None) == binding.GDN_ERR_INVALID_ARG
    assert call(nbytes=1024) == binding.GDN_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(0x1010)) == binding.GDN_ERR_INVALID_ARG
    assert call(B=0) == binding.GDN_OK
