"""GPU parity of the chunkwise backward (gdn_bwd_chunk, through the C ABI) against
the fp64 backward oracle.

Bar: max|g_gpu - g_ref| <= tau * max|g_ref| for each of dq, dk, dv, dalpha,
dbeta, dS0 with tau = 2e-2, the forward's bar for bf16 inputs: the kernels take
bf16 operands (inputs, and the chunk start states, U, W, T, dU and dS' they keep
between launches) into fp32-accumulating MMAs.  The outputs carry no atomics, so
repeated calls agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import record_parity
from linear_attention_recurrence_07_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TAU = 2e-2
DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


def problem(B, T, Hqk, Hv, seed, s0=True, dsf=True):
    d = inputs.prefill_inputs(B, T, Hqk, Hv, dtype=torch.bfloat16, s0_std=0.3 if s0 else 0.0, seed=seed)
    if not s0:
        d["S0"] = None
    g = torch.Generator().manual_seed(seed + 1000)
    d["dO"] = torch.randn(B, T, Hv, 128, generator=g).to(torch.bfloat16)
    d["dS_final"] = torch.randn(B, Hv, 128, 128, generator=g) * 0.1 if dsf else None
    return d


def run(d, workspace=None):
    dd = {k: (None if v is None else v.to(DEV)) for k, v in d.items()}
    B, T, Hqk, _ = dd["q"].shape
    Hv = dd["v"].shape[2]
    f32 = dict(dtype=torch.float32, device=DEV)
    out = dict(dq=torch.full((B, T, Hqk, 128), float("nan"), **f32),
               dk=torch.full((B, T, Hqk, 128), float("nan"), **f32),
               dv=torch.full((B, T, Hv, 128), float("nan"), **f32),
               dalpha=torch.full((B, T, Hv), float("nan"), **f32),
               dbeta=torch.full((B, T, Hv), float("nan"), **f32),
               dS0=torch.full((B, Hv, 128, 128), float("nan"), **f32))
    binding.gdn_bwd_chunk(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"], dd["S0"], dd["dO"],
                          dd["dS_final"], out["dq"], out["dk"], out["dv"], out["dalpha"], out["dbeta"],
                          out["dS0"], workspace=workspace)
    torch.cuda.synchronize()
    return out


def check_all(out, ref, what, heads=None, qk_heads=None):
    for name, r in zip(NAMES, ref):
        got = out[name].double().cpu().numpy()
        if name in ("dq", "dk") and qk_heads is not None:
            got, r = got[:, :, qk_heads], r[:, :, qk_heads]
        elif name in ("dv", "dalpha", "dbeta", "dS0") and heads is not None:
            got, r = (got[:, :, heads], r[:, :, heads]) if name != "dS0" else (got[:, heads], r[:, heads])
        scale = max(float(np.abs(r).max()), 1e-300)
        err = float(np.abs(got - r).max()) / scale
        print(f"{what} {name}: max rel err {err:.3e}")
        record_parity(f"{what} {name}", err, TAU)
        assert np.isfinite(got).all(), f"{what} {name}: non-finite values"
        assert err <= TAU, f"{what} {name}: {err:.3e} > {TAU}"


@pytest.mark.parametrize("T", [1, 64, 77, 130, 200])
def test_bwd_chunk_matches_oracle(T):
    """Ragged and whole chunks, several chunks, shared QK heads, S0 and dS_final."""
    d = problem(2, T, 2, 6, seed=700 + T)
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    check_all(run(d), ref, f"T={T}")


def test_bwd_chunk_without_state_inputs():
    d = problem(1, 100, 1, 3, seed=17, s0=False, dsf=False)
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], None, None)
    check_all(run(d), ref, "no S0 / dS_final")


def test_bwd_chunk_gates_at_the_ends():
    """alpha = 1 on some tokens, beta = 0 on others, small alpha on a third set."""
    d = problem(1, 150, 1, 3, seed=19)
    d["alpha"][:, ::5, 0] = 1.0
    d["alpha"][:, 3::7, 1] = 1e-3
    d["beta"][:, ::4, 2] = 0.0
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    check_all(run(d), ref, "gate ends")


def test_bwd_chunk_empty_sequence():
    d = problem(2, 0, 1, 2, seed=8)
    out = run(d)
    assert torch.equal(out["dS0"].cpu(), d["dS_final"])
    d["dS_final"] = None
    assert torch.count_nonzero(run(d)["dS0"]).item() == 0


def test_bwd_chunk_repeated_calls_identical():
    d = problem(1, 300, 2, 6, seed=23)
    a, b = run(d), run(d)
    for name in NAMES:
        assert torch.equal(a[name], b[name]), name


def test_bwd_chunk_workload_two_head_groups():
    """The bench workload (B=1, T=4096, 16 QK / 48 V heads) in one call: QK heads 0
    and 15 and the V heads 0-2 and 45-47 that read them against the oracle."""
    w = inputs.PREFILL_4K
    d = inputs.workload_inputs(w)
    g = torch.Generator().manual_seed(4242)
    d["dO"] = torch.randn(w.B, w.T, w.Hv, 128, generator=g).to(d["q"].dtype)
    d["dS_final"] = torch.randn(w.B, w.Hv, 128, 128, generator=g) * 0.1
    need = binding.bwd_chunk_workspace_bytes(w.B, w.T, w.Hv)
    out = run(d, workspace=torch.empty(need, dtype=torch.uint8, device=DEV))
    for h0, hq in ((0, 0), (45, 15)):
        ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d.get("S0"),
                              d["dS_final"], h_range=(h0, h0 + 3))
        check_all(out, ref, f"4K workload h={h0}", heads=slice(h0, h0 + 3), qk_heads=slice(hq, hq + 1))
