"""GPU parity of the backward pass (gdn_bwd, through the C ABI) against the fp64
backward oracle.

Bar: max|g_gpu - g_ref| <= tau * max|g_ref| for each of dq, dk, dv, dalpha,
dbeta, dS0, with tau = 1e-4.  The kernel computes in fp32 from the same input
values the oracle sees (bf16 inputs upcast exactly), so bf16 inputs have the
fp32 bar too; the atomically accumulated outputs differ from run to run only
in the order of an fp32 sum.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_attention_recurrence_07_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TAU = 1e-4
DEV = "cuda"
NAMES = ("dq", "dk", "dv", "dalpha", "dbeta", "dS0")


def problem(B, T, Hqk, Hv, dtype, seed, s0=True, dsf=True):
    d = inputs.prefill_inputs(B, T, Hqk, Hv, dtype=dtype, s0_std=0.3 if s0 else 0.0, seed=seed)
    if not s0:
        d["S0"] = None
    g = torch.Generator().manual_seed(seed + 1000)
    d["dO"] = torch.randn(B, T, Hv, 128, generator=g).to(dtype)
    d["dS_final"] = torch.randn(B, Hv, 128, 128, generator=g) * 0.1 if dsf else None
    return d


def run_bwd(d):
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
    binding.gdn_bwd(dd["q"], dd["k"], dd["v"], dd["alpha"], dd["beta"], dd["S0"], dd["dO"], dd["dS_final"],
                    out["dq"], out["dk"], out["dv"], out["dalpha"], out["dbeta"], out["dS0"])
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
        assert np.isfinite(got).all(), f"{what} {name}: non-finite values"
        assert err <= TAU, f"{what} {name}: {err:.3e} > {TAU}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("T", [1, 16, 77, 130])
def test_bwd_matches_oracle(dtype, T):
    """Ragged lengths around the 16-token checkpoint blocks, shared QK heads."""
    d = problem(2, T, 2, 6, dtype, seed=300 + T)
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    check_all(run_bwd(d), ref, f"{dtype} T={T}")


def test_bwd_without_state_inputs():
    d = problem(1, 45, 1, 3, torch.bfloat16, seed=7, s0=False, dsf=False)
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], None, None)
    check_all(run_bwd(d), ref, "no S0 / dS_final")


def test_bwd_empty_sequence():
    """T = 0: no token gradients; dS0 = dS_final (zeros without it)."""
    d = problem(2, 0, 1, 2, torch.bfloat16, seed=8)
    out = run_bwd(d)
    assert torch.equal(out["dS0"].cpu(), d["dS_final"])
    d["dS_final"] = None
    assert torch.count_nonzero(run_bwd(d)["dS0"]).item() == 0


def test_bwd_gates_at_the_ends():
    """alpha = 1 and alpha ~ 1e-30, beta = 0 on some tokens."""
    d = problem(1, 50, 1, 3, torch.float32, seed=9)
    d["alpha"][:, ::5, 0] = 1.0
    d["alpha"][:, 3::7, 1] = 1e-30
    d["beta"][:, ::4, 2] = 0.0
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d["S0"], d["dS_final"])
    check_all(run_bwd(d), ref, "gate ends")


def test_bwd_workload_one_head_group():
    """The bench workload (B=1, T=4096, 16 QK / 48 V heads): the QK head 0 and
    the V heads 0-2 that read it are checked against the oracle."""
    w = inputs.PREFILL_4K
    d = inputs.workload_inputs(w)
    g = torch.Generator().manual_seed(4242)
    d["dO"] = torch.randn(w.B, w.T, w.Hv, 128, generator=g).to(d["q"].dtype)
    d["dS_final"] = None
    out = run_bwd(d)
    ref = oracle.backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["dO"], d.get("S0"), None,
                          h_range=(0, 3))
    check_all(out, ref, "4K workload", heads=slice(0, 3), qk_heads=slice(0, 1))
