"""GPU parity of gdn_chunk_fwd_pipelined (WY preparation on SMs of its own, state
chains on others, one cooperative launch) against the fp64 CPU oracle, through
the C ABI.  Bar: max|x_gpu - x_ref| <= 2e-2 * max|x_ref| for o and S_final
(bf16 inputs, fp32 state).  Also: agreement with the one-CTA tensor-core kernel,
several heads per chain CTA (waves), and a bounded wait made to give up."""
import numpy as np
import pytest
import torch

import oracle
from conftest import record_parity
from linear_attention_recurrence_07_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TAU_BF16 = 2e-2
DEV = "cuda"


def rel_err(got, ref):
    got = got.detach().double().cpu().numpy() if hasattr(got, "detach") else got
    ref = ref.detach().double().cpu().numpy() if hasattr(ref, "detach") else ref
    return float(np.abs(got - ref).max()) / max(float(np.abs(ref).max()), 1e-300)


def check(got, ref, tau, what):
    e = rel_err(got, ref)
    print(f"{what}: max rel err {e:.3e} (tau {tau})")
    record_parity(what, e, tau)
    assert e <= tau, f"{what}: max|err| / max|ref| = {e:.3e} > {tau}"


def run_pipe(d, chain_ctas=0, wait_limit_cycles=0):
    B, T, Hqk, dk = d["q"].shape
    Hv = d["v"].shape[2]
    o = torch.full_like(d["v"], float("nan"))
    S = torch.full((B, Hv, dk, dk), float("nan"), device=DEV)
    binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S,
                                    chain_ctas=chain_ctas, wait_limit_cycles=wait_limit_cycles)
    torch.cuda.synchronize()
    return o, S


def small(B, T, Hqk, Hv, seed, s0=0.02):
    return inputs.prefill_inputs(B, T, Hqk, Hv, dtype=torch.bfloat16, s0_std=s0, seed=seed,
                                 device=DEV)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 385])
def test_pipelined_small_against_oracle(T):
    d = small(1, T, 2, 6, 100 + T)
    o, S = run_pipe(d)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(o, o_ref, TAU_BF16, f"T={T} o")
    check(S, S_ref, TAU_BF16, f"T={T} S_final")
    assert binding.device_status() == "GDN_OK"


@pytest.mark.parametrize("chain_ctas", [3, 6])
def test_pipelined_several_heads_per_chain(chain_ctas):
    """B=2, 6 V heads: 12 states on 3 (or 6) chain CTAs, so each chain CTA carries
    four (or two) heads one after the other, each from its own S0."""
    d = small(2, 385, 2, 6, 7)
    o, S = run_pipe(d, chain_ctas=chain_ctas)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S_final")


@pytest.mark.parametrize("Hqk,Hv", [(4, 4), (2, 8)])
def test_pipelined_group_sizes(Hqk, Hv):
    """One V head per QK head (two prep warpgroups idle) and four per QK head (one
    prep warpgroup serves two of them)."""
    d = small(1, 200, Hqk, Hv, 11)
    o, S = run_pipe(d)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S_final")


def test_pipelined_strong_and_no_decay():
    """Gates at their ends: alpha = 1 and alpha = 1e-30 heads, beta = 1.5 and 0."""
    d = small(1, 256, 2, 6, 5)
    d["alpha"][:, :, 0] = 1.0
    d["alpha"][:, :, 1] = 1e-30
    d["beta"][:, :, 2] = 1.5
    d["beta"][:, :, 3] = 0.0
    o, S = run_pipe(d)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S_final")


def test_pipelined_model_dims_workload():
    """B=1, T=4096, 16/48 heads (the bench workload): every output against the
    oracle, and against the one-CTA tensor-core kernel (the same products, rounded
    to bf16 at slightly different points, e.g. gamma applied to the fp32 S-part of
    O here and to the bf16 Q operand there, so they agree to a few bf16 ulp)."""
    w = inputs.PREFILL_4K
    d = inputs.workload_inputs(w, device=DEV)
    o, S = run_pipe(d)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S_final")
    with binding.prefill_kernel("tc"):
        o1, S1 = binding.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    torch.cuda.synchronize()
    check(o, o1.double().cpu().numpy(), 2 ** -6, "o vs one-CTA kernel")
    check(S, S1.double().cpu().numpy(), 2 ** -6, "S_final vs one-CTA kernel")


def test_pipelined_in_place_state():
    """S_final may be S0 (each head's S0 is read before its final state is written)."""
    d = small(2, 130, 2, 6, 3)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    S = d["S0"].clone()
    o = torch.empty_like(d["v"])
    binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S, o, S,
                                    chain_ctas=3)
    torch.cuda.synchronize()
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S_final (in place)")


def test_pipelined_workspace_checks():
    d = small(1, 64, 2, 6, 1)
    need = binding.pipelined_workspace_bytes(1, 2, 6)
    assert need > 0
    o = torch.empty_like(d["v"])
    small_ws = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(binding.GdnError, match="INVALID_ARG"):
        binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], None, o, None,
                                        workspace=small_ws)


def test_pipelined_wait_gives_up_and_device_recovers():
    """A wait limit far below the time the first chunk's preparation takes: the
    chains' first waits give up, every CTA stops, the call is reported as
    GDN_ERR_TIMEOUT by gdn_device_status, and the next normal call is correct."""
    d = small(1, 4096, 2, 6, 9)
    run_pipe(d, wait_limit_cycles=2000)
    assert binding.device_status() == "GDN_ERR_TIMEOUT"
    assert binding.device_status() == "GDN_OK"        # read and cleared
    o, S = run_pipe(d)
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(o, o_ref, TAU_BF16, "o after the timed-out call")
    check(S, S_ref, TAU_BF16, "S_final after the timed-out call")
    assert binding.device_status() == "GDN_OK"


@pytest.mark.parametrize("shape", [(1, 4096, 16, 48, 0), (2, 385, 2, 6, 3)], ids=["model-dims", "4-heads-per-chain"])
def test_pipelined_repeated_calls_identical(shape):
    """The kernel fixes the order of every reduction, so repeated calls on the same
    inputs must agree bit for bit; a missed wait between its roles (a tile read
    before it has landed, a buffer reused before it is read) shows up as calls that
    differ.  Eight calls each, plus the first against the oracle."""
    B, T, Hqk, Hv, cc = shape
    d = small(B, T, Hqk, Hv, 21)
    outs = [run_pipe(d, chain_ctas=cc) for _ in range(8)]
    for i, (o, S) in enumerate(outs[1:], 1):
        assert torch.equal(o, outs[0][0]), f"call {i}: o differs from call 0"
        assert torch.equal(S, outs[0][1]), f"call {i}: S_final differs from call 0"
    o_ref, S_ref = oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"])
    check(outs[0][0], o_ref, TAU_BF16, "o")
    check(outs[0][1], S_ref, TAU_BF16, "S_final")
