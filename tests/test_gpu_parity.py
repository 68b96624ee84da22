"""GPU parity of libgdn.so against the fp64 CPU oracle, called through the C ABI.

Bar (stated for the method): max|x_gpu - x_ref| <= tau * max|x_ref| over the whole
tensor, for o and for the final state, with tau = 1e-4 for fp32 inputs and
tau = 2e-2 for bf16 inputs with an fp32 state.  Inputs come from the seeded
generators in ``linear_attention_recurrence_07_b200.inputs``; the oracle sees the
exact values the GPU sees (bf16 upcast exactly to fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import record_parity
from linear_attention_recurrence_07_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TAU_F32 = 1e-4
TAU_BF16 = 2e-2
DEV = "cuda"


def tau_for(dtype):
    return TAU_F32 if dtype == torch.float32 else TAU_BF16


def rel_err(got, ref):
    got = got.detach().double().cpu().numpy() if hasattr(got, "detach") else got
    scale = float(np.abs(ref).max())
    return float(np.abs(got - ref).max()) / max(scale, 1e-300)


def check(got, ref, tau, what):
    e = rel_err(got, ref)
    print(f"{what}: max rel err {e:.3e} (tau {tau})")
    record_parity(what, e, tau)
    assert e <= tau, f"{what}: max|err| / max|ref| = {e:.3e} > {tau}"


def to_dev(d):
    return {k: (None if v is None else v.to(DEV)) for k, v in d.items()}


# Prefill kernels a bf16 input can run on; fp32 inputs always take "simt".
BF16_KERNELS = ["tc", "simt"]
TC_KERNELS = ["tc"]


def kernels_for(dtype):
    return BF16_KERNELS if dtype == torch.bfloat16 else ["simt"]


def run_chunk(d, chunk=64, kernel="auto"):
    with binding.prefill_kernel(kernel):
        o, S = binding.chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"],
                                 chunk=chunk)
    torch.cuda.synchronize()
    return o, S


def oracle_ref(d, h_range=None):
    return oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], h_range=h_range)


# ----------------------------------------------------------------------------- prefill
def test_prefill_small_fp32_workload():
    """B=1, T=256, Hqk=2, Hv=6, fp32 end to end, tau = 1e-4."""
    w = inputs.PREFILL_SMALL_FP32
    d = inputs.workload_inputs(w)
    o, S = run_chunk(to_dev(d))
    o_ref, S_ref = oracle_ref(d)
    check(o, o_ref, TAU_F32, "o")
    check(S, S_ref, TAU_F32, "S_final")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 100, 191, 256, 385])
def test_prefill_ragged_lengths(T, dtype):
    """1 to 7 chunks with ragged tails: the cluster kernel's two helpers get 0..4
    chunks each and reuse their receive slots from the third chunk on."""
    d = inputs.prefill_inputs(2, T, 2, 6, dtype=dtype, s0_std=0.5, seed=100 + T)
    o_ref, S_ref = oracle_ref(d)
    dd = to_dev(d)
    for kernel in kernels_for(dtype):
        o, S = run_chunk(dd, kernel=kernel)
        check(o, o_ref, tau_for(dtype), f"{kernel} o T={T}")
        check(S, S_ref, tau_for(dtype), f"{kernel} S_final T={T}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_prefill_one_v_head_per_qk_head(dtype):
    d = inputs.prefill_inputs(3, 130, 3, 3, dtype=dtype, s0_std=0.1, seed=7)
    o_ref, S_ref = oracle_ref(d)
    dd = to_dev(d)
    for kernel in kernels_for(dtype):
        o, S = run_chunk(dd, kernel=kernel)
        check(o, o_ref, tau_for(dtype), f"{kernel} o")
        check(S, S_ref, tau_for(dtype), f"{kernel} S_final")


@pytest.mark.parametrize("kernel", TC_KERNELS)
def test_prefill_tc_kernels_beyond_one_wave(kernel):
    """More (sequence, V head) pairs than the GPU holds at once (B=7, Hv=48: 336
    CTAs): later waves reuse SMs and TMEM of finished ones."""
    d = to_dev(inputs.prefill_inputs(7, 130, 16, 48, dtype=torch.bfloat16, s0_std=0.1, seed=11))
    o, S = run_chunk(d, kernel=kernel)
    o_a, S_a = run_chunk(d, kernel="simt")
    for b, (h0, h1) in [(0, (0, 3)), (6, (45, 48))]:
        o_ref, S_ref = oracle_ref({k: (None if v is None else v.cpu()) for k, v in
                                   _sub_problem(d, b, h0, h1, 48, 16).items()})
        check(o[b:b + 1, :, h0:h1], o_ref, TAU_BF16, f"{kernel} o b={b} h={h0}:{h1}")
        check(S[b:b + 1, h0:h1], S_ref, TAU_BF16, f"{kernel} S_final b={b} h={h0}:{h1}")
    # every pair against the CUDA-core kernel (same inputs, a different evaluation)
    assert (o.float() - o_a.float()).abs().max().item() <= TAU_BF16 * o_a.float().abs().max().item()
    assert (S - S_a).abs().max().item() <= TAU_BF16 * S_a.abs().max().item()


@pytest.mark.parametrize("B,T,Hqk,Hv,seed", [(1, 385, 2, 6, 21), (2, 4096, 16, 48, 22)])
def test_prefill_tc_kernels_agree(B, T, Hqk, Hv, seed):
    """The one-CTA and the pipelined tensor-core kernels round the decay factors
    into their bf16 operands at different points: the one-CTA kernel rounds
    U^T diag(g) for the state update, the pipelined one rounds K~ = diag(g) K.
    Each of those roundings is one bf16 ulp (2^-8 relative), so the two agree to
    a few ulp of the largest value."""
    d = to_dev(inputs.prefill_inputs(B, T, Hqk, Hv, dtype=torch.bfloat16, s0_std=0.3, seed=seed))
    o1, S1 = run_chunk(d, kernel="tc")
    o2 = torch.empty_like(o1)
    S2 = torch.empty_like(S1)
    binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o2, S2)
    torch.cuda.synchronize()
    err_s = (S1 - S2).abs().max().item()
    assert err_s <= 2 ** -6 * S2.abs().max().item(), err_s
    err = (o1.float() - o2.float()).abs().max().item()
    assert err <= 2 ** -6 * o2.float().abs().max().item(), err


def test_prefill_strong_and_no_decay():
    """Gates at the ends of their range: alpha = 1 (no forgetting) on some heads,
    alpha ~ 1e-30 (near-total forgetting) on others; beta outside (0, 1) too."""
    d = inputs.prefill_inputs(1, 200, 2, 4, dtype=torch.float32, s0_std=1.0, seed=9)
    d["alpha"][:, :, 0] = 1.0
    d["alpha"][:, 50:60, 1] = 1e-30
    d["beta"][:, :, 2] = 1.5
    d["beta"][:, :, 3] = 0.0
    o, S = run_chunk(to_dev(d))
    o_ref, S_ref = oracle_ref(d)
    check(o, o_ref, TAU_F32, "o")
    check(S, S_ref, TAU_F32, "S_final")


def test_prefill_model_dims_workload():
    """B=1, T=4096, Hqk=16, Hv=48, bf16 inputs, fp32 state: every output checked,
    for the default kernel choice and each tensor-core kernel."""
    w = inputs.PREFILL_4K
    d = inputs.workload_inputs(w, device=DEV)
    o_ref, S_ref = oracle_ref(d)
    for kernel in ["auto"] + TC_KERNELS:
        o, S = run_chunk(d, kernel=kernel)
        check(o, o_ref, TAU_BF16, f"{kernel} o")
        check(S, S_ref, TAU_BF16, f"{kernel} S_final")


def _sub_problem(d, b, h0, h1, Hv, Hqk):
    """Inputs of sequence b and V heads [h0, h1) (inside one QK group) as a
    standalone problem with one QK head."""
    g = Hv // Hqk
    hq = h0 // g
    assert (h1 - 1) // g == hq
    sl = lambda x: x[b:b + 1]  # noqa: E731
    return dict(q=sl(d["q"])[:, :, hq:hq + 1], k=sl(d["k"])[:, :, hq:hq + 1],
                v=sl(d["v"])[:, :, h0:h1], alpha=sl(d["alpha"])[:, :, h0:h1],
                beta=sl(d["beta"])[:, :, h0:h1],
                S0=None if d["S0"] is None else sl(d["S0"])[:, h0:h1])


def test_prefill_batched_workload_sampled():
    """B=8, T=8192, nonzero S0: the full launch on the GPU; the oracle checks the
    first and last sequence on the first and last QK group (all their tokens)."""
    w = inputs.PREFILL_BATCH8_8K
    d = inputs.workload_inputs(w, device=DEV)
    outs = {kernel: run_chunk(d, kernel=kernel) for kernel in ["auto"]}
    o = torch.empty_like(d["v"])
    S = torch.empty_like(d["S0"])
    binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S)
    torch.cuda.synchronize()
    outs["pipelined"] = (o, S)
    for b, (h0, h1) in [(0, (0, 3)), (7, (45, 48)), (3, (21, 24))]:
        o_ref, S_ref = oracle_ref(_sub_problem(d, b, h0, h1, w.Hv, w.Hqk))
        for kernel, (o, S) in outs.items():
            check(o[b:b + 1, :, h0:h1], o_ref, TAU_BF16, f"{kernel} o b={b} h={h0}:{h1}")
            check(S[b:b + 1, h0:h1], S_ref, TAU_BF16, f"{kernel} S_final b={b} h={h0}:{h1}")


@pytest.mark.timeout(1800)
def test_prefill_long_context_workload_sampled():
    """B=1, T=262144 with long-memory gates: the full launch on the GPU; the oracle
    follows two V heads (first and last) through all 262,144 tokens, which also
    measures the drift of the fp32 state carried across 4096 chunks."""
    w = inputs.PREFILL_256K
    d = inputs.workload_inputs(w, device=DEV)
    outs = {kernel: run_chunk(d, kernel=kernel) for kernel in TC_KERNELS}
    outs["split"] = run_split(d)
    o = torch.empty_like(d["v"])
    S = torch.empty((w.B, w.Hv, w.dk, w.dv), device=DEV)
    binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S)
    torch.cuda.synchronize()
    outs["pipelined"] = (o, S)
    for h in (0, 47):
        o_ref, S_ref = oracle_ref(_sub_problem(d, 0, h, h + 1, w.Hv, w.Hqk))
        for kernel, (o, S) in outs.items():
            check(o[:, :, h:h + 1], o_ref, TAU_BF16, f"{kernel} o h={h}")
            check(S[:, h:h + 1], S_ref, TAU_BF16, f"{kernel} S_final h={h}")


def test_prefill_empty_sequence_copies_state():
    d = to_dev(inputs.prefill_inputs(2, 0, 2, 4, s0_std=1.0, seed=3))
    o, S = run_chunk(d)
    assert o.shape[1] == 0
    assert torch.equal(S, d["S0"])
    # and without S0 the final state is zero
    d["S0"] = None
    _, S = run_chunk(d)
    assert torch.count_nonzero(S) == 0


def test_prefill_in_place_state():
    d = to_dev(inputs.prefill_inputs(2, 100, 2, 4, s0_std=0.3, seed=4))
    o_ref, S_ref = run_chunk(d)
    S = d["S0"].clone()
    o = torch.empty_like(o_ref)
    binding.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S, o, S)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(S, S_ref)


@pytest.mark.parametrize("dtype,kernel", [(torch.bfloat16, "tc"), (torch.float32, "simt")],
                         ids=["bf16-tc", "fp32-simt"])
def test_prefill_split_invariance(dtype, kernel):
    """T1 tokens, then T2 tokens from the saved state, equals one call over T1+T2."""
    d = to_dev(inputs.prefill_inputs(2, 300, 2, 6, dtype=dtype, s0_std=0.2, seed=5))
    o, S = run_chunk(d, kernel=kernel)
    T1 = 130
    first = {k: (v[:, :T1].contiguous() if k != "S0" else v) for k, v in d.items()}
    second = {k: (v[:, T1:].contiguous() if k != "S0" else v) for k, v in d.items()}
    o1, S1 = run_chunk(first, kernel=kernel)
    second["S0"] = S1
    o2, S2 = run_chunk(second, kernel=kernel)
    scale_o = o.abs().max().item()
    tol = 1e-5 if dtype == torch.float32 else 1e-2
    assert (torch.cat([o1, o2], 1).float() - o.float()).abs().max().item() <= tol * scale_o
    assert (S2 - S).abs().max().item() <= tol * S.abs().max().item()


def test_prefill_column_permutation_equivariance():
    d = to_dev(inputs.prefill_inputs(1, 96, 1, 2, dtype=torch.float32, s0_std=0.2, seed=6))
    perm = torch.randperm(128, generator=torch.Generator().manual_seed(0)).to(DEV)
    o, S = run_chunk(d)
    dp = dict(d)
    dp["v"] = d["v"][..., perm].contiguous()
    dp["S0"] = d["S0"][..., perm].contiguous()
    o_p, S_p = run_chunk(dp)
    assert (o_p - o[..., perm]).abs().max().item() <= 1e-6 * o.abs().max().item()
    assert (S_p - S[..., perm]).abs().max().item() <= 1e-6 * S.abs().max().item()


def test_prefill_rejects_misaligned_pointer():
    d = to_dev(inputs.prefill_inputs(1, 8, 1, 1, dtype=torch.float32, seed=8))
    flat = torch.empty(d["q"].numel() + 1, device=DEV)
    q_off = flat[1:].view_as(d["q"])            # contiguous but 4 bytes off alignment
    q_off.copy_(d["q"])
    with pytest.raises(binding.GdnError, match="INVALID_ARG"):
        binding.chunk_fwd(q_off, d["k"], d["v"], d["alpha"], d["beta"], None)


# ----------------------------------------------------------------------------- decode
def decode_run(w, steps, B=None, dtype=None):
    """Runs `steps` decode steps on the GPU (state in place) and returns the per-step
    outputs, the final state and the host copies of every step's inputs."""
    B = B if B is not None else w.B
    S = inputs.decode_state(w, device=DEV, B=B)
    S0 = S.clone()
    outs, ins = [], []
    for s in range(steps):
        x = inputs.decode_inputs(w, s, device=DEV, B=B)
        if dtype is not None:
            x = {k: (v.to(dtype) if v.dtype == torch.bfloat16 else v) for k, v in x.items()}
        outs.append(binding.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S))
        ins.append(x)
    torch.cuda.synchronize()
    return torch.stack(outs, 1), S, S0, ins


def stacked(ins, key, seqs):
    return torch.stack([x[key][seqs] for x in ins], 1)


def test_decode_workload_all_sequences_first_steps():
    """B=256, Hqk=16, Hv=48: 8 steps, every sequence and head against the oracle
    run as one 8-token recurrence per (sequence, head)."""
    w = inputs.DECODE_B256
    o, S, S0, ins = decode_run(w, 8)
    seqs = slice(None)
    o_ref, S_ref = oracle.forward(stacked(ins, "q", seqs), stacked(ins, "k", seqs),
                                  stacked(ins, "v", seqs), stacked(ins, "alpha", seqs),
                                  stacked(ins, "beta", seqs), S0)
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S")


@pytest.mark.timeout(1800)
def test_decode_workload_1000_steps_sampled():
    """The full 1000 decode steps at B=256; the oracle follows 8 sequences (all 48
    heads) through all steps with its own fp64 state."""
    w = inputs.DECODE_B256
    o, S, S0, ins = decode_run(w, w.decode_steps)
    seqs = torch.tensor([0, 1, 63, 100, 128, 200, 254, 255], device=DEV)
    o_ref, S_ref = oracle.forward(stacked(ins, "q", seqs), stacked(ins, "k", seqs),
                                  stacked(ins, "v", seqs), stacked(ins, "alpha", seqs),
                                  stacked(ins, "beta", seqs), S0[seqs])
    check(o[seqs], o_ref, TAU_BF16, "o")
    check(S[seqs], S_ref, TAU_BF16, "S")


def test_decode_fp32():
    w = inputs.DECODE_B256
    o, S, S0, ins = decode_run(w, 5, B=4, dtype=torch.float32)
    seqs = slice(None)
    o_ref, S_ref = oracle.forward(stacked(ins, "q", seqs), stacked(ins, "k", seqs),
                                  stacked(ins, "v", seqs), stacked(ins, "alpha", seqs),
                                  stacked(ins, "beta", seqs), S0)
    check(o, o_ref, TAU_F32, "o")
    check(S, S_ref, TAU_F32, "S")


def test_decode_steps_equal_one_prefill():
    """T decode calls reproduce one gdn_chunk_fwd over the same T tokens."""
    d = to_dev(inputs.prefill_inputs(2, 70, 2, 6, dtype=torch.float32, s0_std=0.3, seed=11))
    o_c, S_c = run_chunk(d)
    S = d["S0"].clone()
    outs = []
    for t in range(70):
        outs.append(binding.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                        d["v"][:, t].contiguous(), d["alpha"][:, t].contiguous(),
                                        d["beta"][:, t].contiguous(), S))
    o_d = torch.stack(outs, 1)
    torch.cuda.synchronize()
    assert (o_d - o_c).abs().max().item() <= 1e-5 * o_c.abs().max().item()
    assert (S - S_c).abs().max().item() <= 1e-5 * S_c.abs().max().item()


def test_decode_out_of_place_leaves_input_state():
    w = inputs.DECODE_B256
    S = inputs.decode_state(w, device=DEV, B=3)
    S_keep = S.clone()
    x = inputs.decode_inputs(w, 0, device=DEV, B=3)
    S_new = torch.empty_like(S)
    o = torch.empty_like(x["v"])
    binding.gdn_decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, o, S_new)
    S_in = S.clone()
    o2 = binding.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S_in)
    torch.cuda.synchronize()
    assert torch.equal(S, S_keep)
    assert torch.equal(S_new, S_in)
    assert torch.equal(o, o2)


# ----------------------------------------------------------------------------- multi-token decode
def decode_tokens_run(d, with_steps=True):
    B, n, Hqk, dk = d["q"].shape
    Hv = d["v"].shape[2]
    o = torch.empty_like(d["v"])
    S_new = torch.empty_like(d["S0"])
    steps = torch.empty((B, n, Hv, dk, dk), dtype=torch.float32, device=DEV) if with_steps else None
    binding.gdn_decode_tokens(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S_new, steps)
    torch.cuda.synchronize()
    return o, S_new, steps


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("n", [1, 2, 5, 8])
def test_decode_tokens_against_oracle(n, dtype):
    """n tokens per call: outputs, the final state and the state after every token
    (for rollback) against the oracle run over the first t+1 tokens."""
    d = inputs.prefill_inputs(3, n, 2, 6, dtype=dtype, s0_std=0.05, seed=300 + n)
    o, S_new, steps = decode_tokens_run(to_dev(d))
    o_ref, S_ref = oracle_ref(d)
    check(o, o_ref, tau_for(dtype), f"o n={n}")
    check(S_new, S_ref, tau_for(dtype), f"S_new n={n}")
    for t in range(n):
        pre = {k: (v if k == "S0" else v[:, :t + 1]) for k, v in d.items()}
        _, S_t = oracle_ref(pre)
        check(steps[:, t], S_t, tau_for(dtype), f"S_steps[{t}] n={n}")


def test_decode_tokens_one_token_is_decode_step():
    w = inputs.DECODE_B256
    S = inputs.decode_state(w, device=DEV, B=5)
    x = inputs.decode_inputs(w, 0, device=DEV, B=5)
    o1 = torch.empty_like(x["v"])
    S1 = torch.empty_like(S)
    binding.gdn_decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, o1, S1)
    o2 = torch.empty_like(x["v"])[:, None].contiguous()
    S2 = torch.empty_like(S)
    binding.gdn_decode_tokens(x["q"][:, None].contiguous(), x["k"][:, None].contiguous(),
                              x["v"][:, None].contiguous(), x["alpha"][:, None].contiguous(),
                              x["beta"][:, None].contiguous(), S, o2, S2)
    torch.cuda.synchronize()
    assert torch.equal(o2[:, 0], o1)
    assert torch.equal(S2, S1)


def test_decode_tokens_in_place_and_workload_sampled():
    """B=256, n=4 at model dims, state updated in place; 6 sequences (all heads)
    against the oracle, and the in-place result equal to the out-of-place one."""
    w = inputs.VERIFY_B256_N4
    d = to_dev(inputs.workload_inputs(w))
    o, S_new, steps = decode_tokens_run(d)
    S_in = d["S0"].clone()
    o2 = torch.empty_like(o)
    binding.gdn_decode_tokens(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S_in, o2, S_in)
    torch.cuda.synchronize()
    assert torch.equal(o2, o) and torch.equal(S_in, S_new)
    assert torch.equal(steps[:, -1], S_new)
    seqs = [0, 1, 77, 128, 254, 255]
    sub = {k: v[seqs].cpu() for k, v in d.items()}
    o_ref, S_ref = oracle_ref(sub)
    check(o[seqs], o_ref, TAU_BF16, "o")
    check(S_new[seqs], S_ref, TAU_BF16, "S_new")


# ----------------------------------------------------------------------------- slot-indexed decode
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_decode_slots_against_oracle(dtype):
    """States gathered from a pool by slot; padding entries (-1, out of range) are
    skipped; pool rows that no sequence names are left untouched."""
    w = inputs.DECODE_B256
    n_slots, B = 10, 6
    pool = inputs.decode_state(w, device=DEV, B=n_slots)
    pool0 = pool.clone()
    x = inputs.decode_inputs(w, 3, device=DEV, B=B)
    if dtype == torch.float32:
        x = {k: v.float() for k, v in x.items()}
    slots = torch.tensor([3, -1, 7, 0, 12, 5], dtype=torch.int32, device=DEV)
    o = torch.full_like(x["v"], 7.0)
    binding.gdn_decode_step_slots(x["q"], x["k"], x["v"], x["alpha"], x["beta"], pool, slots, o)
    torch.cuda.synchronize()
    live = [0, 2, 3, 5]
    sl = [3, 7, 0, 5]
    o_ref, S_ref = oracle.decode_step(*(x[k][live].cpu() for k in ("q", "k", "v", "alpha", "beta")),
                                      pool0[sl].cpu())
    check(o[live], o_ref, tau_for(dtype), "o")
    check(pool[sl], S_ref, tau_for(dtype), "pool")
    assert torch.all(o[[1, 4]] == 7.0)                       # padding rows untouched
    untouched = [i for i in range(n_slots) if i not in sl]
    assert torch.equal(pool[untouched], pool0[untouched])
    # the same as gdn_decode_step on the gathered states
    S_g = pool0[sl].clone()
    o_g = binding.decode_step(*(x[k][live] for k in ("q", "k", "v", "alpha", "beta")), S_g)
    torch.cuda.synchronize()
    assert torch.equal(o_g, o[live]) and torch.equal(S_g, pool[sl])


# ----------------------------------------------------------------------------- packed (varlen) prefill
def run_varlen(d, kernel="auto"):
    T, Hv, dv = d["v"].shape
    N = d["cu_seqlens"].shape[0] - 1
    o = torch.empty_like(d["v"])
    S = torch.empty((N, Hv, d["q"].shape[2], dv), dtype=torch.float32, device=DEV)
    with binding.prefill_kernel(kernel):
        binding.gdn_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S,
                                     d["cu_seqlens"])
    torch.cuda.synchronize()
    return o, S


def varlen_oracle(d, n):
    """The oracle on sequence n of packed inputs d (host tensors), as a B=1 problem."""
    cu = d["cu_seqlens"].tolist()
    a, b = cu[n], cu[n + 1]
    sub = dict(q=d["q"][None, a:b], k=d["k"][None, a:b], v=d["v"][None, a:b],
               alpha=d["alpha"][None, a:b], beta=d["beta"][None, a:b],
               S0=None if d["S0"] is None else d["S0"][n:n + 1])
    return oracle_ref(sub)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_prefill_varlen_against_oracle(dtype):
    """Sequences of 0, 1, 63, 64, 65, 130, 7 and 200 tokens packed back to back:
    every sequence against the oracle, for every kernel that takes the dtype.
    Rows of the next sequence share a chunk with a sequence's tail."""
    lengths = [0, 1, 63, 64, 65, 130, 7, 200]
    d = inputs.varlen_inputs(lengths, 2, 6, dtype=dtype, s0_std=0.3, seed=41)
    dd = to_dev(d)
    refs = [varlen_oracle(d, n) for n in range(len(lengths))]
    cu = d["cu_seqlens"].tolist()
    for kernel in kernels_for(dtype):
        o, S = run_varlen(dd, kernel)
        for n, (o_ref, S_ref) in enumerate(refs):
            if lengths[n]:
                check(o[cu[n]:cu[n + 1]][None], o_ref, tau_for(dtype), f"{kernel} o seq {n}")
            check(S[n:n + 1], S_ref, tau_for(dtype), f"{kernel} S_final seq {n}")
        assert torch.equal(S[0], dd["S0"][0])          # empty sequence: the state passes through


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_prefill_varlen_equal_lengths_is_batched(kernel):
    """Equal lengths packed back to back give the bits of the [B, T] call."""
    B, T = 3, 200
    d = to_dev(inputs.prefill_inputs(B, T, 2, 6, dtype=torch.bfloat16, s0_std=0.2, seed=43))
    o_b, S_b = run_chunk(d, kernel=kernel)
    packed = {k: (v if k == "S0" else v.reshape(B * T, *v.shape[2:]).contiguous()) for k, v in d.items()}
    packed["cu_seqlens"] = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=DEV)
    o_v, S_v = run_varlen(packed, kernel)
    assert torch.equal(o_v.reshape(B, T, *o_v.shape[1:]), o_b)
    assert torch.equal(S_v, S_b)


def test_prefill_varlen_workload_sampled():
    """24 sequences of 64 .. 8192 tokens (91,038 in all), 16/48 heads: the full
    launch on the GPU; the oracle checks 3 sequences on one QK group each."""
    w = inputs.PREFILL_VARLEN
    d = inputs.varlen_workload_inputs(w, device=DEV)
    o, S = run_varlen(d)
    cu = d["cu_seqlens"].tolist()
    for n, (h0, h1) in [(0, (0, 3)), (13, (21, 24)), (23, (45, 48))]:
        a, b = cu[n], cu[n + 1]
        sub = dict(q=d["q"][None, a:b], k=d["k"][None, a:b], v=d["v"][None, a:b],
                   alpha=d["alpha"][None, a:b], beta=d["beta"][None, a:b], S0=d["S0"][n:n + 1])
        o_ref, S_ref = oracle_ref({k: v.cpu() for k, v in _sub_problem(sub, 0, h0, h1, w.Hv, w.Hqk).items()})
        check(o[a:b, h0:h1][None], o_ref, TAU_BF16, f"o seq {n} h={h0}:{h1}")
        check(S[n:n + 1, h0:h1], S_ref, TAU_BF16, f"S_final seq {n} h={h0}:{h1}")


# ----------------------------------------------------------------------------- segment-parallel prefill
def run_split(d, segments=0):
    B, T, Hqk, dk = d["q"].shape
    Hv, dv = d["v"].shape[2], d["v"].shape[3]
    o = torch.empty_like(d["v"])
    S = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=DEV)
    binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S,
                                segments=segments)
    torch.cuda.synchronize()
    return o, S


@pytest.mark.parametrize("segments", [2, 3, 4])
@pytest.mark.parametrize("T", [130, 385])
def test_prefill_split_segments_against_oracle(T, segments):
    """Every sequence cut into segments of whole chunks (the last one ragged),
    nonzero S0: outputs and the final state against the oracle."""
    d = inputs.prefill_inputs(2, T, 2, 6, dtype=torch.bfloat16, s0_std=0.3, seed=500 + T + segments)
    o_ref, S_ref = oracle_ref(d)
    need = binding.split_workspace_bytes(2, T, 6, segments)
    assert need > 0
    o, S = run_split(to_dev(d), segments)
    check(o, o_ref, TAU_BF16, f"o T={T} segments={segments}")
    check(S, S_ref, TAU_BF16, f"S_final T={T} segments={segments}")


def test_prefill_split_model_dims_workload():
    """B=1, T=4096, 16/48 heads with the automatic segment count: every output
    against the oracle."""
    w = inputs.PREFILL_4K
    d = inputs.workload_inputs(w, device=DEV)
    assert binding.split_workspace_bytes(w.B, w.T, w.Hv, 0) > 0
    o, S = run_split(d)
    o_ref, S_ref = oracle_ref(d)
    check(o, o_ref, TAU_BF16, "o")
    check(S, S_ref, TAU_BF16, "S_final")


def test_prefill_split_in_place_and_workspace_checks():
    d = to_dev(inputs.prefill_inputs(1, 300, 2, 6, dtype=torch.bfloat16, s0_std=0.2, seed=61))
    o_ref, S_ref = run_split(d, 2)
    S = d["S0"].clone()
    o = torch.empty_like(o_ref)
    binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S, o, S, segments=2)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
    # without S_final the state kernels are skipped; the outputs stay the same bits
    for segments in (2, 3):
        o_ref_n, _ = run_split(d, segments)
        o_n = torch.full_like(o_ref, float("nan"))
        binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o_n, None,
                                    segments=segments)
        torch.cuda.synchronize()
        assert torch.equal(o_n, o_ref_n), f"segments={segments}: o differs without S_final"
    assert binding.device_status() == "GDN_OK"
    need = binding.split_workspace_bytes(1, 300, 6, 2)
    short = torch.empty(need - 1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(binding.GdnError, match="INVALID_ARG"):
        binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S, o, S,
                                    segments=2, workspace=short)
