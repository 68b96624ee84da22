"""gdn_chunk_fwd_split_noalloc (static scratch, no allocation) against
gdn_chunk_fwd_split with a caller workspace, through the C ABI: two calls in a
row, each within the bf16 tolerance of the reference call.  Kept in its own
file, collected last, so it also runs after every other test in one process."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_07_b200 import binding, inputs

pytestmark = pytest.mark.gpu

TAU_BF16 = 2e-2
MAX_SCRATCH = 48 << 20


def rel_err(got, ref):
    got = got.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float(np.abs(got - ref).max()) / max(float(np.abs(ref).max()), 1e-300)


def test_split_noalloc_matches_split_with_workspace_twice():
    w = inputs.PREFILL_4K      # B=1, T=4096, 16/48 heads: 2 segments, 36 MB of scratch
    d = inputs.workload_inputs(w, device="cuda")
    d["S0"] = torch.randn((w.B, w.Hv, w.dk, w.dv), device="cuda") * 0.02
    need = binding.split_workspace_bytes(w.B, w.T, w.Hv, 0)
    assert 0 < need <= MAX_SCRATCH
    o_ref = torch.empty_like(d["v"])
    S_ref = torch.empty_like(d["S0"])
    binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o_ref, S_ref)
    for call in range(2):
        o = torch.full_like(d["v"], float("nan"))
        S = torch.full_like(d["S0"], float("nan"))
        binding.gdn_chunk_fwd_split_noalloc(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"],
                                            o, S)
        torch.cuda.synchronize()
        e_o, e_s = rel_err(o, o_ref), rel_err(S, S_ref)
        assert e_o <= TAU_BF16 and e_s <= TAU_BF16, f"call {call}: o {e_o:.3e}, S {e_s:.3e}"


def test_split_noalloc_rejects_problems_over_the_scratch():
    # B=1, T=262144, 48 heads: the split needs far more than 48 MiB of scratch
    assert binding.split_workspace_bytes(1, 262144, 48, 2) > MAX_SCRATCH
    q = torch.zeros((1, 262144, 16, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((1, 262144, 48, 128), dtype=torch.bfloat16, device="cuda")
    g = torch.ones((1, 262144, 48), device="cuda")
    with pytest.raises(binding.GdnError, match="UNSUPPORTED"):
        binding.gdn_chunk_fwd_split_noalloc(q, q, v, g, g, None, v, None, segments=2)
