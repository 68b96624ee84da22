"""gdn_chunk_fwd_split_noalloc (static scratch, no allocation) against
gdn_chunk_fwd_split with a caller workspace, through the C ABI.

The two run the same deterministic kernels on the same inputs, so their outputs
must be identical bit for bit; a wrong offset into the static array, or stale
contents of it, would show.  Two calls in a row, for two and four segments, and
the device's free memory must not change across a call once the library is
loaded.  Kept in its own file, collected last, so it also runs after every other
test in one process."""
import pytest
import torch

from linear_attention_recurrence_07_b200 import binding, inputs

pytestmark = pytest.mark.gpu

MAX_SCRATCH = 48 << 20


@pytest.mark.parametrize("T,segments", [(4096, 0), (1536, 4)], ids=["4K-auto", "1536-4seg"])
def test_split_noalloc_matches_split_with_workspace_twice(T, segments):
    w = inputs.PREFILL_4K      # 16 QK / 48 V heads; T=4096 auto-splits in 2 (36 MB of scratch)
    d = inputs.workload_inputs(w, device="cuda", T=T)
    d["S0"] = torch.randn((w.B, w.Hv, w.dk, w.dv), device="cuda") * 0.02
    need = binding.split_workspace_bytes(w.B, T, w.Hv, segments)
    assert 0 < need <= MAX_SCRATCH
    o_ref = torch.empty_like(d["v"])
    S_ref = torch.empty_like(d["S0"])
    binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o_ref, S_ref,
                                segments=segments)
    for call in range(2):
        o = torch.full_like(d["v"], float("nan"))
        S = torch.full_like(d["S0"], float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        binding.gdn_chunk_fwd_split_noalloc(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"],
                                            o, S, segments=segments)
        torch.cuda.synchronize()
        if call > 0:   # the first call may load the module (lazy loading) and so reserve the array
            assert torch.cuda.mem_get_info()[0] == free_before, f"call {call} changed free memory"
        assert torch.equal(o, o_ref), f"call {call}: o differs from the workspace call"
        assert torch.equal(S, S_ref), f"call {call}: S_final differs from the workspace call"


def test_split_noalloc_rejects_problems_over_the_scratch():
    # B=1, T=262144, 48 heads: the split needs far more than 48 MiB of scratch
    assert binding.split_workspace_bytes(1, 262144, 48, 2) > MAX_SCRATCH
    q = torch.zeros((1, 262144, 16, 128), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros((1, 262144, 48, 128), dtype=torch.bfloat16, device="cuda")
    g = torch.ones((1, 262144, 48), device="cuda")
    with pytest.raises(binding.GdnError, match="UNSUPPORTED"):
        binding.gdn_chunk_fwd_split_noalloc(q, q, v, g, g, None, v, None, segments=2)
