"""Runs a few launches of one kernel on one workload, for profiler captures.

    python -m linear_attention_recurrence_07_b200.profile_cases prefill [--T 4096] [--launches 3]
                                                                [--kernel tc|tc_cluster|simt]
    python -m linear_attention_recurrence_07_b200.profile_cases decode [--B 64] [--launches 5]
    python -m linear_attention_recurrence_07_b200.profile_cases prefill-fp32 [--T 1024]
    python -m linear_attention_recurrence_07_b200.profile_cases prefill-split [--segments 0]
    python -m linear_attention_recurrence_07_b200.profile_cases bwd [--T 4096] [--launches 3]

Each case builds its seeded inputs on the GPU, runs the entry point `--launches`
times and synchronizes; it prints nothing but "ok".  Point a profiler at it with
a kernel filter and a launch skip/count, e.g. skip the first two launches to
capture a warm one.
"""
import argparse

import torch

from . import binding, inputs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["prefill", "decode", "prefill-fp32", "prefill-split", "bwd"])
    ap.add_argument("--segments", type=int, default=0)
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--B", type=int, default=None)
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--kernel", choices=sorted(binding.PREFILL_KERNELS), default="auto")
    args = ap.parse_args()
    binding.set_prefill_kernel(args.kernel)
    if args.case in ("prefill", "prefill-fp32", "prefill-split"):
        w = inputs.PREFILL_SMALL_FP32 if args.case == "prefill-fp32" else inputs.PREFILL_4K
        T = args.T or (1024 if args.case == "prefill-fp32" else w.T)
        B = args.B or w.B
        d = inputs.prefill_inputs(B, T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.log_alpha,
                                  w.s0_std, w.seed, "cuda")
        o = torch.empty((B, T, w.Hv, w.dv), dtype=w.dtype, device="cuda")
        S = torch.empty((B, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")
        ws = None
        if args.case == "prefill-split":
            need = binding.split_workspace_bytes(B, T, w.Hv, args.segments)
            ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
        for _ in range(args.launches):
            if ws is not None:
                binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"],
                                            o, S, segments=args.segments, workspace=ws)
            else:
                binding.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S)
    elif args.case == "bwd":
        w = inputs.PREFILL_4K
        T = args.T or w.T
        B = args.B or w.B
        d = inputs.prefill_inputs(B, T, w.Hqk, w.Hv, w.dk, w.dv, w.dtype, w.log_alpha,
                                  w.s0_std, w.seed, "cuda")
        g = torch.Generator(device="cuda").manual_seed(w.seed + 7)
        dO = torch.randn((B, T, w.Hv, w.dv), generator=g, device="cuda").to(w.dtype)
        f32 = dict(dtype=torch.float32, device="cuda")
        grads = [torch.empty((B, T, w.Hqk, w.dk), **f32), torch.empty((B, T, w.Hqk, w.dk), **f32),
                 torch.empty((B, T, w.Hv, w.dv), **f32), torch.empty((B, T, w.Hv), **f32),
                 torch.empty((B, T, w.Hv), **f32), torch.empty((B, w.Hv, w.dk, w.dv), **f32)]
        ws = torch.empty(max(binding.bwd_workspace_bytes(B, T, w.Hv), 1), dtype=torch.uint8, device="cuda")
        for _ in range(args.launches):
            binding.gdn_bwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], dO, None, *grads,
                            workspace=ws)
    else:
        w = inputs.DECODE_B256
        B = args.B or 64
        S = inputs.decode_state(w, device="cuda", B=B)
        x = inputs.decode_inputs(w, 0, device="cuda", B=B)
        for _ in range(args.launches):
            binding.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S)
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main()
