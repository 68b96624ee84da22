"""Benchmark of the Gated DeltaNet token mixer on B200 (prints ONE JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--prefill-entry pipelined|split|plain]
    python bench.py --profile-case CASE [--launches L] ...   (no timing; for profilers)

A step is one pass of the hot path over one batch of synthetic input: the
prefill of the model-dims workload (B=1, T=4096, 16 QK heads, 48 V heads, head
dim 128, bf16 q/k/v, fp32 gates and state, chunk 64) through the library's
prefill entry point (default gdn_chunk_fwd_pipelined, its workspace allocated
once).  The headline ``value`` is prefill tokens/s over all ranks with inputs
resident in HBM; L2 is flushed (256 MiB write) before every timed step and each
step is timed with CUDA events on the launching stream.  Measured in the same
run and reported beside it: the batched prefill (B=8, T=8192, S0 != 0) and the
long-context prefill (B=1, T=262,144) through the same entry point, the decode
step (B=256 sequences, one token, state updated in place), draft verification,
packed prefill and the backward pass.  ``e2e`` repeats the headline prefill
through the same C entry point with pinned HOST buffers, the host<->device
copies inside the timed region.  ``cpu_baseline`` times the fp64 oracle on rank
0 on a bounded sample.  ``--impl reference`` times that oracle alone (the CPU
reference arm).

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
sequences (weak scaling); the only collectives are the timing barrier and the
max-reduction of the elapsed time.

``--profile-case`` runs one entry point a few times on one workload and prints
"ok": the command the committed ncu summaries under profiles/ were taken with.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_recurrence_07_b200 import binding, inputs  # noqa: E402

METRIC = "Gated DeltaNet prefill tokens/s, decode steps/s; % of roofline (1 B200)"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# The backward pass is plain fp32 CUDA-core arithmetic: its ceiling is the FP32 rate,
# 148 SMs x 128 FP32 lanes x 2 FLOP (FMA) x 1965 MHz (the B200's max SM clock).
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# ----------------------------------------------------------------------------- counts
def bwd_flops_per_token(w):
    """fp32 FLOPs per token and V head the gradients need at the least: one forward
    step to rebuild S_{t-1} (S^T k, rank-1 update: 5 dk dv) and the backward step
    (G += q dO^T, G^T k, S^T k, <G, S>, S_t dO, G r, S x, the G update: 16 dk dv)."""
    return 21 * w.dk * w.dv * w.Hv


def bwd_chunk_flops_per_token(w, C=64):
    """Algorithmic FLOPs of the chunkwise backward per token: per V head the start
    states (U = U~ - W S and the state update, 2 dk dv each), W and U~ (2C dk,
    2C dv), the gradient chain (K dS', Q^T dO, W^T dU: 2 dk dv each; P^T dO: 2C dv),
    and per chunk dO S^T, dU S^T, U dS'^T (2 dk dv each), dP, T^T dU, dU V^T (2C dv
    each), (dP o Gam) K, (dP o Gam)^T Q, T^T dW, dW K^T, M K, M^T K (2C dk each),
    T^T dT and Z T^T (2C^2 each); the grams once per QK head (4 C dk)."""
    per_v = 16 * w.dk * w.dv + 2 * C * (7 * w.dk + 5 * w.dv) + 4 * C * C
    return w.Hv * per_v + 4 * C * w.dk * w.Hqk


def prefill_flops_per_token(w, C=64):
    """Algorithmic FLOPs of the chunkwise form per token: per V head the products
    U~, W (2C(dk+dv)), U = U~ - W S, Q S, S update (2 dk dv each) and the masked
    P U (2 C dv); the grams K K^T and Q K^T once per QK head (4 C dk)."""
    return w.Hv * (6 * w.dk * w.dv + 2 * C * (w.dk + 2 * w.dv)) + 4 * C * w.dk * w.Hqk


def prefill_bytes_per_token(w, elt=2):
    """q, k (per QK head), v, o (per V head) in the input dtype; alpha, beta fp32."""
    return 2 * w.Hqk * w.dk * elt + 2 * w.Hv * w.dv * elt + 2 * w.Hv * 4


def prefill_state_bytes(w):
    """S0 read (if any) and S_final write, per sequence."""
    per = w.Hv * w.dk * w.dv * 4
    return per * (2 if w.s0_std > 0 else 1)


def decode_bytes_per_step(w, elt=2):
    """State read + write (fp32) and the token's q, k, v, o, alpha, beta."""
    state = 2 * w.B * w.Hv * w.dk * w.dv * 4
    tok = w.B * (2 * w.Hqk * w.dk * elt + 2 * w.Hv * w.dv * elt + 2 * w.Hv * 4)
    return state + tok


def verify_bytes_per_call(w, elt=2):
    """Multi-token decode with per-token states: the state read once, written after
    each of the n tokens (S_steps) and once more as the final state, plus the n
    tokens' q, k, v, o, alpha, beta."""
    state = w.B * w.Hv * w.dk * w.dv * 4
    tok = w.B * w.T * (2 * w.Hqk * w.dk * elt + 2 * w.Hv * w.dv * elt + 2 * w.Hv * 4)
    return (2 + w.T) * state + tok


# ----------------------------------------------------------------------------- env
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(key, workload):
    """DRAM bytes of one timed step from the committed ncu summary (entry
    ``"<key>:<workload>"``): only if it was captured on this workload (its
    ``workload_name``) from the current sources of every kernel of the step (their
    hash); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f)[f"{key}:{workload}"]
        if entry.get("workload_name") != workload:
            return None
        h = hashlib.sha256()
        for src in entry["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != entry["sources_sha256_16"]:
            return None
        return float(entry["bytes_per_step"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "utilization.gpu", "power.draw",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self, windows):
        """Clock statistics over the samples that arrived inside the timed windows
        (list of (t0, t1) perf_counter pairs)."""
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = [r for r in rows if any(t0 <= r[0] <= t1 for t0, t1 in windows)]
        use = inside or rows
        reasons = sorted({name for r in use for name, val in zip(self.REASONS, r[3])
                          if val.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_in_timed_region": len(inside)}


# ----------------------------------------------------------------------------- dist
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    """Largest value of x over all ranks (the job's elapsed time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_per_step, steps, world, max_total_ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_per_step * steps / (max_total_ms * 1e-3)


# ----------------------------------------------------------------------------- timing
PREFILL_ENTRIES = ("pipelined", "split", "plain")


def prefill_call(w, entry, stream, B=None, T=None):
    """The prefill entry point a step calls: gdn_chunk_fwd_pipelined or
    gdn_chunk_fwd_split (workspace allocated once, here) or plain gdn_chunk_fwd."""
    B = w.B if B is None else B
    T = w.T if T is None else T
    ws = None
    if entry == "split":
        need = binding.split_workspace_bytes(B, T, w.Hv, 0, w.dk, w.dv)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    elif entry == "pipelined":
        ws = torch.empty(max(binding.pipelined_workspace_bytes(B, w.Hqk, w.Hv, w.dk, w.dv), 1),
                         dtype=torch.uint8, device="cuda")

    def call(d, o, S_final):
        if entry == "split":
            binding.gdn_chunk_fwd_split(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o,
                                        S_final, segments=0, workspace=ws, stream=stream)
        elif entry == "pipelined":
            binding.gdn_chunk_fwd_pipelined(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o,
                                            S_final, workspace=ws, stream=stream)
        else:
            binding.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o,
                                  S_final, stream=stream)
    return call


def launches_per_call(w, entry):
    """Kernels of this library one prefill call launches (the pipelined entry also
    clears its flags with one cudaMemsetAsync, not a kernel of ours)."""
    if entry != "split":
        return 1
    if binding.split_workspace_bytes(w.B, w.T, w.Hv, 0, w.dk, w.dv) == 0:
        return 1
    return 3   # segment launch of the chunk kernel, segment chain (or final state), fix-up


def time_prefill(w, steps, warmup, world, rank, entry="pipelined", flush_l2=True):
    d = inputs.workload_inputs(w, device="cuda")
    o = torch.empty((w.B, w.T, w.Hv, w.dv), dtype=w.dtype, device="cuda")
    S_final = torch.empty((w.B, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES if flush_l2 else 16, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    call = prefill_call(w, entry, stream)

    def step():
        call(d, o, S_final)

    for _ in range(warmup):
        flush.fill_(1)
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(world)
    wall0 = time.perf_counter()
    for i in range(steps):
        flush.fill_(i & 0xff)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    barrier(world)
    wall1 = time.perf_counter()
    wall = wall1 - wall0
    times = [a.elapsed_time(b) for a, b in ev]            # ms, per launch
    total_ms = max_over_ranks(sum(times), world)
    return {"total_ms": total_ms, "per_launch_ms": sum(times) / steps,
            "median_ms": statistics.median(times), "wall_s": wall, "launches": steps,
            "window": (wall0, wall1)}


def time_prefill_e2e(w, steps, warmup, world, entry="pipelined"):
    """Same call with inputs from pinned host memory and results read back."""
    host = {k: (None if v is None else v.cpu().pin_memory())
            for k, v in inputs.workload_inputs(w, device="cpu").items()}
    dev = {k: (None if v is None else torch.empty_like(v, device="cuda")) for k, v in host.items()}
    o = torch.empty((w.B, w.T, w.Hv, w.dv), dtype=w.dtype, device="cuda")
    S_final = torch.empty((w.B, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    S_h = torch.empty(S_final.shape, dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * 4
    call = prefill_call(w, entry, stream)

    def step():
        for k_, v in host.items():
            if v is not None:
                dev[k_].copy_(v, non_blocking=True)
        call(dev, o, S_final)
        o_h.copy_(o, non_blocking=True)
        S_h.copy_(S_final, non_blocking=True)

    for _ in range(warmup):
        step()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    barrier(world)
    total_ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"total_ms": total_ms, "h2d": h2d, "d2h": d2h}


def time_decode(w, steps, warmup, world, pool=16):
    S = inputs.decode_state(w, device="cuda")
    xs = [inputs.decode_inputs(w, s, device="cuda") for s in range(pool)]
    o = torch.empty((w.B, w.Hv, w.dv), dtype=w.dtype, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        x = xs[i % pool]
        binding.gdn_decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, o, S,
                                stream=stream)

    for i in range(warmup):
        step(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(world)
    wall0 = time.perf_counter()
    for i in range(steps):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    barrier(world)
    wall1 = time.perf_counter()
    times = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(times), world)
    return {"total_ms": total_ms, "per_launch_ms": sum(times) / steps, "launches": steps,
            "window": (wall0, wall1)}


def time_calls(call, steps, warmup, world):
    """CUDA-event time of `steps` calls of call(i) on the current stream, after
    `warmup` untimed ones; the inputs are larger than L2, so no flush."""
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        call(i)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(world)
    wall0 = time.perf_counter()
    for i in range(steps):
        ev[i][0].record(stream)
        call(i)
        ev[i][1].record(stream)
    barrier(world)
    wall1 = time.perf_counter()
    times = [a.elapsed_time(b) for a, b in ev]
    return {"total_ms": max_over_ranks(sum(times), world), "per_launch_ms": sum(times) / steps,
            "launches": steps, "window": (wall0, wall1)}


def time_backward(w, steps, warmup, world, entry="chunk"):
    """gdn_bwd_chunk (entry "chunk") or gdn_bwd ("token") on the prefill workload:
    dO random, no S0 / dS_final (the workload's own S0 is none either)."""
    d = inputs.workload_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(w.seed + 7)
    dO = torch.randn((w.B, w.T, w.Hv, w.dv), generator=g, device="cuda").to(w.dtype)
    f32 = dict(dtype=torch.float32, device="cuda")
    dq = torch.empty((w.B, w.T, w.Hqk, w.dk), **f32)
    dk = torch.empty_like(dq)
    dv = torch.empty((w.B, w.T, w.Hv, w.dv), **f32)
    da = torch.empty((w.B, w.T, w.Hv), **f32)
    db = torch.empty_like(da)
    dS0 = torch.empty((w.B, w.Hv, w.dk, w.dv), **f32)
    ws_bytes, fn = ((binding.bwd_chunk_workspace_bytes, binding.gdn_bwd_chunk) if entry == "chunk"
                    else (binding.bwd_workspace_bytes, binding.gdn_bwd))
    ws = torch.empty(ws_bytes(w.B, w.T, w.Hv, w.dk, w.dv), dtype=torch.uint8, device="cuda")

    def call(i):
        fn(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], dO, None,
           dq, dk, dv, da, db, dS0, workspace=ws)

    return time_calls(call, steps, warmup, world)


def time_verify(w, steps, warmup, world):
    """gdn_decode_tokens: n draft tokens for each of B sequences, state in place,
    the state after every token written to S_steps."""
    d = inputs.workload_inputs(w, device="cuda")
    S = d["S0"]
    o = torch.empty((w.B, w.T, w.Hv, w.dv), dtype=w.dtype, device="cuda")
    steps_buf = torch.empty((w.B, w.T, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")

    def call(i):
        binding.gdn_decode_tokens(d["q"], d["k"], d["v"], d["alpha"], d["beta"], S, o, S, steps_buf)

    return time_calls(call, steps, warmup, world)


def time_varlen(w, steps, warmup, world):
    """gdn_chunk_fwd_varlen over the packed sequences of w (inputs > L2)."""
    d = inputs.varlen_workload_inputs(w, device="cuda")
    N = w.B
    o = torch.empty_like(d["v"])
    S = torch.empty((N, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")

    def call(i):
        binding.gdn_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], o, S,
                                     d["cu_seqlens"])

    r = time_calls(call, steps, warmup, world)
    r["tokens"] = int(d["q"].shape[0])
    return r


# ----------------------------------------------------------------------------- oracle
def oracle_prefill_sample(w, min_seconds=10.0, max_seconds=30.0):
    """Times the fp64 oracle on the prefill workload (all heads), repeating whole
    passes over the first `T_s` tokens until about `min_seconds` have elapsed."""
    import oracle
    T_s = min(w.T, 4096)
    d = inputs.workload_inputs(w, device="cpu", T=T_s)
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], nthreads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or el * (reps + 1) / reps > max_seconds:
            break
    tok = reps * w.B * T_s
    return {"value": tok / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} x full oracle pass over B={w.B}, T={T_s} (all {w.Hv} V heads), "
                      f"{el:.1f} s"}


def oracle_decode_sample(w, min_seconds=5.0):
    import oracle
    B_s = w.B
    S = inputs.decode_state(w, device="cpu", B=B_s).numpy()
    cores = oracle.default_threads()
    t0 = time.perf_counter()
    n = 0
    while True:
        x = inputs.decode_inputs(w, n, device="cpu", B=B_s)
        _, S64 = oracle.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S, nthreads=cores)
        S = S64.astype("float32")
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return {"value": n / el, "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} decode steps of B={B_s} x {w.Hv} heads, {el:.1f} s"}


# ----------------------------------------------------------------------------- main
def roofline(bound, achieved, peak, unit, traffic):
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": traffic}


def run_reference(args, rank, world):
    """CPU reference arm: the fp64 oracle on a bounded sample of the same workload."""
    if rank != 0:
        return
    w = inputs.PREFILL_4K
    per_step_T = 256
    d = inputs.workload_inputs(w, device="cpu", T=per_step_T)
    import oracle
    cores = oracle.default_threads()
    run = lambda: oracle.forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"],  # noqa
                                 nthreads=cores)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    value = args.steps * w.B * per_step_T / el
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": per_step_T, "Hqk": w.Hqk, "Hv": w.Hv,
                       "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
                       "sample_of": f"{w.name}: the first {per_step_T} of its {w.T} tokens per step"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: oracle pass over B=1, T={per_step_T} "
                                       f"(all {w.Hv} V heads) of the workload"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


ENTRY_NAMES = {"pipelined": "gdn_chunk_fwd_pipelined (prep and chain CTAs, one cooperative launch)",
               "split": "gdn_chunk_fwd_split (segments chosen by the library)",
               "plain": "gdn_chunk_fwd"}
# What each entry's timed step is (for the roofline record).
ENTRY_TIMED = {"pipelined": "the whole pipelined launch (prep and chain CTAs) and its flag reset",
               "split": "the whole split step: segment launch of the chunk kernel, segment chain, output fix-up",
               "plain": "the one-CTA chunk kernel"}
# Targets of the prefill workloads (time per call at 50% of the measured bf16 peak).
PREFILL_TARGET_FRAC = 0.5


def leg_entry(w, entry):
    """The entry point a prefill leg times: the pipelined entry needs SMs for its
    preparation CTAs beside one chain CTA per head, so with more heads than half the
    SMs (B * Hv > SMs / 2) it runs its heads in waves with too few preparation CTAs;
    such workloads go through the split entry (which then runs the one-CTA kernel)."""
    if entry == "pipelined":
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        if 2 * w.B * w.Hv > sms:
            return "split"
    return entry


def prefill_leg(w, entry, steps, warmup, world, rank, peaks, peak_src):
    """One prefill workload through `entry` (inputs larger than L2: no flush)."""
    entry = leg_entry(w, entry)
    r = time_prefill(w, steps, warmup, world, rank, entry=entry, flush_l2=False)
    tok = w.B * w.T
    t = r["per_launch_ms"] * 1e-3
    flops = prefill_flops_per_token(w) * tok
    target_ms = flops / (PREFILL_TARGET_FRAC * peaks["bf16_tflops"] * 1e12) * 1e3
    return {"metric": f"prefill tokens/s ({ENTRY_NAMES[entry]})", "workload": w.name, "B": w.B,
            "T": w.T, "S0": w.s0_std > 0, "value": job_throughput(tok, steps, world, r["total_ms"]),
            "unit": "tokens/s", "ms_per_call": r["total_ms"] / steps,
            "target_ms": target_ms, "meets_target": r["total_ms"] / steps <= target_ms,
            "roofline": dict(roofline("tensor", flops / t / 1e12, peaks["bf16_tflops"], "TFLOP/s",
                                      kernel_traffic(f"prefill_{entry}", w.name)),
                             peak_source=f"{peak_src} bf16 burst", algorithmic_flops_per_launch=flops,
                             hbm_frac=(prefill_bytes_per_token(w) * tok + w.B * prefill_state_bytes(w))
                             / t / 1e9 / peaks["hbm_gbs"]),
            "gpu_launches": r["launches"] * launches_per_call(w, entry),
            "window": r["window"]}


def profile_case(args):
    """Runs one entry point `--launches` times on one workload and synchronizes
    (no timing, prints "ok"): the command the ncu summaries in profiles/ name."""
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    case = args.profile_case
    if case in ("prefill", "prefill-batched", "prefill-long"):
        w = {"prefill": inputs.PREFILL_4K, "prefill-batched": inputs.PREFILL_BATCH8_8K,
             "prefill-long": inputs.PREFILL_256K}[case]
        T = args.T or w.T
        d = inputs.workload_inputs(w, device="cuda", T=T)
        o = torch.empty((w.B, T, w.Hv, w.dv), dtype=w.dtype, device="cuda")
        S = torch.empty((w.B, w.Hv, w.dk, w.dv), dtype=torch.float32, device="cuda")
        call = prefill_call(w, args.prefill_entry, stream, T=T)
        for _ in range(args.launches):
            call(d, o, S)
    elif case == "decode":
        w = inputs.DECODE_B256
        B = args.B or w.B
        S = inputs.decode_state(w, device="cuda", B=B)
        x = inputs.decode_inputs(w, 0, device="cuda", B=B)
        for _ in range(args.launches):
            binding.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], S)
    elif case in ("bwd", "bwd-chunk"):
        w = inputs.PREFILL_4K
        T = args.T or w.T
        d = inputs.workload_inputs(w, device="cuda", T=T)
        g = torch.Generator(device="cuda").manual_seed(w.seed + 7)
        dO = torch.randn((w.B, T, w.Hv, w.dv), generator=g, device="cuda").to(w.dtype)
        f32 = dict(dtype=torch.float32, device="cuda")
        grads = [torch.empty((w.B, T, w.Hqk, w.dk), **f32), torch.empty((w.B, T, w.Hqk, w.dk), **f32),
                 torch.empty((w.B, T, w.Hv, w.dv), **f32), torch.empty((w.B, T, w.Hv), **f32),
                 torch.empty((w.B, T, w.Hv), **f32), torch.empty((w.B, w.Hv, w.dk, w.dv), **f32)]
        ws_bytes, fn = ((binding.bwd_chunk_workspace_bytes, binding.gdn_bwd_chunk) if case == "bwd-chunk"
                        else (binding.bwd_workspace_bytes, binding.gdn_bwd))
        ws = torch.empty(max(ws_bytes(w.B, T, w.Hv), 1), dtype=torch.uint8, device="cuda")
        for _ in range(args.launches):
            fn(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], dO, None, *grads, workspace=ws)
    else:
        raise SystemExit(f"unknown profile case {case}")
    torch.cuda.synchronize()
    print("ok")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--verify-steps", type=int, default=50)
    ap.add_argument("--varlen-steps", type=int, default=20)
    ap.add_argument("--bwd-steps", type=int, default=20)
    ap.add_argument("--bwd-token-steps", type=int, default=3)
    ap.add_argument("--batched-steps", type=int, default=10)
    ap.add_argument("--long-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-entry", choices=PREFILL_ENTRIES, default="pipelined",
                    help="prefill entry point of the timed step (default: gdn_chunk_fwd_pipelined, "
                         "the fastest on B=1, T=4096; the others are timed beside it)")
    ap.add_argument("--prefill-kernel", choices=sorted(binding.PREFILL_KERNELS), default="auto",
                    help="kernel gdn_chunk_fwd / _split / _varlen run (default: the library's choice)")
    ap.add_argument("--profile-case", choices=["prefill", "prefill-batched", "prefill-long", "decode", "bwd-chunk",
                                               "bwd"], default=None)
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--B", type=int, default=None)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    binding.set_prefill_kernel(args.prefill_kernel)
    if args.profile_case:
        profile_case(args)
        return

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return

    rank, world, local = dist_setup(args.gpus)
    peaks, peak_src = load_peaks()
    w = inputs.PREFILL_4K
    wd = inputs.DECODE_B256
    entry = args.prefill_entry
    kernel = binding.prefill_kernel_for(w.B, w.Hv, w.dtype)
    with ClockSampler(local) as clocks:
        pre = time_prefill(w, args.steps, args.warmup, world, rank, entry=entry)
        others = {e: time_prefill(w, max(args.steps // 5, 3), args.warmup, world, rank, entry=e)
                  for e in PREFILL_ENTRIES if e != entry}
        dec = time_decode(wd, args.decode_steps, args.warmup, world)
    with ClockSampler(local) as clocks3:
        batched = prefill_leg(inputs.PREFILL_BATCH8_8K, entry, args.batched_steps, 3, world, rank,
                              peaks, peak_src)
        longctx = prefill_leg(inputs.PREFILL_256K, entry, args.long_steps, 3, world, rank, peaks, peak_src)
    for leg in (batched, longctx):
        leg["clocks"] = clocks3.summary([leg.pop("window")])
    wv, wl = inputs.VERIFY_B256_N4, inputs.PREFILL_VARLEN
    with ClockSampler(local) as clocks2:
        ver = time_verify(wv, args.verify_steps, args.warmup, world)
        vl = time_varlen(wl, args.varlen_steps, args.warmup, world)
        bw = time_backward(w, args.bwd_steps, 3, world, entry="chunk")
        bwt = time_backward(w, args.bwd_token_steps, 1, world, entry="token")
    e2e = time_prefill_e2e(w, args.e2e_steps, 3, world, entry=entry)

    tokens_per_step = w.B * w.T
    value = job_throughput(tokens_per_step, args.steps, world, pre["total_ms"])
    flops_launch = prefill_flops_per_token(w) * tokens_per_step
    bytes_launch = prefill_bytes_per_token(w) * tokens_per_step + w.B * prefill_state_bytes(w)
    t_launch = pre["per_launch_ms"] * 1e-3
    dec_bytes = decode_bytes_per_step(wd)
    t_dec = dec["per_launch_ms"] * 1e-3
    clk = clocks.summary([pre["window"], dec["window"]])

    if rank != 0:
        shutdown(world)
        return
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": pre["total_ms"] / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "Hqk": w.Hqk, "Hv": w.Hv,
                   "dk": w.dk, "dv": w.dv, "chunk": w.chunk, "state": "fp32",
                   "prefill_entry": ENTRY_NAMES[entry],
                   "other_entries_ms": {e: r["total_ms"] / r["launches"] for e, r in others.items()},
                   "one_cta_kernel": kernel,
                   "l2": "flushed before every timed step (256 MiB write)",
                   "parallelism": f"dp{world} (independent sequences per GPU)"},
        "roofline": dict(roofline("tensor", flops_launch / t_launch / 1e12, peaks["bf16_tflops"],
                                  "TFLOP/s", kernel_traffic(f"prefill_{entry}", w.name)),
                         timed=ENTRY_TIMED[entry],
                         peak_source=f"{peak_src} bf16 burst",
                         algorithmic_flops_per_launch=flops_launch,
                         hbm_frac=bytes_launch / t_launch / 1e9 / peaks["hbm_gbs"]),
        "batched_prefill": batched,
        "long_context_prefill": longctx,
        "decode": {
            "metric": "decode steps/s", "workload": wd.name, "B": wd.B,
            "value": job_throughput(1, args.decode_steps, world, dec["total_ms"]), "unit": "steps/s",
            "ms_per_step": dec["total_ms"] / args.decode_steps,
            "roofline": dict(roofline("hbm", dec_bytes / t_dec / 1e9, peaks["hbm_gbs"], "GB/s",
                                      kernel_traffic("decode", wd.name)),
                             peak_source=f"{peak_src} copy bandwidth",
                             algorithmic_bytes_per_launch=dec_bytes),
            "gpu_launches": dec["launches"],
        },
        "verify": {
            "metric": "draft-verify tokens/s (gdn_decode_tokens, per-token states kept)",
            "workload": wv.name, "B": wv.B, "tokens_per_sequence": wv.T,
            "value": job_throughput(wv.B * wv.T, args.verify_steps, world, ver["total_ms"]),
            "unit": "tokens/s", "ms_per_call": ver["total_ms"] / args.verify_steps,
            "roofline": dict(roofline("hbm", verify_bytes_per_call(wv) / (ver["per_launch_ms"] * 1e-3) / 1e9,
                                      peaks["hbm_gbs"], "GB/s", None),
                             peak_source=f"{peak_src} copy bandwidth",
                             algorithmic_bytes_per_launch=verify_bytes_per_call(wv)),
            "gpu_launches": ver["launches"],
        },
        "backward": {
            "metric": "backward tokens/s (gdn_bwd_chunk: dq, dk, dv, dalpha, dbeta, dS0)",
            "workload": w.name, "B": w.B, "T": w.T,
            "value": job_throughput(tokens_per_step, args.bwd_steps, world, bw["total_ms"]),
            "unit": "tokens/s", "ms_per_call": bw["total_ms"] / args.bwd_steps,
            "vs_forward": (bw["total_ms"] / args.bwd_steps) / pre["per_launch_ms"],
            "roofline": dict(roofline("tensor", bwd_chunk_flops_per_token(w) * tokens_per_step
                                      / (bw["per_launch_ms"] * 1e-3) / 1e12,
                                      peaks["bf16_tflops"], "TFLOP/s", None),
                             peak_source=f"{peak_src} bf16 burst",
                             algorithmic_flops_per_launch=bwd_chunk_flops_per_token(w) * tokens_per_step),
            "gpu_launches": 4 * bw["launches"],
            "token_serial": {
                "entry": "gdn_bwd (fp32 CUDA cores, one token at a time)",
                "ms_per_call": bwt["total_ms"] / args.bwd_token_steps,
                "roofline": dict(roofline("alu", bwd_flops_per_token(w) * tokens_per_step
                                          / (bwt["per_launch_ms"] * 1e-3) / 1e12,
                                          FP32_ALU_TFLOPS, "TFLOP/s", None),
                                 peak_source="fp32 lanes x max SM clock (148 x 128 x 2 x 1965 MHz)"),
                "gpu_launches": bwt["launches"],
            },
        },
        "varlen_prefill": {
            "metric": "packed-prefill tokens/s (gdn_chunk_fwd_varlen)",
            "workload": wl.name, "sequences": wl.B, "tokens": vl["tokens"],
            "prefill_kernel": binding.prefill_kernel_for(wl.B, wl.Hv, wl.dtype),
            "value": job_throughput(vl["tokens"], args.varlen_steps, world, vl["total_ms"]),
            "unit": "tokens/s", "ms_per_call": vl["total_ms"] / args.varlen_steps,
            "roofline": dict(roofline("tensor", prefill_flops_per_token(wl) * vl["tokens"]
                                      / (vl["per_launch_ms"] * 1e-3) / 1e12,
                                      peaks["bf16_tflops"], "TFLOP/s", None),
                             peak_source=f"{peak_src} bf16 burst",
                             hbm_frac=(prefill_bytes_per_token(wl) * vl["tokens"] + wl.B * prefill_state_bytes(wl))
                             / (vl["per_launch_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"]),
            "gpu_launches": vl["launches"],
            "clocks": clocks2.summary([ver["window"], vl["window"]]),
        },
        "e2e": {"value": job_throughput(tokens_per_step, args.e2e_steps, world, e2e["total_ms"]),
                "unit": "tokens/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"]},
        "gpu_launches": pre["launches"] * launches_per_call(w, entry),
        "clocks": clk,
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = oracle_prefill_sample(w)
        line["decode"]["cpu_baseline"] = oracle_decode_sample(wd)
    print(json.dumps(line), flush=True)


def shutdown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
    shutdown(int(os.environ.get("WORLD_SIZE", "1")))
