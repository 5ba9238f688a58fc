#!/usr/bin/env python
"""Benchmark of the QLoRA linear layer on B200.

Headline: forward + dX + dA/dB TFLOP/s of a 7B-shaped decoder layer training step
(q,k,v,o 4096x4096; gate/up 4096->11008; down 11008->4096; NF4 with double
quantization, LoRA r=64 alpha=16 on each; M=4096 tokens per GPU). Also reported:
the M=1 decode weight-read bandwidth on 4096x11008 and 8192x28672 NF4 weights.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU: data-parallel replicas, each with its
own 4096 tokens, and one NCCL all-reduce of the LoRA gradients per step (weak
scaling). Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s (M=4096); M=1 decode weight GB/s vs HBM peak"
WORKLOAD = ("7B-shaped decoder layer training step: q,k,v,o 4096x4096, gate/up 4096->11008, "
            "down 11008->4096, NF4 + double-quantized constants, LoRA r=64 alpha=16 on each; "
            "M=4096 tokens per GPU (4x1024); forward + dX + dA/dB through all 7 linears")
M_TOKENS, RANK_R, ALPHA = 4096, 64, 16.0
INPUT_OF = {"q": "attn_in", "k": "attn_in", "v": "attn_in", "o": "attn_out",
            "gate": "mlp_in", "up": "mlp_in", "down": "mlp_act"}
# dram__bytes_read.sum + dram__bytes_write.sum per FLOP of k_fused_nf4_gemm, from one ncu
# capture of the current kernel (forward + dX of the 11008 x 4096 linear at M = 4096)
FUSED_DRAM_BYTES_PER_FLOP = (125.920e6 + 169.601e6) / (3.751e11 + 3.715e11)


def layer_flops(linears, M, r):
    """Algorithmic FLOPs of forward + dX + dA/dB: 4MNK + 6Mr(K+N) per linear."""
    return sum(4 * M * n * k + 6 * M * r * (k + n) for _, n, k in linears)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks
_SAMPLER = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
key = sys.argv[1]
h = (pynvml.nvmlDeviceGetHandleByUUID(key) if key.startswith("GPU-")
     else pynvml.nvmlDeviceGetHandleByPciBusId(key))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    t = time.monotonic()
    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
    print(t, mhz, bits, flush=True)
    time.sleep(0.001)
"""


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, polled through NVML about every
    millisecond by a separate process (a thread of this one would compete for the GIL
    with the launch loop), and kept only between mark() and stop(): the timed region of
    a step loop lasts tens of milliseconds, far shorter than nvidia-smi's -lms sampling
    can resolve."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, device):
        self.device = device
        self.proc = None
        self.lines = []
        self.max_mhz = None
        self.t0 = None
        self._ready = threading.Event()

    def start(self):
        props = torch.cuda.get_device_properties(self.device)
        key = "GPU-" + str(props.uuid)
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _SAMPLER, key],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()
        self._ready.wait(timeout=60)

    def _read(self):
        for line in self.proc.stdout:
            parts = line.split()
            if parts and parts[0] == "max":
                self.max_mhz = float(parts[1])
                self._ready.set()
            elif len(parts) == 3:
                self.lines.append((float(parts[0]), float(parts[1]), int(parts[2])))
        self._ready.set()

    def mark(self):
        """Opens the window of kept samples (call right before the timed region)."""
        self.t0 = time.monotonic()

    def stop(self):
        t1 = time.monotonic()
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampler unavailable"],
                    "samples": 0}
        time.sleep(0.01)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        t0 = self.t0 if self.t0 is not None else 0.0
        kept = [(m, b) for t, m, b in self.lines if t0 <= t <= t1]
        if not kept:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no clock samples"],
                    "samples": 0, "source": "nvml"}
        reasons = sorted({name for _, bits in kept for name, bit in self.REASONS if bits & bit})
        mhz = [m for m, _ in kept]
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(mhz),
                "source": "nvml"}


# ------------------------------------------------------------------ oracle (CPU) leg
def oracle_sample(min_seconds=8.0):
    """Time the CPU oracle on a bounded sample of the workload: the q linear
    (4096x4096) of the layer at 512 tokens, r=64: double dequantization of the stored
    weight, forward, dX and dA/dB in fp64. Returns (TFLOP/s, seconds, description)."""
    from bit_nf4_quantized_unpack_b200 import inputs
    from oracle import nf4_oracle as O
    case = inputs.linear_case(3, 512, 4096, 4096, RANK_R, ALPHA)
    q = O.quantize_nf4_dq(case["W"])
    flops, secs, reps = 0.0, 0.0, 0
    while secs < min_seconds or reps == 0:
        t0 = time.perf_counter()
        What = O.double_dequant(q)
        Y, T = O.linear_forward(case["X"], What, case["A"], case["B"], case["scale"])
        O.linear_backward(case["dY"], case["X"], What, case["A"], case["B"], case["scale"], T=T)
        secs += time.perf_counter() - t0
        flops += layer_flops([("q", 4096, 4096)], 512, RANK_R)
        reps += 1
    desc = (f"oracle (NumPy fp64) on the q linear 4096x4096, 512 tokens, r=64: double dequant + "
            f"forward + dX + dA/dB, {reps} repetition(s)")
    return flops / secs / 1e12, secs, desc


def host_cores():
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        blas = 1
    return max(1, min(len(os.sched_getaffinity(0)), blas))


def run_reference(args, rank, world):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(min_seconds=0.0)
    per_step = []
    for _ in range(args.steps):
        v, secs, desc = oracle_sample(min_seconds=0.0)
        per_step.append((v, secs))
    value = sum(v for v, _ in per_step) / len(per_step)
    ms = 1000.0 * sum(s for _, s in per_step) / len(per_step)
    cores = host_cores()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU leg
def build_layer(device, seed):
    from bit_nf4_quantized_unpack_b200 import inputs, qlora
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    M, r = M_TOKENS, RANK_R
    layer = []
    for name, n, k in inputs.LLAMA7B_LINEARS:
        W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
        q = qlora.qlora_quantize_nf4_dq(W)
        del W
        A = (torch.randn(k, r, generator=g, device=device) * 0.02).to(torch.bfloat16)
        B = (torch.randn(r, n, generator=g, device=device) * 0.02).to(torch.bfloat16)
        layer.append(dict(name=name, n=n, k=k, q=q, A=A, B=B))
    xs = {}
    for lin in layer:
        key = INPUT_OF[lin["name"]]
        if key not in xs:
            xs[key] = torch.randn(M, lin["k"], generator=g, device=device).to(torch.bfloat16)
    grad_numel = sum(lin["k"] * r + r * lin["n"] for lin in layer)
    grads = torch.empty(grad_numel, dtype=torch.float32, device=device)
    off = 0
    ws_f = max(qlora.qlora_linear_fwd_workspace_size(M, l["n"], l["k"], r) for l in layer)
    ws_b = max(qlora.qlora_linear_bwd_workspace_size(M, l["n"], l["k"], r) for l in layer)
    for lin in layer:
        lin["dY"] = torch.randn(M, lin["n"], generator=g, device=device).to(torch.bfloat16)
        lin["Y"] = torch.empty(M, lin["n"], dtype=torch.bfloat16, device=device)
        lin["T"] = torch.empty(M, r, dtype=torch.float32, device=device)
        lin["dX"] = torch.empty(M, lin["k"], dtype=torch.bfloat16, device=device)
        lin["dA"] = grads[off:off + lin["k"] * r].view(lin["k"], r)
        off += lin["k"] * r
        lin["dB"] = grads[off:off + r * lin["n"]].view(r, lin["n"])
        off += r * lin["n"]
    return dict(layer=layer, xs=xs, grads=grads,
                ws_f=torch.empty(ws_f, dtype=torch.uint8, device=device),
                ws_b=torch.empty(ws_b, dtype=torch.uint8, device=device))


def event_pair():
    """Two timing events whose CUDA handles exist (torch creates them on first record)."""
    pair = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for e in pair:
        e.record()
    return pair


def layer_step(L, scale, world, events=None, pool=None):
    from bit_nf4_quantized_unpack_b200 import qlora
    xs = L["xs"]
    for lin in L["layer"]:
        if events is not None:
            events.append((*pool.pop(), "fwd", lin))
            qlora.qlora_profile_events(events[-1][0], events[-1][1])
        qlora.qlora_linear_fwd(xs[INPUT_OF[lin["name"]]], lin["q"], lin["A"], lin["B"], scale,
                               Y=lin["Y"], T=lin["T"], workspace=L["ws_f"])
    slices = linear_grad_slices(L["grads"], L["layer"]) if world > 1 else None
    pending = []
    for idx in reversed(range(len(L["layer"]))):
        lin = L["layer"][idx]
        if events is not None:
            events.append((*pool.pop(), "dgrad", lin))
            qlora.qlora_profile_events(events[-1][0], events[-1][1])
        qlora.qlora_linear_bwd(lin["dY"], xs[INPUT_OF[lin["name"]]], lin["T"], lin["q"], lin["A"],
                               lin["B"], scale, dX=lin["dX"], dA=lin["dA"], dB=lin["dB"],
                               workspace=L["ws_b"])
        # this linear's dA and dB are final: sum them over the ranks while the next
        # linear's backward runs
        pending.append(allreduce_linear_grads_async(slices[idx] if slices else None, world))
    if events is not None:
        qlora.qlora_profile_events(None, None)
    wait_all(pending)


def linear_grad_slices(grads, layer, r=RANK_R):
    """Each linear's [dA | dB] slice of the flat gradient buffer (dA then dB, linear after
    linear)."""
    out, off = [], 0
    for lin in layer:
        n = lin["k"] * r + r * lin["n"]
        out.append(grads[off:off + n])
        off += n
    return out


def allreduce_linear_grads_async(grad, world):
    """The data-parallel exchange of one linear: its LoRA gradients summed over the ranks
    by an all-reduce issued as soon as its backward is enqueued (the collective runs on its
    own stream after that work). Returns the pending work, or None on one rank."""
    if world > 1:
        return torch.distributed.all_reduce(grad, async_op=True)
    return None


def wait_all(pending):
    """The current stream waits for every pending collective of the step."""
    for w in pending:
        if w is not None:
            w.wait()


def allreduce_lora_grads(grads, world):
    """The whole step's LoRA gradients (one flat fp32 buffer) summed over the ranks in one
    blocking all-reduce."""
    if world > 1:
        torch.distributed.all_reduce(grads)


def max_over_ranks(value, world, device):
    """The slowest rank's time (every rank takes part)."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_steps(fn, steps, world):
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        fn()
    stop.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    return max_over_ranks(start.elapsed_time(stop) / steps, world, "cuda")


def decode_bandwidth(device, M=1, iters=40):
    """Weight-read bandwidth of the M-token forward, CUDA-graph timed, cycling through
    enough copies of the weight that no call finds it in L2."""
    from bit_nf4_quantized_unpack_b200 import qlora
    out = {}
    r, alpha = 16, 32.0
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    g = torch.Generator(device=device)
    g.manual_seed(2)
    for (n, k) in ((4096, 11008), (8192, 28672)):
        W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
        q0 = qlora.qlora_quantize_nf4_dq(W)
        del W
        wbytes = q0.codes.numel() + q0.c2.numel() + q0.c1.numel() * 4 + 4
        copies = max(2, int(np.ceil(4 * l2 / wbytes)))
        qs = [q0] + [qlora.NF4Weight(q0.codes.clone(), q0.c2.clone(), q0.c1.clone(), q0.mean.clone(),
                                     n, k) for _ in range(copies - 1)]
        A = (torch.randn(k, r, generator=g, device=device) * 0.02).to(torch.bfloat16)
        B = (torch.randn(r, n, generator=g, device=device) * 0.02).to(torch.bfloat16)
        X = torch.randn(M, k, generator=g, device=device).to(torch.bfloat16)
        Y = torch.empty(M, n, dtype=torch.bfloat16, device=device)
        ws = torch.empty(qlora.qlora_linear_fwd_workspace_size(M, n, k, r), dtype=torch.uint8,
                         device=device)
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            for i in range(3):
                qlora.qlora_linear_fwd(X, qs[i % copies], A, B, alpha / r, save_T=False, Y=Y, workspace=ws)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=s):
                for i in range(iters):
                    qlora.qlora_linear_fwd(X, qs[i % copies], A, B, alpha / r, save_T=False, Y=Y,
                                           workspace=ws)
            graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            e0.record(s)
            for _ in range(reps):
                graph.replay()
            e1.record(s)
            torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1000.0 / (reps * iters)
        algo = 0.515869140625 * n * k + (k + n) * r * 2 + M * k * 2 + M * n * 2
        out[f"{n}x{k}"] = {"M": M, "us_per_call": us, "algorithmic_bytes": int(algo),
                           "GBps": algo / us / 1e3, "weight_copies": copies}
        del graph, qs, q0
        torch.cuda.empty_cache()
    return out


def codec_bandwidth(device, reps=5):
    """HBM throughput of quantization (bf16 in), double dequantization (bf16 out) and
    merge_and_unload (bf16 out, r = 64 adapter) over
    the three Llama-7B weight shapes, cycled so that no pass finds its data in L2 (the
    three matrices hold 107M parameters, 267 MB per pass); CUDA-graph timed."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(1)
    shapes = [(4096, 4096), (4096, 11008), (11008, 4096)]
    Ws, Qs, Outs, wss, As, Bs, Qu = [], [], [], [], [], [], []
    for n, k in shapes:
        W = torch.randn(n, k, generator=g, device=device) * 0.02
        mask = torch.rand(n, k, generator=g, device=device) < 1e-3   # 0.1 % outliers x10
        W = torch.where(mask, W * 10, W).to(torch.bfloat16)
        Ws.append(W)
        Qs.append(qlora.NF4Weight.empty(n, k, device))
        Qu.append(qlora.qlora_quantize_nf4_dq(W, codebook=qlora.CODEBOOK_UNIFORM4))
        Outs.append(torch.empty(n, k, dtype=torch.bfloat16, device=device))
        As.append((torch.randn(k, RANK_R, generator=g, device=device) * 0.02).to(torch.bfloat16))
        Bs.append((torch.randn(RANK_R, n, generator=g, device=device) * 0.02).to(torch.bfloat16))
        wss.append(torch.empty(qlora.qlora_quantize_workspace_size(n, k), dtype=torch.uint8,
                               device=device))
    params = sum(n * k for n, k in shapes)
    per_param = 2.0 + 0.515869140625
    out = {}
    for name in ("quantize", "dequant", "merge", "dequant_uniform4"):
        def one_pass():
            for W, q, o, ws, A, B, qu in zip(Ws, Qs, Outs, wss, As, Bs, Qu):
                if name == "quantize":
                    qlora.qlora_quantize_nf4_dq(W, out=q, workspace=ws)
                elif name == "dequant":
                    qlora.qlora_dequant(q, out=o)
                elif name == "dequant_uniform4":  # the same kernel for the evenly spaced codebook
                    qlora.qlora_dequant(qu, out=o)
                else:  # merge_and_unload with the rank-64 adapter (A, B reads are 0.3 % extra)
                    qlora.qlora_merge_lora(q, A, B, ALPHA / RANK_R, out=o)
        s = torch.cuda.Stream(device)
        with torch.cuda.stream(s):
            one_pass()
            one_pass()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()  # the passes' kernels only, no host work between them
            with torch.cuda.graph(graph, stream=s):
                for _ in range(reps):
                    one_pass()
            graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            graph.replay()
            e1.record(s)
            torch.cuda.synchronize()
        del graph
        us = e0.elapsed_time(e1) * 1000.0 / reps
        out[name] = {"us_per_pass": us, "params": params, "bytes_per_param": per_param,
                     "GBps": params * per_param / us / 1e3}
    return out


def optimizer_bandwidth(device, reps=5):
    """HBM throughput of the paged AdamW step (qlora_adamw_step) over the LoRA parameters
    of a 7B-shaped model: 32 layers of the seven linears at r = 64, 160M fp32 values in
    one flat buffer (2.9 GB moved per 8-bit step, beyond L2). CUDA-graph timed, the
    states in device memory. Algorithmic bytes per parameter: p read and written (8),
    g read (4), the bf16 copy written (2), and the states read and written: 8-bit codes
    (4) plus two fp32 absmax per 256 values (0.0625), or fp32 m and v (16)."""
    from bit_nf4_quantized_unpack_b200 import inputs, qlora
    n = 32 * sum(RANK_R * (k + nn) for _, nn, k in inputs.LLAMA7B_LINEARS)
    g = torch.Generator(device=device)
    g.manual_seed(9)
    p = torch.randn(n, generator=g, device=device) * 0.02
    grad = torch.randn(n, generator=g, device=device) * 1e-3
    pb = torch.empty(n, dtype=torch.bfloat16, device=device)
    out = {}
    for bits, per_param in ((8, 18.0625), (32, 30.0)):
        state = torch.zeros(qlora.qlora_adamw_state_bytes(n, bits), dtype=torch.uint8, device=device)
        step = [0]

        def one():
            step[0] += 1
            qlora.qlora_adamw_step(p, grad, state, 1 + step[0] % 1000, state_bits=bits, p_bf16=pb)
        s = torch.cuda.Stream(device)
        with torch.cuda.stream(s):
            one()
            one()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=s):
                for _ in range(reps):
                    one()
            graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            graph.replay()
            e1.record(s)
            torch.cuda.synchronize()
        del graph, state
        us = e0.elapsed_time(e1) * 1000.0 / reps
        out[f"adamw_{bits}bit"] = {"us_per_step": us, "params": n, "bytes_per_param": per_param,
                                   "GBps": n * per_param / us / 1e3}
    out["workload"] = ("AdamW step over the LoRA parameters of a 7B-shaped model "
                       f"(32 layers x 7 linears, r={RANK_R}): {n} fp32 values, bf16 copy written")
    return out


def e2e_steps(L, scale, world, steps):
    """The same step through the public API with host-resident inputs: every step copies
    its activations and upstream gradients from pinned host memory and reads its LoRA
    gradients back. The copies run on a stream of their own into two sets of device
    buffers, so that step i + 1's inputs arrive, and step i's gradients leave, while step
    i computes (a data loader's prefetch). The timed region spans all copies: it opens
    before the first input copy and closes after the last gradient read."""
    dev = L["grads"].device
    host_x = {k: v.cpu().pin_memory() for k, v in L["xs"].items()}
    host_dy = [lin["dY"].cpu().pin_memory() for lin in L["layer"]]
    host_grads = [torch.empty(L["grads"].shape, dtype=torch.float32).pin_memory()
                  for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_x.values()) + \
        sum(t.numel() * t.element_size() for t in host_dy)
    d2h = host_grads[0].numel() * 4

    def make_set(first):
        if first:
            xs, dys, grads = L["xs"], [lin["dY"] for lin in L["layer"]], L["grads"]
        else:
            xs = {k: torch.empty_like(v) for k, v in L["xs"].items()}
            dys = [torch.empty_like(lin["dY"]) for lin in L["layer"]]
            grads = torch.empty_like(L["grads"])
        views, off = [], 0
        for lin in L["layer"]:
            nA, nB = lin["k"] * RANK_R, RANK_R * lin["n"]
            views.append((grads[off:off + nA].view(lin["k"], RANK_R),
                          grads[off + nA:off + nA + nB].view(RANK_R, lin["n"])))
            off += nA + nB
        return dict(xs=xs, dys=dys, grads=grads, views=views)

    sets = [make_set(True), make_set(False)]
    compute = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]

    def enqueue_inputs(i):
        S = sets[i % 2]
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(computed[i % 2])  # step i - 2 no longer reads this set
            for k, v in host_x.items():
                S["xs"][k].copy_(v, non_blocking=True)
            for d, h in zip(S["dys"], host_dy):
                d.copy_(h, non_blocking=True)
            copied[i % 2].record(copy)

    def run(i):
        S = sets[i % 2]
        compute.wait_event(copied[i % 2])
        if i >= 2:
            compute.wait_event(read_back[i % 2])  # step i - 2's gradients have left
        L["xs"], L["grads"] = S["xs"], S["grads"]
        for lin, d, (dA, dB) in zip(L["layer"], S["dys"], S["views"]):
            lin["dY"], lin["dA"], lin["dB"] = d, dA, dB
        layer_step(L, scale, world)
        computed[i % 2].record(compute)
        with torch.cuda.stream(copy):
            copy.wait_event(computed[i % 2])
            host_grads[i % 2].copy_(S["grads"], non_blocking=True)
            read_back[i % 2].record(copy)

    def timed(n):
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(compute)
        copy.wait_event(start)
        enqueue_inputs(0)
        for i in range(n):
            if i + 1 < n:
                enqueue_inputs(i + 1)
            run(i)
        compute.wait_event(read_back[(n - 1) % 2])
        stop.record(compute)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        return max_over_ranks(start.elapsed_time(stop) / n, world, "cuda")

    timed(2)  # warm-up of both buffer sets
    ms = timed(steps)
    restore = sets[0]
    L["xs"], L["grads"] = restore["xs"], restore["grads"]
    for lin, d, (dA, dB) in zip(L["layer"], restore["dys"], restore["views"]):
        lin["dY"], lin["dA"], lin["dB"] = d, dA, dB
    return ms, h2d, d2h


def stack_65b(device, warmup, steps, layers=80, M=8192, r=RANK_R, alpha=ALPHA):
    """The 65B-shaped stack: `layers` decoder layers of 8192 / 22016 linears, all NF4 with
    double-quantized constants resident at once (about 33 GB for 80 layers), LoRA r on each;
    one step is the forward and backward (dX, dA, dB) of every linear at M tokens. Inputs
    and upstream gradients are synthetic and shared by the layers (one buffer per shape);
    every linear has its own weight, adapter and gradient buffers. Returns the record (with
    the clocks seen during its timed steps); frees its buffers."""
    from bit_nf4_quantized_unpack_b200 import inputs, qlora
    g = torch.Generator(device=device)
    g.manual_seed(4)
    scale = alpha / r
    lins = []
    packed = 0
    for _ in range(layers):
        for name, n, k in inputs.LLAMA65B_LINEARS:
            W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
            q = qlora.qlora_quantize_nf4_dq(W)
            del W
            packed += q.codes.numel() + q.c2.numel() + 4 * q.c1.numel() + 4
            A = (torch.randn(k, r, generator=g, device=device) * 0.02).to(torch.bfloat16)
            B = (torch.randn(r, n, generator=g, device=device) * 0.02).to(torch.bfloat16)
            lins.append(dict(name=name, n=n, k=k, q=q, A=A, B=B,
                             dA=torch.empty(k, r, device=device),
                             dB=torch.empty(r, n, device=device)))
    xs, dys, ys, dxs, ts = {}, {}, {}, {}, {}
    for lin in lins[:7]:
        n, k = lin["n"], lin["k"]
        key = INPUT_OF[lin["name"]]
        if key not in xs:
            xs[key] = torch.randn(M, k, generator=g, device=device).to(torch.bfloat16)
        if n not in dys:
            dys[n] = torch.randn(M, n, generator=g, device=device).to(torch.bfloat16)
            ys[n] = torch.empty(M, n, dtype=torch.bfloat16, device=device)
        if k not in dxs:
            dxs[k] = torch.empty(M, k, dtype=torch.bfloat16, device=device)
    T = torch.empty(M, r, device=device)
    wf = torch.empty(max(qlora.qlora_linear_fwd_workspace_size(M, l["n"], l["k"], r) for l in lins[:7]),
                     dtype=torch.uint8, device=device)
    wb = torch.empty(max(qlora.qlora_linear_bwd_workspace_size(M, l["n"], l["k"], r) for l in lins[:7]),
                     dtype=torch.uint8, device=device)

    def step():
        for lin in lins:  # forward of every linear, then its backward (T reused)
            x = xs[INPUT_OF[lin["name"]]]
            qlora.qlora_linear_fwd(x, lin["q"], lin["A"], lin["B"], scale, Y=ys[lin["n"]], T=T,
                                   workspace=wf)
            qlora.qlora_linear_bwd(dys[lin["n"]], x, T, lin["q"], lin["A"], lin["B"], scale,
                                   dX=dxs[lin["k"]], dA=lin["dA"], dB=lin["dB"], workspace=wb)

    for _ in range(max(1, warmup)):
        step()
    torch.cuda.synchronize()
    if qlora.qlora_device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")
    clocks = ClockSampler(device)
    clocks.start()
    clocks.mark()
    launches0 = qlora.qlora_launch_count()
    ms = time_steps(step, steps, 1)
    launches = qlora.qlora_launch_count() - launches0
    clk = clocks.stop()
    flops = layers * layer_flops(inputs.LLAMA65B_LINEARS, M, r)
    rec = {"metric": "QLoRA 65B-shaped stack fwd+bwd TFLOP/s (M=8192)",
           "value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1,
           "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"{layers} layers x (q,k,v,o 8192x8192, gate/up "
                                  f"8192->22016, down 22016->8192), NF4-DQ, LoRA "
                                  f"r={r} alpha={alpha}; M={M} tokens",
                      "packed_weight_bytes": packed, "flops_per_step": flops,
                      "peak_mem_gb": torch.cuda.max_memory_allocated() / 1e9,
                      "l2": "inputs larger than L2 (33 GB of weights per step)"},
           "gpu_launches": launches, "clocks": clk}
    del lins, xs, dys, ys, dxs, wf, wb
    torch.cuda.empty_cache()
    return rec


def profile_linear(device, scale, warmup, steps):
    """One linear (gate, 11008 x 4096) forward + backward at M=4096, for ncu captures."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(5)
    n, k, M, r = 11008, 4096, M_TOKENS, RANK_R
    W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
    q = qlora.qlora_quantize_nf4_dq(W)
    del W
    A = (torch.randn(k, r, generator=g, device=device) * 0.02).to(torch.bfloat16)
    B = (torch.randn(r, n, generator=g, device=device) * 0.02).to(torch.bfloat16)
    X = torch.randn(M, k, generator=g, device=device).to(torch.bfloat16)
    dY = torch.randn(M, n, generator=g, device=device).to(torch.bfloat16)
    for _ in range(warmup + steps):
        _, T = qlora.qlora_linear_fwd(X, q, A, B, scale)
        qlora.qlora_linear_bwd(dY, X, T, q, A, B, scale)
    torch.cuda.synchronize()
    if qlora.qlora_device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")


def profile_decode(device, warmup, steps, n=8192, k=28672, M=1, r=16, alpha=32.0):
    """M-token forward (decode kernels) on one n x k weight, for ncu captures."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(6)
    W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
    q = qlora.qlora_quantize_nf4_dq(W)
    del W
    A = (torch.randn(k, r, generator=g, device=device) * 0.02).to(torch.bfloat16)
    B = (torch.randn(r, n, generator=g, device=device) * 0.02).to(torch.bfloat16)
    X = torch.randn(M, k, generator=g, device=device).to(torch.bfloat16)
    for _ in range(warmup + steps):
        qlora.qlora_linear_fwd(X, q, A, B, alpha / r, save_T=False)
    torch.cuda.synchronize()


def profile_merge(device, warmup, steps, n=4096, k=11008, r=RANK_R):
    """merge_and_unload of one n x k weight with a rank-r adapter, for ncu captures."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(7)
    W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
    q = qlora.qlora_quantize_nf4_dq(W)
    A = (torch.randn(k, r, generator=g, device=device) * 0.02).to(torch.bfloat16)
    B = (torch.randn(r, n, generator=g, device=device) * 0.02).to(torch.bfloat16)
    for _ in range(warmup + steps):
        qlora.qlora_merge_lora(q, A, B, ALPHA / r, out=W)
    torch.cuda.synchronize()


def profile_dequant(device, warmup, steps, n=4096, k=11008):
    """The standalone double dequantization of one n x k NF4 weight (bf16 out), for ncu
    captures; the quantization launches come first."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(8)
    W = (torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16)
    q = qlora.qlora_quantize_nf4_dq(W)
    for _ in range(warmup + steps):
        qlora.qlora_dequant(q, out=W)
    torch.cuda.synchronize()


def profile_quant(device, warmup, steps):
    """The quantization (NF4 codes and double-quantized constants, bf16 in) of the three
    Llama-7B weight shapes, --steps passes after --warmup, for ncu captures."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(9)
    Ws, Qs, wss = [], [], []
    for n, k in [(4096, 4096), (4096, 11008), (11008, 4096)]:
        Ws.append((torch.randn(n, k, generator=g, device=device) * 0.02).to(torch.bfloat16))
        Qs.append(qlora.NF4Weight.empty(n, k, device))
        wss.append(torch.empty(qlora.qlora_quantize_workspace_size(n, k), dtype=torch.uint8,
                               device=device))
    for _ in range(warmup + steps):
        for W, q, ws in zip(Ws, Qs, wss):
            qlora.qlora_quantize_nf4_dq(W, out=q, workspace=ws)
    torch.cuda.synchronize()


def profile_optimizer(device, warmup, steps, n=40_000_000, state_bits=8):
    """The paged AdamW step (8-bit states by default) on n LoRA-sized fp32 parameters, for
    ncu captures (0.72 GB moved per 8-bit step, beyond L2)."""
    from bit_nf4_quantized_unpack_b200 import qlora
    g = torch.Generator(device=device)
    g.manual_seed(10)
    p = torch.randn(n, generator=g, device=device) * 0.02
    grad = torch.randn(n, generator=g, device=device) * 1e-3
    pb = torch.empty(n, dtype=torch.bfloat16, device=device)
    state = torch.zeros(qlora.qlora_adamw_state_bytes(n, state_bits), dtype=torch.uint8, device=device)
    for t in range(1, warmup + steps + 1):
        qlora.qlora_adamw_step(p, grad, state, t, state_bits=state_bits, p_bf16=pb)
    torch.cuda.synchronize()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stack-65b", action="store_true",
                    help="leave the 65B-shaped stack (1 warm-up + 2 steps) out of the default run")
    ap.add_argument("--decode-m", type=int, default=1,
                    help="tokens of the --profile-decode forward (1..16)")
    ap.add_argument("--decode-n", type=int, default=8192,
                    help="weight rows (out) of the --profile-decode forward")
    ap.add_argument("--decode-k", type=int, default=28672,
                    help="weight columns (in) of the --profile-decode forward")
    ap.add_argument("--profile-decode", action="store_true",
                    help="only run the M-token forward of one n x k weight (8192x28672 unless "
                         "--decode-n/-k say otherwise) --steps times (no graph): a small, "
                         "self-contained case for profiler captures")
    ap.add_argument("--profile-dequant", action="store_true",
                    help="only run the double dequantization of a 4096x11008 weight (for ncu)")
    ap.add_argument("--profile-quant", action="store_true",
                    help="only run the quantization of the three Llama-7B weight shapes "
                         "--steps times (for ncu)")
    ap.add_argument("--profile-optimizer", action="store_true",
                    help="only run the 8-bit AdamW step on 40M parameters (for ncu)")
    ap.add_argument("--profile-merge", action="store_true",
                    help="only run merge_and_unload of a 4096x11008 weight (r=64) --steps times")
    ap.add_argument("--stack-65b", action="store_true",
                    help="time the 65B-shaped stack (80 layers of 8192/22016 linears, ~33 GB of "
                         "NF4 weights resident, M=8192): forward and backward of every linear")
    ap.add_argument("--profile-linear", action="store_true",
                    help="only run forward + backward of the gate linear (11008x4096, M=4096) "
                         "--steps times: a small, self-contained case for profiler captures")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    from bit_nf4_quantized_unpack_b200 import build, inputs, qlora
    build.build()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    scale = ALPHA / RANK_R
    if args.profile_merge:
        profile_merge(device, args.warmup, args.steps)
        return
    if args.profile_quant:
        profile_quant(device, args.warmup, args.steps)
        return
    if args.profile_optimizer:
        profile_optimizer(device, args.warmup, args.steps)
        return
    if args.profile_dequant:
        profile_dequant(device, args.warmup, args.steps)
        return
    if args.stack_65b:
        print(json.dumps(stack_65b(device, args.warmup, args.steps)), flush=True)
        return
    if args.profile_linear:
        profile_linear(device, scale, args.warmup, args.steps)
        return
    if args.profile_decode:
        profile_decode(device, args.warmup, args.steps, n=args.decode_n, k=args.decode_k,
                       M=args.decode_m)
        return
    L = build_layer(device, seed=3 + 1000 * rank)
    flops = layer_flops(inputs.LLAMA7B_LINEARS, M_TOKENS, RANK_R)
    step = lambda: layer_step(L, scale, world)  # noqa: E731

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if qlora.qlora_device_error() != 0:
        raise RuntimeError("a kernel reported a timed-out wait")

    clocks = ClockSampler(device)
    clocks.start()
    clocks.mark()
    launches0 = qlora.qlora_launch_count()
    ms = time_steps(step, args.steps, world)
    launches = qlora.qlora_launch_count() - launches0  # this library's kernels, timed region
    clk = clocks.stop()
    value = world * flops / (ms / 1e3) / 1e12
    print(f"[bench] layer step {ms:.3f} ms -> {value:.1f} TFLOP/s per {world} GPU(s)",
          file=sys.stderr, flush=True)

    # dominant kernel: the fused NF4 GEMM, timed per launch with events on its stream in a
    # pass of its own. The GPU first idles for a second: its clocks fall within ~100 ms of
    # sustained load, and this pass should start from the same state as the timed steps.
    events = []
    pool = [event_pair() for _ in range(2 * len(L["layer"]) * args.steps)]
    torch.cuda.synchronize()
    time.sleep(1.0)
    for _ in range(args.steps):
        layer_step(L, scale, world, events=events, pool=pool)
    torch.cuda.synchronize()
    fused_ms = sum(b.elapsed_time(a) for b, a, _, _ in events)
    fused_flops = 0
    for _, _, kind, lin in events:
        other = lin["n"] if kind == "fwd" else lin["k"]
        fused_flops += 2 * M_TOKENS * lin["n"] * lin["k"] + 2 * M_TOKENS * RANK_R * other
    peaks, peaks_src = load_peaks()
    achieved = fused_flops / (fused_ms / 1e3) / 1e12
    # DRAM bytes per FLOP of the fused kernel from its ncu capture (gate linear, forward and
    # dX), scaled to this step's average launch
    traffic = FUSED_DRAM_BYTES_PER_FLOP * fused_flops / len(events)
    # each launch is timed alone between its events, so the burst peak is the denominator;
    # the sustained one is given beside it
    peak = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", peak))
    roofline = {"bound": "tensor", "kernel": "k_fused_nf4_gemm (forward + dX)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peaks_src} bf16_tflops (burst)",
                "peak_sustained": sustained, "frac_of_sustained": achieved / sustained,
                "fused_share_of_step": fused_ms / args.steps / ms, "traffic": traffic,
                "traffic_unit": "bytes per launch (scaled from the ncu capture)"}

    # as many steps as the device-timed region: the first step's input copy (the pipeline
    # fill) is the one copy nothing overlaps
    e2e_n = max(3, args.steps)
    e2e_ms, h2d, d2h = e2e_steps(L, scale, world, e2e_n)
    e2e = {"value": world * flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "steps": e2e_n}

    decode = codec = optim = None
    if not args.no_decode and rank == 0:
        del L
        torch.cuda.empty_cache()
        decode = decode_bandwidth(device)
        hbm = float(peaks["hbm_gbs"])
        for v in decode.values():
            v["frac_of_hbm"] = v["GBps"] / hbm
        for m in (4, 16):  # the other decode batch sizes, same shapes and timing
            for key, v in decode_bandwidth(device, M=m).items():
                v["frac_of_hbm"] = v["GBps"] / hbm
                decode[f"{key}_m{m}"] = v
        decode["hbm_peak_GBps"] = hbm
        decode["hbm_peak_source"] = f"{peaks_src} hbm_gbs"
        codec = codec_bandwidth(device)
        for v in codec.values():
            v["frac_of_hbm"] = v["GBps"] / hbm
        codec["workload"] = ("bf16 weights 4096x4096, 4096x11008, 11008x4096 ~N(0,0.02), "
                             "0.1% x10 outliers; NF4 block 64, double-quant block 256")
        optim = optimizer_bandwidth(device)
        for k, v in optim.items():
            if isinstance(v, dict):
                v["frac_of_hbm"] = v["GBps"] / hbm

    stack = None
    if rank == 0 and world == 1 and not args.no_stack_65b:
        stack = stack_65b(device, 1, 2)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, secs, desc = oracle_sample()
        cpu = {"value": v, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
               "sample": desc, "seconds": secs}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": WORKLOAD, "tokens_per_gpu": M_TOKENS,
                           "global_tokens": M_TOKENS * world, "lora_rank": RANK_R,
                           "lora_alpha": ALPHA, "parallelism": f"dp{world}",
                           "flops_per_step_per_gpu": flops,
                           "l2": "inputs larger than L2 (weights + activations ~1.3 GB per step)"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches,
                "clocks": clk, "decode": decode, "codec": codec, "optimizer": optim,
                "stack_65b": stack}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
