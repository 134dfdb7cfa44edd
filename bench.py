#!/usr/bin/env python
"""Benchmark of the QLoRA linear layer (libqlora) on B200.

One step = one training pass of the layer: forward (sU = s X A^T, then the
fused NF4-dequant tensor-core GEMM Y = X W'^T + sU B^T) and backward
(sT = s dY B, the fused dX = dY W' + sT A GEMM, dA = sT^T X, dB = dY^T sU),
on the Llama-7B attention-projection workload (W 4096x4096 NF4 with 0.1% x8
outliers, 2048 tokens, r = 16, alpha = 32). The JSON line also carries the
standalone dequantisation bandwidth and the 8-token forward bandwidth over the
8B linear set, the roofline of the dominant kernel, the end-to-end number
through the public API with host buffers, the clocks seen while timing and the
CPU oracle's throughput on a bounded sample.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 (under torchrun) every rank runs an independent replica of
the workload (the layer does not exchange data); the time is the maximum over
ranks and the value counts the work of all ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s & NF4 dequant GB/s (1xB200, % of roofline)"
WORKLOAD = "attn_proj_7b"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-extras", action="store_true", help="skip the 8B-set dequant / decode lines")
    p.add_argument("--oracle-configs", action="store_true",
                   help="time the CPU oracle on every workload (host only) and print one JSON line")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--kernel-case", choices=sorted(KERNEL_CASES),
                   help="run one kernel family on its profiling workload (3 calls, then one more) and exit; "
                        "for ncu -k <kernel> -s 3 -c 1")
    return p.parse_args()


def _kc_setup():
    import torch
    import bit_nf4_quantized_dequant_b200 as q
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    bf = lambda *shape, sc=1.0: (torch.randn(*shape, generator=g, device="cuda") * sc).bfloat16()
    w = lambda n, k: torch.randn(n, k, generator=g, device="cuda") * 0.02
    return torch, q, bf, w


def _kc_dequant():
    torch, q, bf, w = _kc_setup()
    m = q.nf4_quantize(w(8192, 8192))
    o = torch.empty(8192, 8192, dtype=torch.bfloat16, device="cuda")
    return lambda: q.nf4_dequantize(m, out=o)


def _kc_quantize():
    torch, q, bf, w = _kc_setup()
    W, m = w(8192, 8192), q.NF4Matrix.empty(8192, 8192, "cuda")
    return lambda: q.nf4_quantize(W, out=m)


def _kc_merge():
    torch, q, bf, w = _kc_setup()
    N, K, r = 4096, 14336, 16
    m, A, B = q.nf4_quantize(w(N, K)), bf(r, K, sc=0.01), bf(N, r, sc=0.01)
    o = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    return lambda: q.nf4_merge(m, A, B, 2.0, out=o)


def _kc_linear():
    torch, q, bf, w = _kc_setup()
    M, N, K, r = 2048, 4096, 4096, 16
    m, X, A, B, dY = q.nf4_quantize(w(N, K)), bf(M, K), bf(r, K, sc=0.01), bf(N, r, sc=0.01), bf(M, N)
    ws = torch.zeros(q.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")

    def step():
        Y, sU = q.linear_fwd(m, X, A, B, 2.0, ws=ws)
        q.linear_bwd(m, X, A, B, 2.0, dY, sU=sU, ws=ws)
    return step


def _kc_swiglu():
    torch, q, bf, w = _kc_setup()
    M, H, F, r = 4096, 4096, 11008, 16
    qgu = q.nf4_quantize(q.swiglu_interleave(w(F, H), w(F, H)))
    X, Bgu = bf(M, H), q.swiglu_pack_b(bf(F, r, sc=0.01), bf(F, r, sc=0.01))
    sU, dH = bf(M, 2 * r, sc=0.1), bf(M, F)

    def step():
        q.swiglu_fwd(qgu, X, Bgu, sU)
        q.swiglu_bwd(qgu, X, Bgu, sU, dH)
    return step


def _kc_decode():
    # one grouped few-token launch of sixteen 8B linears (two layers' q, k, v,
    # o, gate, up, down, then q and k: 236 MB of codes, more than L2), L2
    # flushed before each call
    torch, q, bf, w = _kc_setup()
    M, r = 8, 16
    probs, X = [], {}
    layer = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)]
    for (N, K) in layer * 2 + layer[:2]:
        if K not in X:
            X[K] = bf(M, K)
        probs.append(q.LinearProblem(q.nf4_quantize(w(N, K)), X[K], bf(r, K, sc=0.06), bf(N, r, sc=0.01), 2.0,
                                     torch.empty(M, N, dtype=torch.bfloat16, device="cuda"),
                                     torch.empty(M, r, dtype=torch.bfloat16, device="cuda")))
    ws = torch.zeros(q.linear_fwd_group_workspace(probs, M), dtype=torch.uint8, device="cuda")
    arr = q._binding._problem_array(probs)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def step():
        flush.zero_()
        q.linear_fwd_group(probs, ws=ws, arr=arr)
    return step


KERNEL_CASES = {"dequant": _kc_dequant, "quantize": _kc_quantize, "merge": _kc_merge, "linear": _kc_linear,
                "swiglu": _kc_swiglu, "decode": _kc_decode}


def run_kernel_case(name):
    import torch
    from bit_nf4_quantized_dequant_b200 import _build
    _build.build()
    f = KERNEL_CASES[name]()
    for _ in range(4):
        f()
    torch.cuda.synchronize()
    print(json.dumps({"kernel_case": name, "calls": 4}))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x20: "sync_boost", 0x40: "sw_thermal_slowdown", 0x80: "hw_thermal_slowdown",
           0x100: "hw_power_brake_slowdown", 0x200: "display_clock_setting"}


class ClockSampler:
    """Samples the SM clock and the clock-event reasons while active. The
    period is short (0.5 ms) and start() takes one sample at once, so even a
    timed region of a few milliseconds is covered."""

    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._active = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _sample(self):
        if self.nv is None:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            reasons = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            self.samples.append((mhz, reasons))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            if self._active.is_set():
                self._sample()
            time.sleep(self.period)

    def start(self):
        self._active.set()
        self._sample()

    def stop(self):
        self._active.clear()

    def close(self):
        self._stop.set()
        self.t.join(timeout=1)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        names = [n for b, n in REASONS.items() if bits & b and b != 0x1]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(mhz)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only: the only collective is the timing max)
# ---------------------------------------------------------------------------
def init_dist(backend: str = "nccl"):
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the
    launcher). The replicas exchange nothing but the timing maximum; "gloo"
    runs the same plumbing on CPU processes."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(world: int, flops_per_step: float, steps: int, ms_total_max: float) -> float:
    """Whole-job TFLOP/s of N replicas (weak scaling): every rank runs the same
    steps, the job takes the slowest rank's time."""
    return world * flops_per_step * steps / (ms_total_max * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------
def step_flops(M, N, K, r):
    """Algorithmic flops of one fwd+bwd: the two dense products 2MNK each and
    the six rank-r products 2Mr(K) or 2Mr(N) (no dW)."""
    return 4 * M * N * K + 6 * M * r * (K + N)


def fused_flops(mode, M, N, K, r):
    return 2 * M * N * K + (2 * M * N * r if mode == "fwd" else 2 * M * K * r)


def make_sets(q, torch, n_sets, N, K, M, r, outliers):
    from bit_nf4_quantized_dequant_b200 import inputs
    sets = []
    for i in range(n_sets):
        c = inputs.linear_case(N, K, M, r, index=i, outliers=outliers)
        bf = lambda b: torch.from_numpy(b.view("int16")).view(torch.bfloat16).cuda()
        Wf = torch.from_numpy(c["W"]).cuda()
        nf4 = q.nf4_quantize(Wf)
        del Wf
        d = dict(q=nf4, X=bf(c["X"]), A=bf(c["A"]), B=bf(c["B"]), dY=bf(c["dY"]))
        d["Y"] = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        d["dX"] = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        d["sU"] = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        d["sT"] = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        d["dA"] = torch.empty((r, K), dtype=torch.float32, device="cuda")
        d["dB"] = torch.empty((N, r), dtype=torch.float32, device="cuda")
        d["ws"] = torch.zeros(q.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")
        d["gws"] = torch.zeros(q.fused_workspace(M), dtype=torch.uint8, device="cuda")
        sets.append(d)
    torch.cuda.synchronize()
    return sets


def set_bytes(M, N, K, r):
    packed = N * K // 2 + N * K // 64 + 4 * -(-(N * K // 64) // 256)
    return packed + 2 * (2 * M * K + 2 * M * N) + 2 * r * (K + N) + 4 * M * r + 4 * r * (K + N)


def make_side(torch):
    """A second stream and the events of one step's fork / join."""
    return (torch.cuda.Stream(),) + tuple(torch.cuda.Event() for _ in range(4))


def run_step(q, d, s, ev=None, side=None):
    """One forward + backward of the layer. The five launches form a DAG: the
    main stream runs sU -> Y -> dX (the two fused GEMMs need sU and sT); a side
    stream computes sT and then dA, dB (which need sU and sT) while the main
    stream's GEMMs run, so the skinny kernels fill SMs that a GEMM's last wave
    leaves idle. The step forks and joins, so steps never overlap each other."""
    import torch
    main = torch.cuda.current_stream()
    stream, e_fork, e_su, e_st, e_done = side
    e_fork.record(main)
    stream.wait_event(e_fork)
    q.lora_dyb(d["dY"], d["B"], s, d["sT"], d["ws"], stream=stream)
    e_st.record(stream)
    q.lora_xa(d["X"], d["A"], s, d["sU"], d["ws"])
    e_su.record(main)
    stream.wait_event(e_su)
    q.lora_grads(d["X"], d["dY"], d["sU"], d["sT"], d["dA"], d["dB"], d["ws"], stream=stream)
    e_done.record(stream)
    if ev is not None:
        ev[0].record()
    q.fused_fwd(d["q"], d["X"], d["B"], d["sU"], d["Y"], ws=d["gws"])
    if ev is not None:
        ev[1].record()
    main.wait_event(e_st)
    if ev is not None:
        ev[2].record()
    q.fused_dx(d["q"], d["dY"], d["A"], d["sT"], d["dX"], ws=d["gws"])
    if ev is not None:
        ev[3].record()
    main.wait_event(e_done)


LAUNCHES_PER_STEP = 5   # lora_xa, fused_fwd, lora_dyb, fused_dx, lora_grads: one kernel each


def profile_traffic(kernel_file_hash):
    """dram bytes per launch of the fused GEMM from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "fused_nf4_gemm_attn_proj_7b.md")
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if line.startswith("- ") and ":" in line:
                    k, v = line[2:].split(":", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("kernel_source_sha256") != kernel_file_hash:
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


def kernel_source_hash():
    h = hashlib.sha256()
    for name in ("qlora_gemm.cu", "qlora_device.cuh"):
        with open(os.path.join(ROOT, "bit_nf4_quantized_dequant_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ---------------------------------------------------------------------------
# extras on the 8B linear set: standalone dequant and the 8-token forward
# ---------------------------------------------------------------------------
def eight_b_set(q, torch):
    from bit_nf4_quantized_dequant_b200 import inputs
    wl = inputs.WORKLOADS["set_8b"]
    g = torch.Generator(device="cuda")
    mats = []
    for i, lin in enumerate(wl.linears):
        g.manual_seed(1000 + i)
        Wf = torch.randn((lin.N, lin.K), generator=g, device="cuda", dtype=torch.float32) * 0.02
        mats.append((lin, q.nf4_quantize(Wf)))
        del Wf
    torch.cuda.synchronize()
    return mats


def bench_quantize(q, torch, steps, warmup):
    """a1-a3 (blockwise absmax, NF4 encode + pack, double quantisation) from
    fp32 weights resident in HBM, over the seven linears of one 8B layer
    (218 M weights); algorithmic bytes: 4 B read + 0.516 B written per weight."""
    from bit_nf4_quantized_dequant_b200 import inputs
    wl = inputs.WORKLOADS["set_8b"]
    g = torch.Generator(device="cuda")
    g.manual_seed(4040)
    layer = wl.linears[:len({lin.name for lin in wl.linears})]
    Ws = [torch.randn((lin.N, lin.K), generator=g, device="cuda", dtype=torch.float32) * 0.02 for lin in layer]
    outs = [q.nf4_quantize(W) for W in Ws]
    moved = sum(lin.N * lin.K * 4 + sum(q.nf4_sizes(lin.N, lin.K)) for lin in layer)
    for _ in range(warmup):
        for W, o in zip(Ws, outs):
            q.nf4_quantize(W, out=o)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        for W, o in zip(Ws, outs):
            q.nf4_quantize(W, out=o)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del Ws, outs
    return {"workload": "quantize fp32 -> NF4 + double quant: the 7 linears of one set_8b layer",
            "GB/s": moved / ms / 1e6, "bytes_per_pass": moved, "ms_per_pass": ms, "launches_per_pass": len(layer)}


def bench_dequant(q, torch, mats, steps, warmup):
    outs = [torch.empty((lin.N, lin.K), dtype=torch.bfloat16, device="cuda") for lin, _ in mats]
    moved = sum(lin.N * lin.K * 2 + sum(q.nf4_sizes(lin.N, lin.K)) for lin, _ in mats)
    for _ in range(warmup):
        for (lin, m), o in zip(mats, outs):
            q.nf4_dequantize(m, out=o)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        for (lin, m), o in zip(mats, outs):
            q.nf4_dequantize(m, out=o)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del outs
    return {"workload": "set_8b dequant: 224 matrices (32 layers x 7) to bf16", "GB/s": moved / ms / 1e6,
            "bytes_per_pass": moved, "ms_per_pass": ms, "launches_per_pass": len(mats)}


def bench_merge(q, torch, mats, steps, warmup):
    """Adapter merge W' + s B A to bf16 over the 8B set (r=16): HBM-bound like
    the standalone dequantisation (0.516 B read + 2 B written per weight)."""
    r, s = 16, 2.0
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    outs = [torch.empty((lin.N, lin.K), dtype=torch.bfloat16, device="cuda") for lin, _ in mats]
    adapters = {}
    for lin, _ in mats:
        if (lin.N, lin.K) not in adapters:
            adapters[(lin.N, lin.K)] = ((torch.randn((r, lin.K), generator=g, device="cuda") / r).bfloat16(),
                                        (torch.randn((lin.N, r), generator=g, device="cuda") * 0.01).bfloat16())
    moved = sum(lin.N * lin.K * 2 + sum(q.nf4_sizes(lin.N, lin.K)) + 2 * r * (lin.N + lin.K) for lin, _ in mats)

    def one_pass():
        for (lin, m), o in zip(mats, outs):
            A, B = adapters[(lin.N, lin.K)]
            q.nf4_merge(m, A, B, s, out=o)

    for _ in range(warmup):
        one_pass()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one_pass()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del outs
    return {"workload": "set_8b merge W' + s B A (r=16) of 224 matrices to bf16", "GB/s": moved / ms / 1e6,
            "bytes_per_pass": moved, "ms_per_pass": ms, "launches_per_pass": len(mats)}


def bench_decode(q, torch, mats, steps, warmup, grouping="layer"):
    """Forward of every linear of the 8B set at 8 tokens, captured once in a
    CUDA graph and replayed as a serving loop would run it. grouping="layer"
    follows a decoder layer: q, k and v read one input and run as one grouped
    launch, then o, then gate and up (one launch), then down; each launch may
    start streaming its weights while the one before it finishes
    (QLORA_FWD_OVERLAP_PREVIOUS) but reads its activations only after.
    grouping="set" treats the 224 linears as independent problems, 16 per
    launch (an upper bound on what the launch structure costs)."""
    M, r = 8, 16
    s = 2.0
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    xs = {}
    moved = 0
    probs = []
    for lin, m in mats:
        if lin.K not in xs:
            xs[lin.K] = (torch.randn((M, lin.K), generator=g, device="cuda")).to(torch.bfloat16)
        A = (torch.randn((r, lin.K), generator=g, device="cuda") / r).to(torch.bfloat16)
        B = (torch.randn((lin.N, r), generator=g, device="cuda") * 0.01).to(torch.bfloat16)
        Y = torch.empty((M, lin.N), dtype=torch.bfloat16, device="cuda")
        sU = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        probs.append((lin, q.LinearProblem(m, xs[lin.K], A, B, s, Y, sU)))
        moved += sum(q.nf4_sizes(lin.N, lin.K)) + 2 * r * (lin.N + lin.K) + 2 * M * (lin.N + lin.K)
    groups = []
    if grouping == "layer":
        together = {"q": "qkv", "k": "qkv", "v": "qkv", "gate": "gu", "up": "gu"}
        i = 0
        while i < len(probs):
            grp = together.get(probs[i][0].name)
            j = i + 1
            while grp is not None and j < len(probs) and together.get(probs[j][0].name) == grp:
                j += 1
            groups.append([p for _, p in probs[i:j]])
            i = j
    else:
        groups = [[p for _, p in probs[i:i + 16]] for i in range(0, len(probs), 16)]
    ws = torch.zeros(max(q.linear_fwd_group_workspace(grp, M) for grp in groups), dtype=torch.uint8, device="cuda")
    arrs = [q._binding._problem_array(grp) for grp in groups]

    def one_pass():
        for grp, arr in zip(groups, arrs):
            q.linear_fwd_group(grp, ws=ws, flags=q.FWD_OVERLAP_PREVIOUS, arr=arr)

    for _ in range(warmup):
        one_pass()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        one_pass()
    graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del graph
    gbs = moved / ms / 1e6
    peaks, kind = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    layout = ("4 grouped launches per layer (q+k+v, o, gate+up, down), each overlapping the previous one's tail"
              if grouping == "layer" else "224 independent linears, 16 per launch")
    return {"workload": "set_8b forward at 8 tokens: 224 matrices, r=16", "GB/s": gbs,
            "bytes_per_pass": moved, "ms_per_pass": ms, "launches_per_pass": len(groups),
            "launch": "CUDA graph of the pass; " + layout,
            "roofline": {"kernel": "nf4_small_m_kernel", "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "peak_kind": f"{kind} HBM copy"}}


def codec_error(q, torch):
    """RMSE of NF4, of the evenly spaced int4 comparison codebook (same
    format) and of NF4 with the fp8 mean-centred second level, on the
    attention-projection weight, through the GPU codecs."""
    from bit_nf4_quantized_dequant_b200 import inputs
    W = torch.from_numpy(inputs.weight_f32(4096, 4096, index=0, outliers=True)).cuda()
    out = {"workload": "attn_proj_7b weight 4096x4096, N(0, 0.02) with 0.1% x8 outliers"}
    for name, book in (("nf4", q.CODEBOOK_NF4), ("int4", q.CODEBOOK_INT4)):
        back = q.codec_dequantize(q.codec_quantize(W, book), book).float()
        out[f"rmse_{name}"] = torch.sqrt(torch.mean((back - W) ** 2)).item()
    back = q.dqfp8_dequantize(q.dqfp8_quantize(W)).float()
    out["rmse_nf4_fp8_second_level"] = torch.sqrt(torch.mean((back - W) ** 2)).item()
    out["nf4_over_int4"] = out["rmse_nf4"] / out["rmse_int4"]
    out["fp8_over_linear_second_level"] = out["rmse_nf4_fp8_second_level"] / out["rmse_nf4"]
    return out


def bench_adamw8(q, torch, steps, warmup):
    """The adapter-gradient launch with the 8-bit AdamW step of A and B fused
    into its epilogue, against the gradients followed by two standalone steps,
    on the attention projection (4096 x 4096, 2048 tokens, r = 16)."""
    M, N, K, r = 2048, 4096, 4096, 16
    g = torch.Generator(device="cuda")
    g.manual_seed(5151)
    bf = lambda *shape: torch.randn(*shape, generator=g, device="cuda").bfloat16()
    X, dY, sU, sT = bf(M, K), bf(M, N), bf(M, r), bf(M, r)
    Am = torch.randn(K, r, generator=g, device="cuda") / r
    Bm = torch.randn(N, r, generator=g, device="cuda") * 0.01
    Ab, Bb = torch.empty(r, K, dtype=torch.bfloat16, device="cuda"), torch.empty(N, r, dtype=torch.bfloat16, device="cuda")
    dA, dB = torch.empty(r, K, device="cuda"), torch.empty(N, r, device="cuda")
    dAt = torch.empty(K, r, device="cuda")
    ws = torch.zeros(q.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")
    sA, sB = q.AdamW8State(K * r), q.AdamW8State(N * r)

    def fused():
        q.lora_grads_adamw8(X, dY, sU, sT, Am, Bm, sA, sB, 1e-4, A_bf16=Ab, B_bf16=Bb)

    def separate():
        q.lora_grads(X, dY, sU, sT, dA, dB, ws)
        dAt.copy_(dA.t())
        q.adamw8_step(Am.view(-1), dAt.view(-1), sA, 1e-4, p_bf16=Ab)
        q.adamw8_step(Bm.view(-1), dB.view(-1), sB, 1e-4, p_bf16=Bb)

    out = {"workload": "adapter gradients + 8-bit AdamW of A [16 x 4096] and B [4096 x 16], 2048 tokens"}
    for name, fn in (("fused_us", fused), ("separate_us", separate)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / steps * 1e3
    return out


def bench_mlp_chain(q, torch, steps, warmup):
    """Llama-7B SiLU-gated MLP (gate/up 4096->11008, down 11008->4096), 4096
    tokens, r=16, alpha=32, one training step with gradient checkpointing:
    forward, recompute of the layer's internals, backward (dX, dA, dB; no dW).
    Two schedules of the same chain: three separate QLoRA linears with
    silu(g) * u in torch between them, and the fused SwiGLU projection (gate
    and up in one GEMM, h in its epilogue, g and u recomputed inside the
    backward GEMM). Useful flops: 4 M N K per linear (fwd + dX)."""
    import torch.nn.functional as Fn
    H, F, M, r, s = 4096, 11008, 4096, 16, 2.0
    g = torch.Generator(device="cuda")
    g.manual_seed(4242)
    rnd = lambda *shape, std=1.0: torch.randn(*shape, generator=g, device="cuda") * std
    Wg, Wu, Wd = rnd(F, H, std=0.02), rnd(F, H, std=0.02), rnd(H, F, std=0.02)
    qg, qu, qd = q.nf4_quantize(Wg), q.nf4_quantize(Wu), q.nf4_quantize(Wd)
    qgu = q.nf4_quantize(q.swiglu_interleave(Wg, Wu))
    del Wg, Wu, Wd
    bf = lambda t: t.bfloat16()
    Ag, Au, Ad = bf(rnd(r, H, std=1 / r)), bf(rnd(r, H, std=1 / r)), bf(rnd(r, F, std=1 / r))
    Bg, Bu, Bd = bf(rnd(F, r, std=0.01)), bf(rnd(F, r, std=0.01)), bf(rnd(H, r, std=0.01))
    X, dY = bf(rnd(M, H)), bf(rnd(M, H))
    Agu, Bgu = torch.cat([Ag, Au]), q.swiglu_pack_b(Bg, Bu)
    ws_gu = torch.zeros(q.linear_workspace(M, 2 * F, H, 2 * r), dtype=torch.uint8, device="cuda")
    ws_g = torch.zeros(q.linear_workspace(M, F, H, r), dtype=torch.uint8, device="cuda")
    ws_d = torch.zeros(q.linear_workspace(M, H, F, r), dtype=torch.uint8, device="cuda")
    e = lambda *shape, dt=torch.bfloat16: torch.empty(*shape, dtype=dt, device="cuda")
    b = dict(g=e(M, F), u=e(M, F), h=e(M, F), y=e(M, H), dh=e(M, F), dX=e(M, H), dXu=e(M, H),
             sUg=e(M, r), sUu=e(M, r), sUd=e(M, r), sUgu=e(M, 2 * r), sTgu=e(M, 2 * r), dGU=e(M, 2 * F),
             dAg=e(r, H, dt=torch.float32), dBg=e(F, r, dt=torch.float32), dAu=e(r, H, dt=torch.float32),
             dBu=e(F, r, dt=torch.float32), dAd=e(r, F, dt=torch.float32), dBd=e(H, r, dt=torch.float32),
             dAgu=e(2 * r, H, dt=torch.float32), dBgu=e(2 * F, 2 * r, dt=torch.float32))

    def unfused():
        for _ in range(2):   # forward, then the recompute before the backward
            q.linear_fwd(qg, X, Ag, Bg, s, Y=b["g"], sU=b["sUg"], ws=ws_g)
            q.linear_fwd(qu, X, Au, Bu, s, Y=b["u"], sU=b["sUu"], ws=ws_g)
            torch.mul(Fn.silu(b["g"]), b["u"], out=b["h"])
        q.linear_fwd(qd, b["h"], Ad, Bd, s, Y=b["y"], sU=b["sUd"], ws=ws_d)
        q.linear_bwd(qd, b["h"], Ad, Bd, s, dY, sU=b["sUd"], dX=b["dh"], dA=b["dAd"], dB=b["dBd"], ws=ws_d)
        gf, uf, dhf = b["g"].float(), b["u"].float(), b["dh"].float()
        sig = torch.sigmoid(gf)
        dg = (dhf * uf * sig * (1 + gf * (1 - sig))).bfloat16()
        du = (dhf * Fn.silu(gf)).bfloat16()
        q.linear_bwd(qg, X, Ag, Bg, s, dg, sU=b["sUg"], dX=b["dX"], dA=b["dAg"], dB=b["dBg"], ws=ws_g)
        q.linear_bwd(qu, X, Au, Bu, s, du, sU=b["sUu"], dX=b["dXu"], dA=b["dAu"], dB=b["dBu"], ws=ws_g)
        b["dX"].add_(b["dXu"])

    def fused():
        q.lora_xa(X, Agu, s, b["sUgu"], ws_gu)
        q.swiglu_fwd(qgu, X, Bgu, b["sUgu"], H=b["h"])
        q.linear_fwd(qd, b["h"], Ad, Bd, s, Y=b["y"], sU=b["sUd"], ws=ws_d)
        q.swiglu_fwd(qgu, X, Bgu, b["sUgu"], H=b["h"])                   # recompute
        q.linear_bwd(qd, b["h"], Ad, Bd, s, dY, sU=b["sUd"], dX=b["dh"], dA=b["dAd"], dB=b["dBd"], ws=ws_d)
        q.swiglu_bwd(qgu, X, Bgu, b["sUgu"], b["dh"], dGU=b["dGU"])      # g, u recomputed inside
        q.lora_dyb(b["dGU"], Bgu, s, b["sTgu"], ws_gu)
        q.fused_dx(qgu, b["dGU"], Agu, b["sTgu"], b["dX"])
        q.lora_grads(X, b["dGU"], b["sUgu"], b["sTgu"], b["dAgu"], b["dBgu"], ws_gu)
        q.swiglu_unpack_db(b["dBgu"], b["dBg"], b["dBu"])

    out = {"workload": "mlp_7b: gate/up 4096->11008, down 11008->4096, 4096 tokens, r=16, "
                       "forward + recompute + backward"}
    useful = 3 * 4 * M * F * H
    for name, fn, executed in (("unfused", unfused, 3 * 6 * M * F * H), ("fused_swiglu", fused, 20 * M * F * H)):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        out[name] = {"ms_per_step": ms, "useful_TFLOP/s": useful / (ms * 1e-3) / 1e12,
                     "executed_TFLOP/s": executed / (ms * 1e-3) / 1e12}
    return out


def bench_stack(q, torch, name, mats, steps, warmup):
    """fwd+bwd of every linear of a model's linear set (the 3B decoder stack
    at 2048 tokens, the 8B set at 4096 tokens): each linear is one run_step
    (the five-launch DAG) over its own NF4 weight and adapter, in layer order.
    Activations and output gradients rotate over two layers' worth of buffers
    (several hundred MB, > L2); q, k, v read the same X, as do gate and up."""
    from bit_nf4_quantized_dequant_b200 import inputs
    wl = inputs.WORKLOADS[name]
    M, r, s = wl.M, wl.r, wl.s
    g = torch.Generator(device="cuda")
    g.manual_seed(7000)
    rnd = lambda *shape, std=1.0: (torch.randn(*shape, generator=g, device="cuda") * std).bfloat16()
    if mats is None:
        mats = []
        for i, lin in enumerate(wl.linears):
            Wf = torch.randn((lin.N, lin.K), generator=g, device="cuda", dtype=torch.float32) * 0.02
            mats.append((lin, q.nf4_quantize(Wf)))
            del Wf
    shapes = sorted({(lin.N, lin.K) for lin, _ in mats})
    acts = [{nk: dict(X=rnd(M, nk[1]), dY=rnd(M, nk[0])) for nk in shapes} for _ in range(2)]
    e = lambda *shape, dt=torch.bfloat16: torch.empty(*shape, dtype=dt, device="cuda")
    outs = {(N, K): dict(Y=e(M, N), dX=e(M, K), dA=e(r, K, dt=torch.float32), dB=e(N, r, dt=torch.float32))
            for N, K in shapes}
    ws = torch.zeros(max(q.linear_workspace(M, N, K, r) for N, K in shapes), dtype=torch.uint8, device="cuda")
    gws = torch.zeros(q.fused_workspace(M), dtype=torch.uint8, device="cuda")
    sU, sT = e(M, r), e(M, r)
    per_layer = len({lin.name for lin in wl.linears})   # q, k, v, o, gate, up, down
    steps_d = []
    for i, (lin, m) in enumerate(mats):
        nk = (lin.N, lin.K)
        d = dict(q=m, A=rnd(r, lin.K, std=1 / r), B=rnd(lin.N, r, std=0.01), sU=sU, sT=sT, ws=ws, gws=gws)
        d.update(acts[(i // per_layer) % 2][nk])
        d.update(outs[nk])
        steps_d.append(d)
    side = make_side(torch)

    def one_pass():
        for d in steps_d:
            run_step(q, d, s, side=side)

    for _ in range(warmup):
        one_pass()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one_pass()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = sum(step_flops(M, lin.N, lin.K, r) for lin, _ in mats)
    return {"workload": wl.description + ", fwd+bwd of every linear (no dW)", "TFLOP/s": flops / (ms * 1e-3) / 1e12,
            "ms_per_pass": ms, "flops_per_pass": flops, "launches_per_pass": LAUNCHES_PER_STEP * len(mats)}


# ---------------------------------------------------------------------------
# CPU oracle (bounded sample)
# ---------------------------------------------------------------------------
def oracle_sample(min_seconds=10.0, max_reps=4):
    """The oracle as it stands on one full step of the attention-projection
    workload: dequantise W, forward and backward over all 2048 tokens."""
    import numpy as np
    from oracle import linear as olin, nf4 as onf4
    from bit_nf4_quantized_dequant_b200 import inputs
    wl = inputs.WORKLOADS[WORKLOAD]
    lin = wl.linears[0]
    N, K, M, r, s = lin.N, lin.K, wl.M, wl.r, wl.s
    c = inputs.linear_case(N, K, M, r, outliers=True)
    codes, s8, s2 = onf4.quantize(c["W"])
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    X, A, B, dY = f(c["X"]), f(c["A"]), f(c["B"]), f(c["dY"])
    reps, t0 = 0, time.perf_counter()
    while True:
        Wd = onf4.dequantize(codes, s8, s2, N, K)
        olin.linear_fwd(Wd, X, A, B, s)
        olin.linear_bwd(Wd, X, A, B, s, dY)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    try:
        import threadpoolctl
        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        cores = os.cpu_count()
    flops = step_flops(M, N, K, r) * reps
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} full step(s) of {WORKLOAD} (dequantise W 4096x4096, fwd+bwd over 2048 tokens) "
                      f"in numpy float64, {el:.1f} s"}


def bench_linear_1k(q, torch, steps, warmup):
    """The single 1024x1024 linear (64 tokens, r = 8, alpha = 16): a latency
    case. fwd+bwd through the composite calls, timed back to back (each call
    launched from Python) and as a replayed CUDA graph of the same launches."""
    from bit_nf4_quantized_dequant_b200 import inputs
    wl = inputs.WORKLOADS["linear_1k"]
    lin = wl.linears[0]
    N, K, M, r, s = lin.N, lin.K, wl.M, wl.r, wl.s
    c = inputs.linear_case(N, K, M, r)
    dev = lambda b: torch.from_numpy(b.view("int16")).view(torch.bfloat16).cuda()
    qw = q.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    X, A, B, dY = dev(c["X"]), dev(c["A"]), dev(c["B"]), dev(c["dY"])
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sU = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
    dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
    ws = torch.zeros(q.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")

    def step():
        q.linear_fwd(qw, X, A, B, s, Y=Y, sU=sU, ws=ws)
        q.linear_bwd(qw, X, A, B, s, dY, sU=sU, dX=dX, dA=dA, dB=dB, ws=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    eager_us = e0.elapsed_time(e1) / steps * 1e3
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    graph_us = e0.elapsed_time(e1) / steps * 1e3
    del g
    fl = step_flops(M, N, K, r)
    return {"workload": wl.description, "us_per_fwd_bwd_eager": eager_us, "us_per_fwd_bwd_graph": graph_us,
            "TFLOP/s_graph": fl / (graph_us * 1e-6) / 1e12, "flops_per_step": fl,
            "launches_per_step": 5, "launches": "lora_xa, fused fwd GEMM; lora_dyb, fused dX GEMM, lora_grads"}


def oracle_configs():
    """The CPU oracle on every workload, on this machine's host cores. The
    codec (quantise + dequantise) is timed in full on the 1024x1024 and
    4096x4096 weights; larger sets use the 4096x4096 rate per weight
    ("extrapolated"). The linear fwd+bwd is timed in full for the 1024x1024,
    the attention projection and the MLP chain (forward, recompute, backward);
    for the 3B and 8B stacks one layer's seven linears are timed with
    dequantised weights and the time multiplied by the layer count
    ("extrapolated"), plus the codec's dequantisation at the measured rate."""
    import numpy as np
    from oracle import linear as olin, nf4 as onf4
    from bit_nf4_quantized_dequant_b200 import inputs
    try:
        import threadpoolctl
        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        cores = os.cpu_count()
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    out = {"cores": cores, "kind": "oracle (numpy float64)"}

    def codec(N, K):
        W = inputs.weight_f32(N, K, outliers=True)
        t0 = time.perf_counter()
        packed = onf4.quantize(W)
        t1 = time.perf_counter()
        Wd = onf4.dequantize(*packed, N, K)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1, Wd

    q1, d1, _ = codec(1024, 1024)
    q2, d2, Wd2 = codec(4096, 4096)
    qrate, drate = q2 / 4096 ** 2, d2 / 4096 ** 2   # seconds per weight

    def fwd_bwd(Wd, M, r, s, idx=0, recompute=False):
        N, K = Wd.shape
        c = inputs.linear_case(16, K, M, r, index=idx)
        X, A = f(c["X"]), f(c["A"])
        B = f(inputs.lora_b_bf16(N, r, idx))
        dY = f(inputs.grad_out_bf16(M, N, idx))
        t0 = time.perf_counter()
        olin.linear_fwd(Wd, X, A, B, s)
        if recompute:
            olin.linear_fwd(Wd, X, A, B, s)
        olin.linear_bwd(Wd, X, A, B, s, dY)
        return time.perf_counter() - t0

    wl1 = inputs.WORKLOADS["linear_1k"]
    _, _, Wd1 = codec(1024, 1024)
    t = fwd_bwd(Wd1, wl1.M, wl1.r, wl1.s)
    out["linear_1k"] = {"codec_s": q1 + d1, "fwd_bwd_s": t, "TFLOP/s": step_flops(64, 1024, 1024, 8) / t / 1e12}
    wl2 = inputs.WORKLOADS["attn_proj_7b"]
    t = fwd_bwd(Wd2, wl2.M, wl2.r, wl2.s)
    out["attn_proj_7b"] = {"codec_s": q2 + d2, "fwd_bwd_s": t, "step_s_with_dequant": t + d2,
                           "TFLOP/s": step_flops(2048, 4096, 4096, 16) / (t + d2) / 1e12}
    # MLP chain: each linear dequantised once, forward, recomputed forward, backward
    wl3 = inputs.WORKLOADS["mlp_7b"]
    tot, fl = 0.0, 0.0
    for i, lin in enumerate(wl3.linears):
        Wd = np.asarray(np.random.default_rng(i).standard_normal((lin.N, lin.K)) * 0.02)
        tot += fwd_bwd(Wd, wl3.M, wl3.r, wl3.s, idx=i, recompute=True) + drate * lin.N * lin.K
        fl += 6 * wl3.M * lin.N * lin.K
        del Wd
    w3 = sum(lin.N * lin.K for lin in wl3.linears)
    out["mlp_7b"] = {"codec_s_extrapolated": (qrate + drate) * w3, "chain_s": tot,
                     "executed_TFLOP/s": fl / tot / 1e12,
                     "note": "GEMMs timed in full; dequantisation at the measured 4096x4096 rate"}
    for name in ("stack_3b", "set_8b"):
        wl = inputs.WORKLOADS[name]
        per = len({lin.name for lin in wl.linears})
        layers = len(wl.linears) // per
        t_layer, fl_layer, w_layer = 0.0, 0.0, 0
        for i, lin in enumerate(wl.linears[:per]):
            Wd = np.random.default_rng(i).standard_normal((lin.N, lin.K)) * 0.02
            t_layer += fwd_bwd(Wd, wl.M, wl.r, wl.s, idx=i)
            fl_layer += step_flops(wl.M, lin.N, lin.K, wl.r)
            w_layer += lin.N * lin.K
            del Wd
        t_layer += drate * w_layer
        out[name] = {"fwd_bwd_s_extrapolated": t_layer * layers, "layers": layers, "one_layer_s": t_layer,
                     "TFLOP/s": fl_layer / t_layer / 1e12, "codec_s_extrapolated": (qrate + drate) * w_layer * layers}
    wl5 = inputs.WORKLOADS["set_8b"]
    w5 = sum(lin.N * lin.K for lin in wl5.linears)
    moved = w5 * (0.5 + 1 / 64 + 4 / 16384)
    out["set_8b_decode"] = {"fwd_s_extrapolated": drate * w5, "GB/s": moved / (drate * w5) / 1e9,
                            "note": "dequantisation dominates; 8-token products add < 1 %"}
    out["set_8b_dequant"] = {"s_extrapolated": drate * w5, "GB/s": (moved + 2 * w5) / (drate * w5) / 1e9}
    return out


def run_reference(args):
    rank, world, _ = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    if rank != 0:
        return
    import numpy as np
    from oracle import linear as olin, nf4 as onf4
    from bit_nf4_quantized_dequant_b200 import inputs
    wl = inputs.WORKLOADS[WORKLOAD]
    lin = wl.linears[0]
    N, K, M, r, s = lin.N, lin.K, wl.M, wl.r, wl.s
    c = inputs.linear_case(N, K, M, r, outliers=True)
    codes, s8, s2 = onf4.quantize(c["W"])
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    X, A, B, dY = f(c["X"]), f(c["A"]), f(c["B"]), f(c["dY"])

    def one(k):
        # one full step of the workload: dequantise W, fwd + bwd over all tokens
        Wd = onf4.dequantize(codes, s8, s2, N, K)
        olin.linear_fwd(Wd, X, A, B, s)
        olin.linear_bwd(Wd, X, A, B, s, dY)

    steps = max(1, min(args.steps, 60))   # about a second per step: at most a minute
    warm = min(args.warmup, 1)
    for k in range(warm):
        one(k)
    t0 = time.perf_counter()
    for k in range(steps):
        one(k)
    el = time.perf_counter() - t0
    flops = step_flops(M, N, K, r) * steps
    val = flops / el / 1e12
    try:
        import threadpoolctl
        cores = max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas")
    except Exception:
        cores = os.cpu_count()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": el / steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "N": N, "K": K, "M": M, "r": r, "alpha": wl.alpha},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{steps} full steps of {M} tokens (dequantise W + fwd + bwd), float64"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ---------------------------------------------------------------------------
def main():
    args = parse_args()
    if args.kernel_case:
        return run_kernel_case(args.kernel_case)
    if args.impl == "reference":
        run_reference(args)
        return
    if args.oracle_configs:
        print(json.dumps(oracle_configs()))
        return
    rank, world, local = init_dist()
    import torch
    torch.cuda.set_device(local)
    import bit_nf4_quantized_dequant_b200 as q
    from bit_nf4_quantized_dequant_b200 import _build, inputs
    if rank == 0:
        _build.build()
    barrier(world)
    q.library()
    peaks, peak_kind = load_peaks()

    wl = inputs.WORKLOADS[WORKLOAD]
    lin = wl.linears[0]
    N, K, M, r, s = lin.N, lin.K, wl.M, wl.r, wl.s
    per_set = set_bytes(M, N, K, r)
    n_sets = max(2, -(-3 * L2_BYTES // per_set))
    sets = make_sets(q, torch, n_sets, N, K, M, r, wl.outliers)

    side = make_side(torch)
    for k in range(max(3, args.warmup)):
        run_step(q, sets[k % n_sets], s, side=side)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    K_steps = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    e0.record()
    for k in range(K_steps):
        run_step(q, sets[k % n_sets], s, evs[k], side)
    e1.record()
    torch.cuda.synchronize()
    sampler.stop()
    barrier(world)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    ms_step = ms_total / K_steps
    flops = step_flops(M, N, K, r)
    value = replica_value(world, flops, K_steps, ms_total)

    fwd_ms = [ev[0].elapsed_time(ev[1]) for ev in evs]
    dx_ms = [ev[2].elapsed_time(ev[3]) for ev in evs]
    fused_total_ms = sum(fwd_ms) + sum(dx_ms)
    fused_total_flops = K_steps * (fused_flops("fwd", M, N, K, r) + fused_flops("dx", M, N, K, r))
    achieved = fused_total_flops / (fused_total_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    traffic = profile_traffic(kernel_source_hash())

    # end to end through the public API with pinned host buffers: each step
    # copies its inputs (X, dY) in and its results (Y, dX, dA, dB) out. The
    # copies run on two copy streams, double-buffered, so the H2D of step k+1
    # and the D2H of step k overlap the compute of the steps between them.
    d = sets[0]
    Xh = d["X"].cpu().pin_memory()
    dYh = d["dY"].cpu().pin_memory()
    outs_h = [dict(Y=torch.empty_like(d["Y"], device="cpu").pin_memory(),
                   dX=torch.empty_like(d["dX"], device="cpu").pin_memory(),
                   dA=torch.empty_like(d["dA"], device="cpu").pin_memory(),
                   dB=torch.empty_like(d["dB"], device="cpu").pin_memory()) for _ in range(2)]
    ins_d = [dict(X=torch.empty_like(d["X"]), dY=torch.empty_like(d["dY"])) for _ in range(2)]
    outs_d = [dict(Y=torch.empty_like(d["Y"]), dX=torch.empty_like(d["dX"]), dA=torch.empty_like(d["dA"]),
                   dB=torch.empty_like(d["dB"])) for _ in range(2)]
    comp, h2d_s, d2h_s = torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n):
        """n pipelined steps; returns after recording the last D2H."""
        in_ready = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        out_done = [torch.cuda.Event() for _ in range(n)]

        def h2d(k):
            with torch.cuda.stream(h2d_s):
                if k >= 2:
                    h2d_s.wait_event(comp_done[k - 2])       # the step that read this buffer is done
                b = ins_d[k % 2]
                b["X"].copy_(Xh, non_blocking=True)
                b["dY"].copy_(dYh, non_blocking=True)
                in_ready[k].record(h2d_s)

        h2d(0)
        for k in range(n):
            if k + 1 < n:
                h2d(k + 1)
            comp.wait_event(in_ready[k])
            if k >= 2:
                comp.wait_event(out_done[k - 2])             # results of step k-2 have left this buffer
            b, o = ins_d[k % 2], outs_d[k % 2]
            q.linear_fwd(d["q"], b["X"], d["A"], d["B"], s, Y=o["Y"], sU=d["sU"], ws=d["ws"])
            q.linear_bwd(d["q"], b["X"], d["A"], d["B"], s, b["dY"], sU=d["sU"], dX=o["dX"], dA=o["dA"],
                         dB=o["dB"], ws=d["ws"])
            comp_done[k].record(comp)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[k])
                for key in ("Y", "dX", "dA", "dB"):
                    outs_h[k % 2][key].copy_(o[key], non_blocking=True)
                out_done[k].record(d2h_s)
        comp.wait_event(out_done[n - 1])

    e2e_run(3)
    torch.cuda.synchronize()
    e2e_steps = max(10, K_steps // 4)
    barrier(world)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    e2e_run(e2e_steps)
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), world) / e2e_steps
    h2d_bytes = Xh.numel() * 2 + dYh.numel() * 2
    oh = outs_h[0]
    d2h_bytes = oh["Y"].numel() * 2 + oh["dX"].numel() * 2 + oh["dA"].numel() * 4 + oh["dB"].numel() * 4
    # the copies alone, for reference: the PCIe floor of this step
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(h2d_s)
    with torch.cuda.stream(h2d_s):
        for _ in range(3):
            ins_d[0]["X"].copy_(Xh, non_blocking=True)
            ins_d[0]["dY"].copy_(dYh, non_blocking=True)
    c1.record(h2d_s)
    torch.cuda.synchronize()
    h2d_ms = c0.elapsed_time(c1) / 3

    extras = {}
    if not args.no_extras:
        del sets
        torch.cuda.empty_cache()
        extras["linear_1k"] = bench_linear_1k(q, torch, steps=200, warmup=10)
        extras["quantize"] = bench_quantize(q, torch, steps=5, warmup=2)
        extras["quantize"]["frac_of_hbm"] = extras["quantize"]["GB/s"] / peaks.get("hbm_gbs", 6650.0)
        torch.cuda.empty_cache()
        mats = eight_b_set(q, torch)
        extras["dequant"] = bench_dequant(q, torch, mats, steps=5, warmup=2)
        extras["dequant"]["frac_of_hbm"] = extras["dequant"]["GB/s"] / peaks.get("hbm_gbs", 6650.0)
        torch.cuda.empty_cache()
        extras["merge"] = bench_merge(q, torch, mats, steps=5, warmup=2)
        extras["merge"]["frac_of_hbm"] = extras["merge"]["GB/s"] / peaks.get("hbm_gbs", 6650.0)
        # the forward of every linear of the 8B set at 8 tokens: as independent
        # linears (the workload's own definition, 16 per launch), and as the
        # dependent chain of a decoder layer's four launches
        extras["decode_fwd"] = bench_decode(q, torch, mats, steps=20, warmup=3, grouping="set")
        extras["decode_fwd"]["frac_of_hbm"] = extras["decode_fwd"]["GB/s"] / peaks.get("hbm_gbs", 6650.0)
        extras["decode_fwd_layer_chain"] = bench_decode(q, torch, mats, steps=20, warmup=3, grouping="layer")
        extras["decode_fwd_layer_chain"]["frac_of_hbm"] = (extras["decode_fwd_layer_chain"]["GB/s"]
                                                          / peaks.get("hbm_gbs", 6650.0))
        extras["set_8b_fwd_bwd"] = bench_stack(q, torch, "set_8b", mats, steps=3, warmup=1)
        del mats
        torch.cuda.empty_cache()
        extras["stack_3b_fwd_bwd"] = bench_stack(q, torch, "stack_3b", None, steps=3, warmup=1)
        for k in ("set_8b_fwd_bwd", "stack_3b_fwd_bwd"):
            extras[k]["frac_of_bf16_burst"] = extras[k]["TFLOP/s"] / peak
            extras[k]["frac_of_bf16_sustained"] = extras[k]["TFLOP/s"] / peaks.get(
                "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        torch.cuda.empty_cache()
        extras["mlp_chain"] = bench_mlp_chain(q, torch, steps=5, warmup=2)
        extras["codec_error"] = codec_error(q, torch)
        extras["adamw8"] = bench_adamw8(q, torch, steps=20, warmup=3)
    sampler.close()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = oracle_sample()

    # The measured peaks hold a burst figure (a GEMM timed alone) and a
    # sustained one (a GEMM loop held at the board's power cap). The timed
    # region is the kernel inside a long run of steps: when the clock sampler
    # saw the power cap active, the sustained figure is the denominator.
    clocks = sampler.summary()
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if "sw_power_cap" in clocks.get("reasons", []):
        gemm_peak, gemm_peak_kind = sustained, f"{peak_kind} bf16 sustained (sw_power_cap active in the timed region)"
    else:
        gemm_peak, gemm_peak_kind = peak, f"{peak_kind} bf16 burst"
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K_steps,
            "warmup": max(3, args.warmup),
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "N": N, "K": K, "M": M, "r": r, "alpha": wl.alpha,
                       "outliers": "0.1% of W x8", "flops_per_step": flops,
                       "l2": f"inputs rotate over {n_sets} sets of {per_set/1e6:.0f} MB (> L2)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"kernel": "fused_nf4_gemm_kernel (fwd and dX launches)", "bound": "tensor",
                         "achieved": achieved, "peak": gemm_peak, "unit": "TFLOP/s", "frac": achieved / gemm_peak,
                         "peak_kind": gemm_peak_kind, "frac_of_burst": achieved / peak,
                         "frac_of_sustained": achieved / sustained, "traffic": traffic,
                         "launch_ms_fwd": statistics.mean(fwd_ms), "launch_ms_dx": statistics.mean(dx_ms),
                         "share_of_step": fused_total_ms / (ms_step * K_steps)},
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes, "ms_per_step": e2e_ms,
                    "h2d_copy_ms_alone": h2d_ms,
                    "pipeline": "H2D of step k+1 and D2H of step k on two copy streams, double-buffered"},
            "gpu_launches": LAUNCHES_PER_STEP * K_steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
