"""Benchmark of the Flash PD-SSM forward pass on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload lm]
                    [--pass forward|backward] [--tau T]

A step is one pdssm_forward call (selection + dictionary preparation + the
whole chunked scan) over one batch of the LM-layer workload (batch 8, L 2048,
heads 32, N = P = 64, K = 16; bf16 inputs, fp32 state, bf16 y). Under
torchrun every rank runs its own batch (weak scaling; the batch shards need no
collective), the timed region is bracketed by a barrier and a device
synchronise on every rank, and the slowest rank's time is reported.

Rank 0 prints one JSON line. On one GPU the LM line also carries, unless
``--no-extras``: ``per_config`` (the tiny, Z5, long and complex workloads, each
with its dominant kernel's roofline and the oracle beside it), the original
PD-SSM's soft selection timed against the Flash path at the LM shape
(``contrast_original_pdssm``), and the fused projection + selection GEMM
(``projection``). ``--impl reference`` times the dense CPU oracle on the host
cores on a bounded sample of the same workload instead.
``--pass backward`` measures the backward pass (pdssm_scan_bwd, real or complex states)
the same way instead of the forward pass; the default is the forward pass.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "PD-SSM forward scan tokens·heads/s at LM shape; achieved HBM GB/s vs B200 peak"
BWD_METRIC = "PD-SSM backward scan tokens·heads/s (straight-through tempered softmax); achieved HBM GB/s"
UNIT = "token·heads/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# ------------------------------------------------------------ distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (the slowest rank's time)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(rank: int) -> int:
    """Each rank draws its own batch of the workload (independent problems)."""
    return 1000 + rank


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {  # NVML clocks-event-reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self._stop = threading.Event()
        self._thread = None
        self.max_mhz = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            # NVML enumerates physical devices; map through CUDA_VISIBLE_DEVICES
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = self.idx
            if vis:
                ids = [v for v in vis.split(",") if v.strip()]
                if self.idx < len(ids) and ids[self.idx].strip().isdigit():
                    phys = int(ids[self.idx])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = repr(e)
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "error": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ peaks

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


# ------------------------------------------------------------ recorded traffic

# Kernel sources whose hash a profile summary records; the DRAM traffic it
# reports is valid only for exactly these sources.
KERNEL_SOURCES = {
    "fused_scan": ["structured_sparse_selective_b200/csrc/scan_fused.cu",
                   "structured_sparse_selective_b200/csrc/sm100.cuh"],
    "chunked_phase_a": ["structured_sparse_selective_b200/csrc/scan_chunked.cu",
                        "structured_sparse_selective_b200/csrc/common.cuh"],
}


def recorded_traffic(kernel: str, workload: str):
    """dram bytes (read + write) per launch from profiles/<kernel>_<workload>.md, or None
    when there is no summary or the kernel's sources changed since it was captured."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    srcs = KERNEL_SOURCES.get(kernel)
    if not srcs or not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            k, _, v = line.strip().partition(":")
            if k in ("traffic_bytes_per_launch", "kernel_sources_sha256"):
                fields[k] = v.strip()
    h = hashlib.sha256()
    for src in srcs:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if fields.get("kernel_sources_sha256") != h.hexdigest() or "traffic_bytes_per_launch" not in fields:
        return None
    return int(fields["traffic_bytes_per_launch"])


# ------------------------------------------------------------ workload

def workload_config(sp: workloads.Spec, chunk: int, world: int):
    return {
        "workload": (f"{sp.recipe}: batch {sp.batch}, L {sp.seqlen}, heads {sp.heads}, N {sp.N}, P {sp.P}, "
                     f"K {sp.K}; logits/d/B/C/x {str(sp.in_dtype).replace('torch.', '')}, "
                     f"state {'complex64' if sp.state_complex else 'float32'}, "
                     f"y {str(sp.out_dtype).replace('torch.', '')}"),
        "batch_per_gpu": sp.batch, "seqlen": sp.seqlen, "heads": sp.heads, "N": sp.N, "P": sp.P,
        "K": sp.K, "chunk": chunk,
        "l2": "inputs larger than L2 (%.0f MB per step vs 126 MB) and an L2 flush between timed steps"
              % (sp.token_heads * sp.algorithmic_bytes_per_token_head() / 1e6),
        "parallelism": f"dp{world} (independent batch shards, no collective)",
    }


def cpu_baseline(sp: workloads.Spec, target_s: float = 12.0, seqlen_cap: int = 0):
    """The oracle as it stands, on the host cores, on (batch, head) slices of the workload:
    whole slices, or their first ``seqlen_cap`` steps (the oracle's cost per step does not
    depend on the position in the sequence)."""
    import oracle
    cores = oracle.threads()
    idx = workloads.generate_idx(sp)
    picks = []
    total = 0.0
    n = max(1, cores)
    Ls = min(sp.seqlen, seqlen_cap) if seqlen_cap else sp.seqlen

    def slice_of(b, h):
        sl_ = workloads.generate_slice(sp, b, h)
        return {k: v[:Ls] for k, v in sl_.items()}

    # one calibration slice, then enough slices for ~target_s of work
    sl = [slice_of(0, 0)]
    t0 = time.perf_counter()
    oracle.scan_slices(sl[0]["logits"][None], idx, sl[0]["d"][None], sl[0]["B"][None], sl[0]["C"][None],
                       sl[0]["x"][None], want_prod=False)
    one = time.perf_counter() - t0
    n = int(max(1, min(sp.batch * sp.heads, round(target_s / max(one, 1e-3) * cores))))
    n = max(1, (n // cores) * cores) if n >= cores else n
    for i in range(n):
        picks.append((i // sp.heads % sp.batch, i % sp.heads))
    sls = [slice_of(b, h) for b, h in picks]
    stack = {k: torch.stack([s[k] for s in sls]) for k in sls[0]}
    t0 = time.perf_counter()
    oracle.scan_slices(stack["logits"], idx, stack["d"], stack["B"], stack["C"], stack["x"], want_prod=False)
    total = time.perf_counter() - t0
    units = n * Ls
    what = "whole (batch, head) slices" if Ls == sp.seqlen else f"(batch, head) slices cut to their first {Ls} steps"
    return {"value": units / total, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} {what} x L={Ls} of the {sp.recipe} workload "
                      f"({units} token-heads), dense fp64 oracle, {total:.1f} s wall"}


def kernel_alg_bytes(sp: workloads.Spec, kernel: str):
    """Algorithmic bytes of one launch of ``kernel`` on the whole workload (None if unknown):
    what the kernel must read and write once, never workspace traffic."""
    def sz(dt):
        return torch.empty((), dtype=dt).element_size()
    units = sp.token_heads
    with_logits = sp.K * sz(sp.logits_dtype)
    return {
        "fused_scan": units * sp.algorithmic_bytes_per_token_head(with_logits=True),
        # phase A reads s, d, B, C and x of every token-head (its y_loc and chunk-state
        # writes are workspace traffic, not algorithmic)
        "chunked_phase_a": units * (sp.algorithmic_bytes_per_token_head(with_logits=False) - sp.P * sz(sp.out_dtype)),
        "chunked_phase_c": units * (4 + sp.N * (sz(sp.d_dtype) + sz(sp.in_dtype)) + sp.P * sz(sp.out_dtype)),
        "select": units * (with_logits + 4),
    }.get(kernel)


def time_forward(sp, inp, device, steps: int, warmup: int, flush: torch.Tensor, chunk: int = 0):
    """Device time of pdssm_forward on ``inp`` (already on the device): mean ms per step,
    per-kernel ms per step (CUDA events the library records around its launches), launches."""
    import structured_sparse_selective_b200 as pd
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"], chunk=chunk)
    Bt, L, H, N = inp["B"].shape
    P = inp["x"].shape[-1]
    sdt = torch.complex64 if sp.state_complex else torch.float32
    out = {"y": torch.empty(Bt, L, H, P, dtype=sp.out_dtype, device=device),
           "h_final": torch.empty(Bt, H, N, P, dtype=sdt, device=device)}
    ws = pd.alloc_workspace(pb, device)
    stream = torch.cuda.current_stream(device)

    def step():
        pd.pdssm_forward(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None, out["y"],
                         out["h_final"], None, None, None, ws, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    traces = [pd.KernelTrace(max_launches=16) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        with traces[i]:
            step()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    check = pd.pdssm_read_device_check(ws)
    if check:
        raise RuntimeError(f"device check status {check} on the {sp.recipe} workload")
    per_kernel = {}
    launches = 0
    for tr in traces:
        for name, t in tr.timings():
            per_kernel.setdefault(name, []).append(t)
            launches += 1
    ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)) / steps
    return ms, {k: sum(v) / steps for k, v in per_kernel.items()}, launches


def roofline_entry(sp, per_kernel_ms, peaks, traffic=None, traffic_source=None):
    dominant = max(per_kernel_ms, key=per_kernel_ms.get)
    alg = kernel_alg_bytes(sp, dominant)
    if alg is None:
        return None
    dom_ms = per_kernel_ms[dominant]
    achieved = alg / (dom_ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
            "peak_source": peaks["source"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "traffic_source": traffic_source, "algorithmic_bytes_per_launch": int(alg),
            "launch_ms": round(dom_ms, 4)}


def per_config(device, flush, names=("tiny", "z5", "long", "complex"), steps: int = 5, warmup: int = 3):
    """Throughput and roofline of the other configurations (one GPU), with the oracle beside each."""
    peaks = load_peaks()
    res = {}
    for name in names:
        sp = workloads.spec(name)
        on_host = sp.token_heads * sp.algorithmic_bytes_per_token_head() < 2e9
        inp = (workloads.generate(sp, seed=7) if on_host else workloads.generate_on_device(sp, seed=7, device=device))
        inp = {k: v.to(device) for k, v in inp.items()}
        ms, kms, launches = time_forward(sp, inp, device, steps, warmup, flush)
        del inp
        torch.cuda.empty_cache()
        dom = max(kms, key=kms.get)
        traffic = recorded_traffic(dom, name)
        source = f"profiles/{dom}_{name}.md (ncu capture of the same kernel sources)" if traffic is not None else None
        res[name] = {
            "workload": workload_config(sp, 0, 1)["workload"],
            "inputs": "host recipe (workloads.generate)" if on_host else "drawn on the device (same recipe)",
            "value": round(sp.token_heads / (ms / 1e3), 1), "unit": UNIT, "ms_per_step": round(ms, 4),
            "steps": steps, "warmup": warmup, "kernels_ms_per_step": {k: round(v, 4) for k, v in kms.items()},
            "gpu_launches": launches,
            "roofline": roofline_entry(sp, kms, peaks, traffic, source),
            "cpu_baseline": cpu_baseline(sp, target_s=2.0, seqlen_cap=0 if name != "complex" else 128),
        }
    return res


def contrast_original(device, flush, flash_ms: float, steps: int = 5, warmup: int = 3):
    """The original PD-SSM's selection (soft mixture of dense dictionary matrices + column-wise
    hardmax, then the scan with per-step transitions) at the LM-layer shape, timed like the
    Flash PD-SSM forward pass, and the memory each needs for its transitions."""
    import structured_sparse_selective_b200 as pd
    sp = workloads.spec("lm")
    inp = {k: v.to(device) for k, v in workloads.generate_on_device(sp, seed=8, device=device).items()}
    g = torch.Generator(device=device).manual_seed(9)
    M = torch.randn(sp.K, sp.N, sp.N, generator=g, device=device)
    Bt, L, H, N, P = sp.batch, sp.seqlen, sp.heads, sp.N, sp.P
    pbs = pd.Problem(batch=Bt, seqlen=L, heads=H, N=N, P=1, K=sp.K, chunk=0, logits_t=pd.BF16, in_t=pd.F32,
                     d_t=pd.F32, state_t=pd.F32, out_t=pd.F32, flags=0)
    wss = torch.empty(pd.pdssm_soft_select_workspace_size(pbs), dtype=torch.uint8, device=device)
    steps_t = torch.empty(Bt, L, H, N, dtype=torch.uint8, device=device)
    pb = pd.Problem(batch=Bt, seqlen=L, heads=H, N=N, P=P, K=16, chunk=0, logits_t=pd.BF16, in_t=pd.BF16,
                    d_t=pd.BF16, state_t=pd.F32, out_t=pd.BF16, flags=0)
    ws = pd.alloc_workspace(pb, device)
    y = torch.empty(Bt, L, H, P, dtype=torch.bfloat16, device=device)
    hf = torch.empty(Bt, H, N, P, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        pd.pdssm_soft_select(pbs, inp["logits"], M, 1.0, steps_t, wss, stream)
        pd.pdssm_scan_fwd_steps(pb, steps_t, inp["d"], inp["B"], inp["C"], inp["x"], None, y, hf, None, None, ws,
                                stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    traces = [pd.KernelTrace(max_launches=8) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        with traces[i]:
            step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    if pd.pdssm_read_device_check(wss) or pd.pdssm_read_device_check(ws):
        raise RuntimeError("device check failed in the original PD-SSM contrast")
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    kms = {}
    for tr in traces:
        for name, t in tr.timings():
            kms[name] = kms.get(name, 0.0) + t / steps
    units = sp.token_heads
    return {
        "what": "original PD-SSM: softmax mixture of K dense N x N dictionary matrices + column-wise hardmax "
                "per step (tensor cores), then the scan with per-step transitions; LM-layer shape",
        "original_ms_per_step": round(ms, 4), "flash_ms_per_step": round(flash_ms, 4),
        "original_over_flash": round(ms / flash_ms, 3),
        "original_value": round(units / (ms / 1e3), 1), "unit": UNIT,
        "kernels_ms_per_step": {k: round(v, 4) for k, v in kms.items()},
        "transition_bytes": {
            "dense_mixtures_if_materialised": units * N * N * 4,
            "original_per_step_index_arrays": units * N,
            "flash_dictionary": sp.K * N * 4,
            "flash_selections": units * 4,
        },
    }


def projection_entry(device, steps: int = 10, warmup: int = 3, D: int = 1024):
    """The fused projection + selection GEMM (u [Bt*L, D] x W [D, H*K], argmax epilogue) at the
    LM-layer shape with an embedding width D, against the measured bf16 tensor-core peak."""
    import structured_sparse_selective_b200 as pd
    sp = workloads.spec("lm")
    rows, HK = sp.batch * sp.seqlen, sp.heads * sp.K
    g = torch.Generator(device=device).manual_seed(10)
    u = torch.randn(sp.batch, sp.seqlen, D, generator=g, device=device).to(torch.bfloat16)
    W = (torch.randn(D, HK, generator=g, device=device) / D ** 0.5).to(torch.bfloat16)
    pb = pd.Problem(batch=sp.batch, seqlen=sp.seqlen, heads=sp.heads, N=1, P=1, K=sp.K, chunk=0, logits_t=pd.BF16,
                    in_t=pd.BF16, d_t=pd.BF16, state_t=pd.F32, out_t=pd.BF16, flags=0)
    s = torch.empty(sp.batch, sp.seqlen, sp.heads, dtype=torch.int32, device=device)
    ws = torch.zeros(256, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        pd.pdssm_select_proj(pb, D, u, W, s, None, ws, stream)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        pd.pdssm_select_proj(pb, D, u, W, s, None, ws, stream)
    b.record(stream)
    torch.cuda.synchronize(device)
    if pd.pdssm_read_device_check(ws):
        raise RuntimeError("device check failed in the projection")
    ms = a.elapsed_time(b) / steps
    peaks = load_peaks()
    tflops = 2.0 * rows * D * HK / (ms / 1e3) / 1e12
    return {"what": f"s = argmax_k (u W) per head: rows {rows}, D {D}, heads x K {HK} (bf16, fp32 accumulate)",
            "ms": round(ms, 4), "roofline": {"bound": "tensor", "achieved": round(tflops, 1),
                                              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                              "frac": round(tflops / peaks["bf16_tflops"], 4),
                                              "peak_source": peaks["source"]},
            "inputs_l2_resident": "u and W (34 MB) stay in L2 across the back-to-back launches"}


# ------------------------------------------------------------- our arm

def bench_spec(args) -> workloads.Spec:
    """The workload the command line names; --batch / --seqlen shorten it (profiling captures)."""
    kw = {}
    if getattr(args, "batch", 0):
        kw["batch"] = args.batch
    if getattr(args, "seqlen", 0):
        kw["seqlen"] = args.seqlen
    return workloads.spec(args.workload, **kw)


def run_ours(args, rank, world, local):
    import structured_sparse_selective_b200 as pd

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    sp = bench_spec(args)
    inp = {k: v.to(device) for k, v in workloads.generate(sp, seed=shard_seed(rank)).items()}
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"], chunk=args.chunk)
    Bt, L, H, N = inp["B"].shape
    P = inp["x"].shape[-1]
    sdt = torch.float32 if not sp.state_complex else torch.complex64
    out = {
        "y": torch.empty(Bt, L, H, P, dtype=sp.out_dtype, device=device),
        "h_final": torch.empty(Bt, H, N, P, dtype=sdt, device=device),
        "prod_idx": torch.empty(Bt, H, N, dtype=torch.int32, device=device),
        "prod_val": torch.empty(Bt, H, N, dtype=sdt, device=device),
    }
    ws = pd.alloc_workspace(pb, device)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        pd.pdssm_forward(pb, inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None,
                         out["y"], out["h_final"], out["prod_idx"], out["prod_val"], None, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    # ---- headline: K device-timed steps, L2 flushed between steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    traces = [pd.KernelTrace(max_launches=16) for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            with traces[i]:
                step()
            ends[i].record(stream)
        torch.cuda.synchronize(device)
    barrier(world, device)
    # a bounded wait that gave up, or a range error, voids the measurement
    check = pd.pdssm_read_device_check(ws)
    if check:
        raise RuntimeError(f"device check status {check} after the timed steps")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_local = sum(step_ms) / len(step_ms)
    ms = max_over_ranks(ms_local, world, device)
    per_kernel = {}
    launches = 0
    for tr in traces:
        for name, t in tr.timings():
            per_kernel.setdefault(name, []).append(t)
            launches += 1
    totals = {k: sum(v) for k, v in per_kernel.items()}
    dominant = max(totals, key=totals.get)
    dom_ms = sum(per_kernel[dominant]) / len(per_kernel[dominant])
    units = sp.token_heads
    value = units * world / (ms / 1e3)

    # ---- algorithmic bytes of the dominant kernel (per launch)
    with_logits = sp.K * torch.empty((), dtype=sp.logits_dtype).element_size()
    bytes_fwd = units * sp.algorithmic_bytes_per_token_head(with_logits=True)
    alg_bytes = {
        "fused_scan": bytes_fwd,
        # phase A reads s, d, B, C and x of every token-head (its y_loc and
        # chunk-state writes are workspace traffic, not algorithmic)
        "chunked_phase_a": units * (4 + sp.algorithmic_bytes_per_token_head(with_logits=False) - 4
                                    - sp.P * torch.empty((), dtype=sp.out_dtype).element_size()),
        "chunked_phase_c": units * (4 + sp.N * (torch.empty((), dtype=sp.d_dtype).element_size()
                                                + torch.empty((), dtype=sp.in_dtype).element_size())
                                    + sp.P * torch.empty((), dtype=sp.out_dtype).element_size()),
        "select": units * (with_logits + 4),
    }.get(dominant)
    peaks = load_peaks()
    traffic = None if (args.batch or args.seqlen) else recorded_traffic(dominant, args.workload)
    traffic_source = (f"profiles/{dominant}_{args.workload}.md (ncu capture of the same kernel sources)"
                      if traffic is not None else None)
    roofline = None
    if alg_bytes is not None:
        achieved = alg_bytes / (dom_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1),
                    "peak": peaks["hbm_gbs"], "peak_source": peaks["source"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                    "traffic_source": traffic_source,
                    "algorithmic_bytes_per_launch": int(alg_bytes), "launch_ms": round(dom_ms, 4)}

    # ---- end to end through the public API with host buffers. Every step uploads its
    # inputs from pinned host memory, runs pdssm_forward and downloads y and h_final, as
    # a serving loop does: the upload of step i + 1 and the download of step i - 1 run on
    # their own streams (the copy engines) while step i computes, with two device buffer
    # sets; the timed region covers every step's copies, from the first upload to the
    # last download.
    host_in = {k: v.cpu().pin_memory() for k, v in inp.items()}
    sets = [{"in": {k: torch.empty_like(v) for k, v in inp.items()},
             "out": {k: torch.empty_like(v) for k, v in out.items()},
             "host_y": torch.empty_like(out["y"], device="cpu").pin_memory(),
             "host_h": torch.empty_like(out["h_final"], device="cpu").pin_memory()} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(st["host_y"].numel() * st["host_y"].element_size() + st["host_h"].numel() * st["host_h"].element_size()
              for st in sets[:1])
    s_up, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]
    e2e_launched = [0]

    def e2e_step(i):
        j = i % 2
        st = sets[j]
        if e2e_launched[0] > j:  # buffer set j was used two steps ago
            s_up.wait_event(ev_fwd[j])  # its inputs are read
            stream.wait_event(ev_down[j])  # its outputs are downloaded
        with torch.cuda.stream(s_up):
            for k in st["in"]:
                st["in"][k].copy_(host_in[k], non_blocking=True)
            ev_up[j].record(s_up)
        stream.wait_event(ev_up[j])
        o = st["out"]
        pd.pdssm_forward(pb, st["in"]["logits"], st["in"]["idx"], st["in"]["d"], st["in"]["B"], st["in"]["C"],
                         st["in"]["x"], None, o["y"], o["h_final"], o["prod_idx"], o["prod_val"], None, ws, stream)
        ev_fwd[j].record(stream)
        s_down.wait_event(ev_fwd[j])
        with torch.cuda.stream(s_down):
            st["host_y"].copy_(o["y"], non_blocking=True)
            st["host_h"].copy_(o["h_final"], non_blocking=True)
            ev_down[j].record(s_down)
        e2e_launched[0] += 1

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(device)
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize(device)
    e_s.record(stream)
    s_up.wait_stream(stream)  # the first upload starts after the start event
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(ev_down[(args.steps - 1) % 2])
    e_e.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e_s.elapsed_time(e_e) / args.steps, world, device)
    check = pd.pdssm_read_device_check(ws)
    if check:
        raise RuntimeError(f"device check status {check} after the end-to-end steps")

    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(sp, args.chunk, world),
            "roofline": roofline,
            "kernels_ms_per_step": {k: round(sum(v) / args.steps, 5) for k, v in per_kernel.items()},
            "e2e": {"value": round(units * world / (e2e_ms / 1e3), 1), "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
        }
    return result


# ------------------------------------------------------------ backward pass

def bwd_bytes_per_token_head(sp: workloads.Spec) -> int:
    """Bytes the backward pass must move per (b, t, h): s, logits, d, B, C, x and dy read once,
    dd, dB, dC, dx and dlogits (float32) written once."""
    def sz(dt):
        return torch.empty((), dtype=dt).element_size()
    reads = 4 + sp.K * sz(sp.logits_dtype) + sp.N * sz(sp.d_dtype) + 2 * sp.N * sz(sp.in_dtype)
    reads += sp.P * sz(sp.in_dtype) + sp.P * sz(sp.out_dtype)
    state = 8 if sp.state_complex else 4  # dd has the state's type
    return reads + sp.N * state + (2 * sp.N + sp.P + sp.K) * 4


def run_ours_backward(args, rank, world, local):
    import structured_sparse_selective_b200 as pd

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    sp = bench_spec(args)
    if sp.state_complex:  # ~10 GB of inputs: drawn on the device (same recipe, other numbers)
        inp = workloads.generate_on_device(sp, seed=shard_seed(rank), device=device)
    else:
        inp = {k: v.to(device) for k, v in workloads.generate(sp, seed=shard_seed(rank)).items()}
    fwd = pd.forward(inp["logits"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], want_s=True,
                     want_prod=False)
    gen = torch.Generator(device=device).manual_seed(shard_seed(rank))
    sdt = torch.complex64 if sp.state_complex else torch.float32
    dy = torch.randn(fwd["y"].shape, generator=gen, device=device, dtype=sdt).to(fwd["y"].dtype)
    pb = pd.make_problem(inp["logits"], inp["d"], inp["B"], inp["x"], out_dtype=dy.dtype)
    Bt, L, H, N = inp["B"].shape
    P = inp["x"].shape[-1]
    f32 = dict(dtype=torch.float32, device=device)
    fst = dict(dtype=sdt, device=device)
    gr = {"dlogits": torch.empty(Bt, L, H, sp.K, **f32), "dd": torch.empty(Bt, L, H, N, **fst),
          "dB": torch.empty(Bt, L, H, N, **f32), "dC": torch.empty(Bt, L, H, N, **f32),
          "dx": torch.empty(Bt, L, H, P, **f32), "dh0": torch.empty(Bt, H, N, P, **fst)}
    ws = torch.empty(max(1, pd.pdssm_bwd_workspace_size(pb)), dtype=torch.uint8, device=device)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        pd.pdssm_scan_bwd(pb, inp["logits"], fwd["s"], inp["idx"], inp["d"], inp["B"], inp["C"], inp["x"], None,
                          dy, None, args.tau, gr["dlogits"], gr["dd"], gr["dB"], gr["dC"], gr["dx"], gr["dh0"], ws,
                          stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    traces = [pd.KernelTrace(max_launches=8) for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            with traces[i]:
                step()
            ends[i].record(stream)
        torch.cuda.synchronize(device)
    barrier(world, device)
    check = pd.pdssm_read_device_check(ws)
    if check:
        raise RuntimeError(f"device check status {check} after the timed steps")
    ms = max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends)) / args.steps, world, device)
    per_kernel = {}
    launches = 0
    for tr in traces:
        for name, t in tr.timings():
            per_kernel.setdefault(name, []).append(t)
            launches += 1
    dom_ms = sum(per_kernel["scan_bwd"]) / len(per_kernel["scan_bwd"])
    units = sp.token_heads
    alg = units * bwd_bytes_per_token_head(sp)
    peaks = load_peaks()
    achieved = alg / (dom_ms / 1e3) / 1e9
    if rank != 0:
        return None
    return {
        "metric": BWD_METRIC, "pass": "backward", "value": round(units * world / (ms / 1e3), 1), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "c64" if sp.state_complex else "f32", "data": "synthetic",
        "config": dict(workload_config(sp, 0, world), tau=args.tau),
        "roofline": {"bound": "hbm", "kernel": "scan_bwd", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "peak_source": peaks["source"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 5),
                     "traffic": None, "algorithmic_bytes_per_launch": int(alg), "launch_ms": round(dom_ms, 4)},
        "kernels_ms_per_step": {k: round(sum(v) / args.steps, 5) for k, v in per_kernel.items()},
        "gpu_launches": launches, "clocks": clocks.summary(),
    }


def run_reference_backward(args, rank, world):
    """The backward oracle (numpy, dense fp64, one thread) on whole (batch, head) slices."""
    if rank != 0:
        return None
    from oracle import backward as obwd
    sp = bench_spec(args)
    idx = workloads.generate_idx(sp).numpy()
    # complex slices (N = 128, dense N x N products per step) are cut to their first 256 steps
    n, lcap = (1, 256) if sp.state_complex else (2, sp.seqlen)
    picks = [(i // sp.heads % sp.batch, i % sp.heads) for i in range(n)]
    sls = [workloads.generate_slice(sp, b, h) for b, h in picks]

    def np64(t):
        return (t.to(torch.complex128) if t.is_complex() else t.double()).numpy()
    stack = {k: np64(torch.stack([s_[k][:lcap] for s_ in sls])) for k in sls[0]}
    sdt = torch.complex64 if sp.state_complex else torch.float32
    dy = np64(torch.randn(n, lcap, sp.P, generator=torch.Generator().manual_seed(0), dtype=sdt).to(sp.out_dtype))

    def step():
        obwd.scan_backward(stack["logits"], idx, stack["d"], stack["B"], stack["C"], stack["x"], dy, tau=args.tau)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    sec = (time.perf_counter() - t0) / args.steps
    units = n * lcap
    value = units / sec
    cut = "whole" if lcap == sp.seqlen else f"cut to their first {lcap} steps,"
    sample = (f"each step: {n} {cut} (batch, head) slices x L={lcap} of the {sp.recipe} workload "
              f"({units} token-heads), dense fp64 backward oracle (numpy, one thread)")
    return {
        "impl": "reference", "metric": BWD_METRIC, "pass": "backward", "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "c128" if sp.state_complex else "f64", "data": "synthetic",
        "config": dict(workload_config(sp, 0, world), tau=args.tau),
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------ reference arm

def run_reference(args, rank, world):
    """The dense CPU oracle on the host cores; each step a bounded slice sample."""
    if rank != 0:
        return None
    import oracle
    sp = bench_spec(args)
    cores = oracle.threads()
    idx = workloads.generate_idx(sp)
    n = max(1, cores)
    picks = [(i // sp.heads % sp.batch, i % sp.heads) for i in range(n)]
    sls = [workloads.generate_slice(sp, b, h) for b, h in picks]
    stack = {k: torch.stack([s[k] for s in sls]) for k in sls[0]}

    def step():
        oracle.scan_slices(stack["logits"], idx, stack["d"], stack["B"], stack["C"], stack["x"], want_prod=False)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    sec = (time.perf_counter() - t0) / args.steps
    units = n * sp.seqlen
    value = units / sec
    sample = (f"each step: {n} whole (batch, head) slices x L={sp.seqlen} of the {sp.recipe} workload "
              f"({units} token-heads), dense fp64 oracle")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(sp, args.chunk, world),
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="lm", choices=list(workloads.RECIPES))
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations, the original PD-SSM contrast and the projection")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "backward"], default="forward")
    ap.add_argument("--tau", type=float, default=1.0, help="softmax temperature of the backward pass")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (shorter runs for profiling captures; 0 = full)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (profiling captures; 0 = full)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = (run_reference_backward if args.pass_ == "backward" else run_reference)(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    init_dist(world, "nccl")
    try:
        if args.pass_ == "backward":
            res = run_ours_backward(args, rank, world, local)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return 0
        res = run_ours(args, rank, world, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(bench_spec(args))
            if world == 1 and not args.no_extras and args.workload == "lm":
                dev = torch.device("cuda", local)
                flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
                res["per_config"] = per_config(dev, flush)
                res["contrast_original_pdssm"] = contrast_original(dev, flush, res["ms_per_step"])
                res["projection"] = projection_entry(dev)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
