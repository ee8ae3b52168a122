"""Throughput of the gated delta-rule recurrence on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One "step" is one chunked prefill (decay, grams, UT solve, WY factors, the
sequential state pass and the output/final-state write) of the H = 16,
d = 128, T = 8192 workload: B = 8 sequences, per-channel decay, decoupled
per-channel erase and write gates, bf16 inputs, float32 state with a random
N(0, 0.1) initial state.  `value` is tokens/s (B*T per step) over all ranks.
The same line carries the decode step's HBM bandwidth (batch 256, H = 32,
d = 128, float32 state read and written in place), the roofline fraction of
the prefill kernel, the backward pass on the same inputs (training: the
gradients of every input, its issued tensor flops against the bf16 tensor
peak, or the CUDA cores' float32 FMA peak for float32 inputs), the float64
oracle's throughput on this host, the end-to-end figure
through host buffers, and the SM clocks seen while timing.

Under torchrun each rank runs its own B = 8 batch (weak scaling, no
collective on the data path); the barrier and the max-over-ranks timing use
torch.distributed.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "gdn2_bf16"
DECODE = "decode_bf16"
METRIC = "gated delta-rule tokens/s at H=16,d=128,T=8k; % of roofline; decode GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def measured_traffic(name: str = "chunked_tc_gdn2_bf16_T1024.json"):
    """DRAM bytes per launch of the bench's prefill workload from the committed
    ncu counters (a JSON data file under profiles/), or None when the kernel
    sources it names changed since that capture."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None, None
    rec = json.load(open(path))
    if rec.get("code_sha256") != code_digest(rec.get("sources", [])):
        return None, rec.get("note")
    return int(rec["traffic_bytes_per_launch"]), rec.get("note")


def code_digest(sources) -> str:
    """sha256 of the listed sources' code with comments and blank space
    removed: a comment edit leaves the counters attached to the code they
    were taken from, any change to the code detaches them."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in sources:
        src = open(os.path.join(ROOT, rel)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def prefill_bytes(wl) -> int:
    """Algorithmic HBM bytes of one prefill: every input read once, o written
    once, s0 read and S_T written once (no intermediates)."""
    e = 2 if wl.dtype == "bf16" else 4
    th = wl.B * wl.T * wl.H
    per_th = e * (2 * wl.dk + wl.dv)                         # q, k, v
    per_th += e * (wl.dk if wl.decay == "vector" else 1)       # a
    per_th += e * (wl.dk if wl.erase == "vector" else 1)       # b
    if wl.write != "shared":
        per_th += e * (wl.dv if wl.write == "vector" else 1)   # w
    per_th += e * wl.dv                                        # o
    state = 4 * wl.B * wl.H * wl.dk * wl.dv
    return th * per_th + state * (2 if wl.random_s0 else 1)


def prefill_flops(wl) -> int:
    """Tensor-core flops of the chunked form per token-head, counted 2mnk:
    8 d^2 + 16 C d + C^2 with decoupled vector gates."""
    d, C = wl.dk, wl.chunk
    return wl.B * wl.T * wl.H * (8 * d * d + 16 * C * d + C * C)


BWD_CHUNK = 32  # the CUDA-core / mma.sync backward walks 32-token chunks


def backward_tc_path(wl) -> bool:
    """bf16, d = 128: the tensor-core backward (three launches)."""
    return wl.dtype == "bf16" and wl.dk == 128 and wl.dv == 128


def backward_flops(wl) -> int:
    """Tensor-core flops of one backward call, per token-head.
    Tensor-core path (bf16, d = 128): the state-writing prefill launch
    (8 d^2 + 16 C d + C^2 as for the prefill) plus the reverse sweep's
    products as issued, 76 K-steps of a 128 x 128 x 16 tcgen05.mma per
    64-token chunk (zero halves of padded A operands included) = 622,592.
    Otherwise, 2mnk over dense tiles: the forward sweep that stores the
    chunk-start states (6 dk dv + 4 C dk + 4 C dv) plus the reverse sweep
    (18 dk dv + 20 C dv + 24 C dk), C = 32."""
    if backward_tc_path(wl):
        d = wl.dk
        fwd = 8 * d * d + 16 * 64 * d + 64 * 64
        rev = 76 * 2 * 128 * 128 * 16 // 64
        return wl.B * wl.T * wl.H * (fwd + rev)
    dk, dv, C = wl.dk, wl.dv, BWD_CHUNK
    fwd = 6 * dk * dv + 4 * C * dk + 4 * C * dv
    rev = 18 * dk * dv + 20 * C * dv + 24 * C * dk
    return wl.B * wl.T * wl.H * (fwd + rev)


def backward_bytes(wl) -> int:
    """Algorithmic HBM bytes of one backward call: the forward's inputs and
    do read once, their gradients written once, s0 and dS_T read, dS0 written
    (no intermediates: the chunk-start states are workspace traffic)."""
    e = 2 if wl.dtype == "bf16" else 4
    th = wl.B * wl.T * wl.H
    per_th = e * (2 * wl.dk + wl.dv)                         # q, k, v
    per_th += e * (wl.dk if wl.decay == "vector" else 1)       # a
    per_th += e * (wl.dk if wl.erase == "vector" else 1)       # b
    if wl.write != "shared":
        per_th += e * (wl.dv if wl.write == "vector" else 1)   # w
    per_th = 2 * per_th + 2 * e * wl.dv                        # + gradients, do
    state = 4 * wl.B * wl.H * wl.dk * wl.dv
    return th * per_th + state * (3 if wl.random_s0 else 2)


TF32_OVER_BF16 = 1.1 / 2.25  # nominal dense tensor rates of the B200


def fp32_alu_peak_tflops(peaks) -> float:
    """FP32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flop x the
    maximum SM clock."""
    return 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12


def decode_bytes(wl) -> int:
    e = 2 if wl.dtype == "bf16" else 4
    per = 8 * wl.dk * wl.dv + e * (4 * wl.dk + 3 * wl.dv)
    return wl.B * wl.H * per


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="gdr_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(1, 5)
                          if r[3][i].lower() in ("active", "1")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "samples": len(rows),
                "samples_under_load": len(loaded), "reasons": reasons}


def config_dict(wl, world: int) -> dict:
    """The `config` object of the JSON line, the same in both arms."""
    return {"workload": "%s: B=%d T=%d H=%d dk=dv=%d chunk=%d, per-channel decay, "
                        "decoupled vector erase/write gates, s0~N(0,0.1)"
                        % (wl.name, wl.B, wl.T, wl.H, wl.dk, wl.chunk),
            "global_batch": wl.B * world, "seq_len": wl.T, "heads": wl.H,
            "parallelism": "dp%d (independent sequences per rank)" % world,
            "l2": "inputs (%.2f GB per rank) larger than L2" % (prefill_bytes(wl) / 1e9)}


# --------------------------------------------------------------- the oracle arm

def oracle_throughput(wl, seed: int, target_s: float = 15.0):
    """float64 oracle on a bounded sample of the prefill workload: every
    (b, h) of the batch over the first T_s tokens, T_s sized for about
    `target_s` seconds.  Returns (tokens/s, cores, sample description)."""
    import oracle
    from gated_delta_rule_154_b200 import workload as W

    cores = oracle.max_threads()
    # calibrate on 512 tokens: shorter runs are dominated by thread start-up
    # and overestimate the rate
    cal = wl.replace(T=min(512, wl.T))
    x = W.make_prefill(cal, seed=seed)
    f = lambda k: W.as_f32(x[k], wl.dtype)
    t = time.perf_counter()
    oracle.forward(f("q"), f("k"), f("v"), f("a"), f("b"),
                   f("w") if x["w"] is not None else f("b"), x["s0"])
    per_tok = (time.perf_counter() - t) / cal.T
    Ts = int(max(64, min(wl.T, round(target_s / max(per_tok, 1e-9)))))
    sub = wl.replace(T=Ts)
    x = W.make_prefill(sub, seed=seed)
    f = lambda k: W.as_f32(x[k], wl.dtype)
    t = time.perf_counter()
    oracle.forward(f("q"), f("k"), f("v"), f("a"), f("b"),
                   f("w") if x["w"] is not None else f("b"), x["s0"])
    dt = time.perf_counter() - t
    sample = "all %d (b,h) pairs x first %d of %d tokens (%d token-heads), float64" % (
        wl.B * wl.H, Ts, wl.T, wl.B * wl.H * Ts)
    return wl.B * Ts / dt, cores, sample, dt


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_delta_rule_154_b200 import workload as W
    wl = W.WORKLOADS[PREFILL]
    vals = []
    # each step is a bounded sample so the whole run stays within a few minutes
    per_step = min(args.ref_seconds, 150.0 / max(1, args.warmup + args.steps))
    for i in range(args.warmup + args.steps):
        v, cores, sample, dt = oracle_throughput(wl, seed=0, target_s=per_step)
        if i >= args.warmup:
            vals.append((v, dt))
    value = statistics.median(v for v, _ in vals)
    ms = statistics.median(dt for _, dt in vals) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ rank plumbing

class Ranks:
    """Barrier and max-over-ranks timing over whatever process group is
    initialised (NCCL on GPUs; gloo in the CPU tests).  A world of one needs
    no process group."""

    def __init__(self, world: int, device=None):
        self.world = world
        self.device = device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (weak scaling): seed = rank."""
    return rank


# ------------------------------------------------------------------ the GPU arm

def run_gpu(args):
    import torch
    import torch.distributed as dist

    from gated_delta_rule_154_b200 import api
    from gated_delta_rule_154_b200 import workload as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    ranks = Ranks(world, dev)
    barrier = ranks.barrier
    max_over_ranks = ranks.max

    peaks, peak_src = load_peaks()
    wl = W.WORKLOADS[PREFILL]
    if args.T:
        wl = wl.replace(T=args.T)
    inp = W.make_prefill(wl, seed=rank_seed(rank))

    def dev_t(x, dtype):
        if x is None:
            return None
        if dtype == "bf16":
            return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev)

    d = {k: dev_t(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    d["s0"] = dev_t(inp["s0"], "f32")
    o = torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=d["q"].dtype, device=dev)
    sT = torch.empty((wl.B, wl.H, wl.dk, wl.dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step():
        api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                            chunk=wl.chunk, out=o, s_final=sT, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    if api.last_device_error(stream) != 0:
        raise RuntimeError("device error during warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    clk = clocks.summary()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end))
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    ms_step = total_ms / args.steps
    if api.last_device_error(stream) != 0:
        raise RuntimeError("device error during the timed region")

    tokens_step = wl.B * wl.T * world
    value = tokens_step / (ms_step * 1e-3)
    traffic, traffic_note = measured_traffic() if wl.T == 8192 else (None, None)
    alg_bytes = prefill_bytes(wl)
    avg_launch_s = statistics.mean(launch_ms) * 1e-3
    achieved = alg_bytes / avg_launch_s / 1e9
    hbm_peak = float(peaks["hbm_gbs"])
    flops = prefill_flops(wl)
    t_tc = flops / (float(peaks["bf16_tflops"]) * 1e12)

    # ---- end to end through host buffers: pinned host inputs -> device ->
    # the library call -> o and S_T back to pinned host memory, every step.
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in d.items()}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    s_host = torch.empty(sT.shape, dtype=sT.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = o_host.numel() * o_host.element_size() + s_host.numel() * s_host.element_size()
    scratch = {k: (None if v is None else torch.empty_like(v)) for k, v in d.items()}

    def e2e_step():
        for k, v in host.items():
            if v is not None:
                scratch[k].copy_(v, non_blocking=True)
        api.forward_chunked(scratch["q"], scratch["k"], scratch["v"], scratch["a"],
                            scratch["b"], scratch["w"], scratch["s0"], chunk=wl.chunk,
                            out=o, s_final=sT, stream=stream)
        o_host.copy_(o, non_blocking=True)
        s_host.copy_(sT, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 5))
    with torch.cuda.stream(stream):
        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1)) / e2e_steps
    del scratch, host

    # ---- the same q, k, v, a under other gate forms: KDA (one scalar beta per
    # token for erase and write, here b[..., 0]) and FG^2-GDN / FG^2-GDN+
    # (vector learning rates entering through their square roots); context for
    # the FG^2-GDN page's "<5 % prefill overhead over KDA" (section 4)
    variants = None
    if not args.no_variants and wl.dtype == "bf16":
        beta_s = d["b"][..., 0].contiguous()
        kw = dict(chunk=wl.chunk, out=o, s_final=sT, stream=stream)
        runs = {
            "kda": lambda: api.forward_chunked(d["q"], d["k"], d["v"], d["a"], beta_s, beta_s,
                                               d["s0"], **kw),
            "fg2": lambda: api.forward_fg2(d["q"], d["k"], d["v"], d["a"], d["b"], None,
                                           d["s0"], **kw),
            "fg2_plus": lambda: api.forward_fg2(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"],
                                                d["s0"], **kw),
        }
        variants = {}
        for name, fn in runs.items():
            with torch.cuda.stream(stream):
                for _ in range(2):
                    fn()
                torch.cuda.synchronize()
                barrier()
                v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                v0.record(stream)
                for _ in range(5):
                    fn()
                v1.record(stream)
                torch.cuda.synchronize()
                barrier()
            vms = max_over_ranks(v0.elapsed_time(v1)) / 5
            variants[name] = {"ms_per_step": vms, "tokens/s": tokens_step / (vms * 1e-3)}
        if api.last_device_error(stream) != 0:
            raise RuntimeError("device error during the gate-form variants")
        variants["fg2_over_kda"] = variants["fg2"]["ms_per_step"] / variants["kda"]["ms_per_step"] - 1.0
        variants["note"] = ("5 launches each on the main step's q, k, v, a; kda: scalar beta = "
                            "b[..., 0] for erase and write; fg2: beta = b as sqrt(beta) on k "
                            "and v; fg2_plus: beta^k = b, beta^v = w")

    # ---- the other prefill workloads: KDA (per-channel decay, scalar beta),
    # long-context (B=1 H=32 T=65536) and the float32 Gated DeltaNet case,
    # each timed on its own with its HBM roofline (inputs drawn on the device)
    others = None
    if not args.no_other_configs:
        others = {}
        for name in ("kda_bf16", "long_bf16", "gdn_fp32"):
            owl = W.WORKLOADS[name]
            x = W.make_prefill_device(owl, seed=rank_seed(rank), device=dev)
            torch.cuda.synchronize()   # drawn on the default stream; timed on `stream`
            xw = x["w"] if x["w"] is not None else x["b"]
            oo = torch.empty((owl.B, owl.T, owl.H, owl.dv), dtype=x["q"].dtype, device=dev)
            ss = torch.empty((owl.B, owl.H, owl.dk, owl.dv), dtype=torch.float32, device=dev)
            # the library's own choice: few heads with long sequences take the
            # sequence split, which needs the workspace it asks for
            need = api.workspace_size(api.desc_for(x["q"], x["v"], x["a"], x["b"], xw,
                                                   owl.chunk))
            ows = torch.empty(max(need, 16), dtype=torch.uint8, device=dev) if need else None

            def ostep(split=True):
                api.forward_chunked(x["q"], x["k"], x["v"], x["a"], x["b"], xw, x["s0"],
                                    chunk=owl.chunk, out=oo, s_final=ss, workspace=ows,
                                    stream=stream, split=split)

            n_t = args.steps if name != "gdn_fp32" else 100
            with torch.cuda.stream(stream):
                for _ in range(3):
                    ostep()
                torch.cuda.synchronize()
                barrier()
                c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                c0.record(stream)
                for _ in range(n_t):
                    ostep()
                c1.record(stream)
                torch.cuda.synchronize()
                barrier()
            oms = max_over_ranks(c0.elapsed_time(c1)) / n_t
            err = api.last_device_error(stream)
            if err != 0:
                from gated_delta_rule_154_b200 import _lib
                raise RuntimeError("device error during the %s timing: %s"
                                   % (name, _lib.status_string(err)))
            ob = prefill_bytes(owl)
            ogbs = ob / (oms * 1e-3) / 1e9
            others[name] = {
                "workload": "%s: B=%d T=%d H=%d dk=dv=%d chunk=%d %s, decay %s, erase %s, "
                            "write %s, s0 %s" % (name, owl.B, owl.T, owl.H, owl.dk, owl.chunk,
                                                 owl.dtype, owl.decay, owl.erase, owl.write,
                                                 "N(0,0.1)" if owl.random_s0 else "0"),
                "steps": n_t, "ms_per_step": oms,
                "tokens/s": owl.B * owl.T * world / (oms * 1e-3),
                "roofline": {"bound": "hbm", "achieved": ogbs, "peak": hbm_peak, "unit": "GB/s",
                             "frac": ogbs / hbm_peak, "algorithmic_bytes_per_launch": ob,
                             "t_hbm_min_us": ob / (hbm_peak * 1e9) * 1e6}}
            others[name]["sequence_split"] = (
                "%d segments per sequence (maps, scan, second pass)" % (148 // (owl.B * owl.H))
                if need else "none (one launch)")
            if need:
                # the same inputs on the one-pass kernel, for comparison
                with torch.cuda.stream(stream):
                    for _ in range(2):
                        ostep(split=False)
                    torch.cuda.synchronize()
                    barrier()
                    c0.record(stream)
                    for _ in range(3):
                        ostep(split=False)
                    c1.record(stream)
                    torch.cuda.synchronize()
                    barrier()
                sms = max_over_ranks(c0.elapsed_time(c1)) / 3
                err = api.last_device_error(stream)
                if err != 0:
                    from gated_delta_rule_154_b200 import _lib
                    raise RuntimeError("device error during the one-launch timing: %s"
                                       % _lib.status_string(err))
                others[name + "_one_launch"] = {
                    "workload": "%s on the one-pass kernel (no sequence split)" % name,
                    "steps": 3, "ms_per_step": sms,
                    "tokens/s": owl.B * owl.T * world / (sms * 1e-3),
                    "roofline": {"bound": "hbm", "frac": ob / (sms * 1e-3) / 1e9 / hbm_peak,
                                 "algorithmic_bytes_per_launch": ob}}
            del x, xw, oo, ss, ows
        torch.cuda.empty_cache()

    # ---- backward (training): gradients of the main step's prefill for
    # seeded upstream gradients; one call = one launch (a forward sweep that
    # stores the chunk-start states, then the reverse sweep)
    bwd = None
    if not args.no_backward:
        up = W.make_upstream(wl, seed=rank_seed(rank))
        d_o = dev_t(up["do"], wl.dtype)
        dsT = dev_t(up["dsT"], "f32")
        del up
        bdesc = api.desc_for(d["q"], d["v"], d["a"], d["b"], d["w"], BWD_CHUNK)
        ws = torch.empty(api.backward_workspace_size(bdesc), dtype=torch.uint8, device=dev)

        def bstep():
            api.backward(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"], d_o, dsT,
                         workspace=ws, stream=stream)

        with torch.cuda.stream(stream):
            for _ in range(2):
                bstep()
            torch.cuda.synchronize()
            barrier()
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            for _ in range(args.backward_steps):
                bstep()
            b1.record(stream)
            torch.cuda.synchronize()
            barrier()
        bms = max_over_ranks(b0.elapsed_time(b1)) / args.backward_steps
        if api.last_device_error(stream) != 0:
            raise RuntimeError("device error during backward timing")
        bflops, bbytes = backward_flops(wl), backward_bytes(wl)
        achieved_tf = bflops / (bms * 1e-3) / 1e12
        if backward_tc_path(wl):  # tcgen05, bf16 operands: the bf16 tensor peak
            broof = {"bound": "tensor", "achieved": achieved_tf,
                     "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                     "peak_source": "%s bf16_tflops" % peak_src}
        elif wl.dtype == "bf16":  # products on tf32 mma.sync: tf32 tensor peak
            broof = {"bound": "tensor", "achieved": achieved_tf,
                     "peak": float(peaks["bf16_tflops"]) * TF32_OVER_BF16, "unit": "TFLOP/s",
                     "peak_source": "%s bf16_tflops x %.4f (nominal dense tf32 : bf16, "
                                    "1.1 : 2.25 PFLOP/s)" % (peak_src, TF32_OVER_BF16)}
        else:  # float32 inputs: CUDA-core FMA
            broof = {"bound": "alu", "achieved": achieved_tf, "peak": fp32_alu_peak_tflops(peaks),
                     "unit": "TFLOP/s",
                     "peak_source": "148 SMs x 128 FP32 lanes x 2 x sm_max_mhz"}
        broof["frac"] = achieved_tf / broof["peak"]
        broof["flops_per_step"] = bflops
        bwd = {"workload": "gradients of the main step (%s), do ~ N(0,1), dS_T ~ N(0,0.1)"
                           % wl.name,
               "steps": args.backward_steps, "ms_per_step": bms,
               "tokens/s": tokens_step / (bms * 1e-3),
               # bf16, d = 128: the tensor-core prefill writing S~, E and S_T,
               # the reverse sweep, the elementwise gradient kernel
               "launches_per_step": 3 if backward_tc_path(wl) else 1,
               "roofline": broof,
               "hbm": {"algorithmic_bytes_per_step": bbytes,
                       "GB/s": bbytes / (bms * 1e-3) / 1e9,
                       "frac": bbytes / (bms * 1e-3) / 1e9 / hbm_peak}}
        del ws, d_o, dsT

    # ---- decode: batch 256, H = 32, d = 128, float32 state in place
    dec = None
    if not args.no_decode:
        dwl = W.WORKLOADS[DECODE]
        if args.decode_batch:
            dwl = dwl.replace(B=args.decode_batch)
        state = torch.from_numpy(W.make_decode_state(dwl, seed=rank_seed(rank))).to(dev)
        # fresh inputs for every step (warm-up and timed), drawn on the device:
        # [steps, B, H, d] per tensor, 12.6 MB per step at the decode workload
        n_in = args.decode_steps + 10
        seq = W.make_decode_steps_device(dwl, n_in, seed=1000 + rank_seed(rank), device=dev)
        torch.cuda.synchronize()   # drawn on the default stream; used on `stream`
        od = torch.empty((dwl.B, dwl.H, dwl.dv), dtype=torch.bfloat16, device=dev)

        def dstep(i):
            api.decode_step(seq["q"][i], seq["k"][i], seq["v"][i], seq["a"][i], seq["b"][i],
                            seq["w"][i], state, out=od, stream=stream)

        with torch.cuda.stream(stream):
            for i in range(10):
                dstep(i)
            torch.cuda.synchronize()
            barrier()
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d0.record(stream)
            for i in range(args.decode_steps):
                dstep(10 + i)
            d1.record(stream)
            torch.cuda.synchronize()
            barrier()
        dms = max_over_ranks(d0.elapsed_time(d1)) / args.decode_steps
        if api.last_device_error(stream) != 0:
            raise RuntimeError("device error during decode timing")
        gbs = decode_bytes(dwl) / (dms * 1e-3) / 1e9
        dec = {"workload": "%s: batch %d, H=%d, dk=dv=%d, bf16 inputs, f32 state in place"
                           % (dwl.name, dwl.B, dwl.H, dwl.dk),
               "steps": args.decode_steps, "us_per_step": dms * 1e3,
               "inputs": "fresh every step (drawn on the device before timing)",
               "GB/s": gbs, "frac_of_hbm": gbs / hbm_peak,
               "bytes_per_step": decode_bytes(dwl),
               "tokens/s": dwl.B * world / (dms * 1e-3)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, _ = oracle_throughput(wl, seed=0, target_s=args.ref_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": config_dict(wl, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak,
                     "traffic": traffic,
                     "traffic_source": traffic_note,
                     "peak_source": "%s hbm_gbs" % peak_src,
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "tensor_flops_per_launch": flops,
                     "t_tensor_min_us": t_tc * 1e6,
                     "t_hbm_min_us": alg_bytes / (hbm_peak * 1e9) * 1e6},
        "decode": dec,
        "prefill_configs": others,
        "backward": bwd,
        "variants": variants,
        "e2e": {"value": tokens_step / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "cpu_baseline": cpu,
        "gpu_launches": args.steps * 1,  # prefill launches in the timed region
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--T", type=int, default=0, help="override the sequence length")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--decode-batch", type=int, default=0, help="override the decode batch")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the KDA / FG^2-GDN gate-form timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the KDA / long-context / float32 prefill timings")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward timing")
    ap.add_argument("--backward-steps", type=int, default=3)
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
