#!/usr/bin/env python
"""Benchmark of the In-Place TTT MLP layer forward (libipttt) on B200.

One step = one full layer forward (all stages: metadata, masked conv, gate/up
GEMM, target GEMM, Gram/clip pass, chunk scan with apply and update) over one
batch of the workload, inputs resident in HBM.  With --gpus N under torchrun,
every rank runs its own replica on its own batch (weak scaling, no collective on
the data path); the time is the max over ranks.

--impl reference times the fp64 CPU oracle instead (rank 0 only), on a bounded
sample of the same workload.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunk_wise_weight_gate_b200 import ipttt as ip  # noqa: E402
from chunk_wise_weight_gate_b200 import synth  # noqa: E402

METRIC = "In-Place TTT MLP layer tokens/s and TFLOP/s (% of bf16 peak) at Qwen3-4B shape"
DEFAULT_WORKLOAD = "qwen3_4b_128k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WEIGHTS = ("Wgate", "Wup", "Wdown0", "conv_w", "Wtarget")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons, power = [], [], set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, pg, device) -> float:
    """Max of x over all ranks of the default process group (identity when pg is None)."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def layer_flops(w: synth.Workload) -> int:
    """Credited flops of one step (all layers): 10 d F + 2 d^2 + 10 d per token."""
    return ip.flops_per_token(w.d, w.F) * w.B * w.T * w.layers


def phase_flops(w: synth.Workload) -> dict:
    """Algorithmic flops per call of each phase (per layer)."""
    B, T, d, F, C = w.B, w.T, w.d, w.F, w.C
    k = (T + C - 1) // C
    ct = max(1, C // 256) if C % 256 == 0 else max(1, C // 128)
    tr = C // ct
    return {
        "prep": 0,
        "gate_up": 4 * B * T * d * F,
        "target": 2 * B * T * d * d + 10 * B * T * d,
        "gram": 2 * B * k * (ct * (ct + 1) // 2) * tr * tr * (d + F),
        "apply": 4 * B * T * d * F,
        "update": 2 * B * T * d * F,
    }


def scan_step_tokens(w: synth.Workload) -> int:
    """Tokens per step of the library's chunk scan: chunks of 64, 128 or 256 tokens
    are scanned in groups of 512 tokens (one state snapshot per group), others one
    by one."""
    return 512 if w.dtype == "bf16" and w.C < 512 and 512 % w.C == 0 and w.T > w.C else w.C


def phase_bytes(w: synth.Workload, phase: str, launches: float) -> float:
    """Algorithmic DRAM bytes per call of a phase (per layer): every input read once,
    every output written once.  `launches` is the phase's launch count per layer (the
    state update reads and writes the fp32 state once per launch; the apply reads
    Wdown0 once per launch)."""
    B, T, d, F = w.B, w.T, w.d, w.F
    k = (T + scan_step_tokens(w) - 1) // scan_step_tokens(w)  # state snapshots per row (+1)
    e = 2  # bf16
    if phase == "prep":
        return 2 * B * T
    if phase == "gate_up":
        return B * T * d * e + 2 * F * d * e + B * T * F * e
    if phase == "target":
        return B * T * d * e + d * d * e + 5 * d * e + B * T * d * e
    if phase == "gram":  # Z and V read; V read and written again by the pre-scale
        return B * T * (F + d) * e + 2 * B * T * d * e
    if phase == "update":  # V, Z read; a bf16 snapshot per chunk; the fp32 state per launch
        return B * T * (F + d) * e + B * (k - 1) * d * F * e + launches * B * d * F * 4 * 2
    if phase == "apply":  # Z and every snapshot read, Wdown0 per launch, O written (H read: residual)
        return B * T * F * e + B * (k - 1) * d * F * e + launches * d * F * e + B * T * d * e * (2 if w.layers > 1 else 1)
    return 0.0


def fp32_fma_tflops(sms: int, mhz: float) -> float:
    """Peak fp32 rate of the CUDA cores: 128 fp32 lanes per SM, an FMA = 2 flops."""
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def phase_roofline(w: synth.Workload, phase: str, ms: float, launches: float, steps: int, peaks: dict) -> dict:
    """Achieved rate of one phase against the bound that limits it: the tensor time
    (algorithmic flops at the sustained bf16 peak) or the HBM time (algorithmic bytes
    at the measured copy bandwidth), whichever is longer."""
    per = launches / max(1, steps * w.layers)
    fl = phase_flops(w).get(phase, 0) * w.layers * steps
    by = phase_bytes(w, phase, per) * w.layers * steps
    tflops = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    t_tensor = fl / (tflops * 1e12)
    t_hbm = by / (peaks["hbm_gbs"] * 1e9)
    sec = max(ms, 1e-9) / 1000.0
    if t_tensor >= t_hbm:
        ach = fl / sec / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": tflops, "unit": "TFLOP/s", "frac": ach / tflops,
                "algorithmic_bytes_per_step": by / steps}
    ach = by / sec / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
            "algorithmic_bytes_per_step": by / steps, "tflops": fl / sec / 1e12}


def oracle_sample(w: synth.Workload, inp: dict, chunks: int) -> tuple[float, int]:
    """Runs the fp64 oracle on the first `chunks` chunks of row 0; returns (seconds, tokens)."""
    from oracle import ipttt_oracle as orc
    n = min(w.T, chunks * w.C)
    a = {k: inp[k][:1, :n].double().numpy() for k in ("H", "X0")}
    wts = {k: inp[k].double().numpy() for k in WEIGHTS}
    ds = inp["doc_starts"].numpy()
    ds = ds[(ds // w.T == 0) & (ds % w.T < n)]
    t0 = time.perf_counter()
    orc.layer_forward(a["H"], a["X0"], wts["Wgate"], wts["Wup"], wts["Wdown0"], wts["conv_w"], wts["Wtarget"], w.C,
                      ds, w.eta, w.clip)
    return time.perf_counter() - t0, n


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def config_dict(w: synth.Workload, n: int) -> dict:
    return {"workload": w.name, "batch": w.B, "seq_len": w.T, "chunk": w.C, "d_model": w.d, "d_ff": w.F,
            "layers": w.layers, "eta": w.eta, "clip": w.clip, "docs": w.docs,
            "global_batch": w.B * n, "parallelism": f"replicas{n}" if n > 1 else "single",
            "l2": "inputs larger than L2 (H and X0 are B*T*d bf16; Z is B*T*F bf16)"}


# DRAM bytes (read + written) per launch of a kernel, the mean over the launches of
# one step captured by ncu, keyed by (workload, chunk size, phase); the summaries in
# profiles/ give the commands.  The roofline object carries a figure only for the
# kernel and workload it was taken on.
MEASURED_TRAFFIC = {("qwen3_4b_128k", 1024, "apply"): 2514658005.3}


def sample_chunks(w: synth.Workload, tokens: int) -> int:
    """Whole chunks of row 0 covering at least `tokens` tokens (at least one chunk)."""
    k = (w.T + w.C - 1) // w.C
    return max(1, min(k, (max(1, tokens) + w.C - 1) // w.C))


def run_reference(args, w: synth.Workload):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    inp = synth.make_inputs(w.replace(B=1), seed=0)
    chunks = sample_chunks(w, args.ref_sample_tokens)
    for _ in range(args.warmup):
        oracle_sample(w, inp, chunks)
    secs, toks = 0.0, 0
    for _ in range(args.steps):
        s, n = oracle_sample(w, inp, chunks)
        secs += s
        toks += n
    value = toks / secs
    sample = f"first {chunks} chunk(s) ({toks // args.steps} tokens) of row 0 per step, fp64 numpy oracle"
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_dict(w, 1),
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_ours(args, w: synth.Workload):
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
        pg = dist

    layers = []
    for layer in range(w.layers):
        inp = synth.make_inputs(w, seed=rank, layer=layer, with_activations=(layer == 0))
        layers.append(inp)
    host = {k: layers[0][k] for k in ("H", "X0")}
    dev_in = {k: v.to(dev) for k, v in host.items()}
    dev_w = [{k: l[k].to(dev) for k in WEIGHTS} for l in layers]
    docs = layers[0]["doc_starts"]
    cfg = ip.LayerConfig(B=w.B, T=w.T, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip, dtype=w.dtype)
    ws = ip.alloc_workspace(cfg, dev, state_clip=args.state_clip)
    O = torch.empty(w.B, w.T, w.d, dtype=cfg.torch_dtype, device=dev)
    Hbuf = [torch.empty_like(dev_in["H"]) for _ in range(2)] if w.layers > 1 else None
    docs_dev = docs.to(dev)
    stream = torch.cuda.current_stream()

    def step(H, X0, out):
        if w.layers == 1:
            ip.forward(cfg, H, X0, *(dev_w[0][k] for k in WEIGHTS), docs_dev, O=out, workspace=ws,
                       state_clip=args.state_clip)
            return
        cur = H
        for l in range(w.layers):
            nxt = Hbuf[l % 2] if l + 1 < w.layers else out
            ip.forward(cfg, cur, X0, *(dev_w[l][k] for k in WEIGHTS), docs_dev, O=nxt, workspace=ws,
                       residual=True)
            cur = nxt

    for _ in range(args.warmup):
        step(dev_in["H"], dev_in["X0"], O)
    torch.cuda.synchronize()
    if ip.get_status() != 0:
        raise RuntimeError("device status set during warm-up")

    gpu_id = str(local)
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_id.startswith("GPU-"):
            gpu_id = "GPU-" + gpu_id
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    ip.profile_read()
    ip.profile_enable(True)
    launches0 = ip.kernel_launches()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(dev_in["H"], dev_in["X0"], O)
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if pg:
        pg.barrier()
    ip.profile_enable(False)
    launches = ip.kernel_launches() - launches0
    phases = ip.profile_read()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, pg, dev)
    status = ip.get_status()

    tokens = w.B * w.T * w.layers
    value = world * tokens / (ms / 1000.0)
    flops = layer_flops(w)
    tflops = world * flops / (ms / 1000.0) / 1e12
    peaks, peak_src = load_peaks()

    # roofline of the dominant kernel (the phase with the largest share of device time)
    timed = {k: v for k, v in phases.items() if v[1] > 0}
    if timed:
        dom = max(timed, key=lambda k: timed[k][0])
        dom_ms, dom_launches = phases[dom]
        roof = {"kernel": dom, **phase_roofline(w, dom, dom_ms, dom_launches, args.steps, peaks),
                "launches": dom_launches, "avg_launch_ms": dom_ms / max(1, dom_launches),
                "peak_note": f"sustained bf16 and copy bandwidth ({peak_src}); burst bf16 {peaks['bf16_tflops']}"}
    else:
        # the fp32 path runs on the CUDA cores and does not time its phases: the
        # whole step against the fp32 FMA rate of the device
        dom = "step"
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        mhz = (clocks or {}).get("sm_max_mhz") or peaks.get("sm_max_mhz", 1965.0)
        fp32_peak = fp32_fma_tflops(sms, mhz)
        ach = flops / (ms / 1000.0) / 1e12
        roof = {"kernel": "whole step (fp32 CUDA-core path)", "bound": "alu", "achieved": ach, "peak": fp32_peak,
                "unit": "TFLOP/s", "frac": ach / fp32_peak, "launches": launches / max(1, args.steps),
                "avg_launch_ms": ms / max(1, launches / max(1, args.steps)),
                "peak_note": f"fp32 FMA rate: {sms} SMs x 128 lanes x 2 flops x {mhz:.0f} MHz"}
    traffic = MEASURED_TRAFFIC.get((w.name, w.C, dom))
    roof["traffic"] = traffic
    roof["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    phase_report = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps,
                        **phase_roofline(w, k, v[0], v[1], args.steps, peaks)}
                    for k, v in phases.items() if v[1] > 0}

    # end to end through the public API: pinned host inputs in, result read back, every step
    e2e = None
    if not args.no_e2e:
        # Inputs start in page-locked host memory and O ends there, every step.  One
        # layer: the library's host-buffer entry point, which pipelines the sequence
        # in pieces so that the copies overlap the compute.  A stack: copy H, X0 in,
        # run the layers, copy the last O out.
        hp = {k: v.pin_memory() for k, v in host.items()}
        o_host = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        if w.layers == 1:
            docs_host = docs.to(torch.int32).contiguous()
            hbuf = torch.empty(ip.forward_host_size(cfg, args.piece_tokens, docs_host.numel()), dtype=torch.uint8,
                               device=dev)

            def e2e_step():
                ip.forward_host(cfg, hp["H"], hp["X0"], *(dev_w[0][k] for k in WEIGHTS), docs_host, O=o_host,
                                piece_tokens=args.piece_tokens, buffer=hbuf)
            api = "ipttt_forward_host (host H, X0, O; pieces copied in and out while others compute)"
        else:
            def e2e_step():
                dev_in["H"].copy_(hp["H"], non_blocking=True)
                dev_in["X0"].copy_(hp["X0"], non_blocking=True)
                step(dev_in["H"], dev_in["X0"], O)
                o_host.copy_(O, non_blocking=True)
            api = "copies in, ipttt_forward per layer, copy out"
        e2e_step()
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(a0.elapsed_time(a1) / args.steps, pg, dev)
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        e2e = {"value": world * tokens / (ems / 1000.0), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": o_host.numel() * o_host.element_size(), "ms_per_step": ems, "api": api}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.state_clip:
        chunks = sample_chunks(w, args.cpu_sample_tokens)
        secs, n = oracle_sample(w, layers[0], chunks)
        cpu = {"value": n / secs, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"first {chunks} chunk(s) ({n} tokens) of row 0, one layer, "
                         f"fp64 numpy oracle, {secs:.1f} s"}

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
               "config": {**config_dict(w, world),
                          **({"clip_on": "accumulated state (ablation)"} if args.state_clip else {})},
               "tflops": tflops, "frac_of_peak": tflops / world / peaks.get("bf16_tflops_sustained", 1.0),
               "flops_per_token": ip.flops_per_token(w.d, w.F),
               # the count for exact arithmetic, where W0 + S_i would be one operand: 8dF + 2d^2
               "tflops_exact_arith_count": tflops * (8 * w.d * w.F + 2 * w.d * w.d) / ip.flops_per_token(w.d, w.F),
               "frac_of_burst_peak": tflops / world / peaks["bf16_tflops"], "peak_source": peak_src,
               "roofline": roof, "phases": phase_report, "clocks": clocks, "e2e": e2e,
               "gpu_launches": launches, "cpu_baseline": cpu, "device_status": status}
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_decode(args, w: synth.Workload):
    """Token-by-token decoding of --decode-batch rows at the workload's d, F and C:
    --steps chunks of C tokens after --warmup chunks, each chunk's commit included.
    The per-token kernels read Wgate, Wup, Wdown0 and every row's bf16 state copy;
    their roofline is HBM bandwidth."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B = args.decode_batch
    wd = w.replace(B=B, T=w.C)
    inp = synth.make_inputs(wd, seed=rank)
    cfg = ip.LayerConfig(B=B, T=1, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip)
    wts = [inp[k].to(dev) for k in WEIGHTS]
    H = inp["H"].to(dev)      # [B, C, d]: one chunk of tokens, reused every chunk
    X0 = inp["X0"].to(dev)
    hs = [H[:, t].contiguous() for t in range(w.C)]
    xs = [X0[:, t].contiguous() for t in range(w.C)]
    o = torch.empty(B, w.d, dtype=torch.bfloat16, device=dev)
    st = ip.DecodeState(cfg, dev)
    stream = torch.cuda.current_stream()

    def chunk():
        for t in range(w.C):
            st.step(hs[t], xs[t], *wts, None, o=o)

    for _ in range(max(1, args.warmup)):
        chunk()
    torch.cuda.synchronize()
    ip.profile_read()
    ip.profile_enable(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        chunk()
    e1.record(stream)
    torch.cuda.synchronize()
    ip.profile_enable(False)
    commit_ms = sum(v[0] for v in ip.profile_read().values()) / args.steps  # the chunk commits (streaming path)
    ms = e0.elapsed_time(e1) / args.steps                                  # per chunk of C tokens
    status = ip.get_status()
    tokens = B * w.C
    per_token_ms = (ms - commit_ms) / w.C
    bytes_per_step = (3 * w.d * w.F + B * w.d * w.F) * 2 + 4 * B * w.d * 2 + 2 * B * w.F * 2
    peaks, peak_src = load_peaks()
    achieved = bytes_per_step / (per_token_ms / 1000.0) / 1e9
    out = {"metric": "In-Place TTT MLP layer decode tokens/s (token-by-token, chunk commits included)",
           "value": tokens / (ms / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"decode_{w.name}", "batch": B, "chunk": w.C, "d_model": w.d, "d_ff": w.F,
                      "step": f"one chunk of {w.C} tokens per row", "l2": "weights and state copies larger than L2"},
           "per_token_ms": per_token_ms, "commit_ms_per_chunk": commit_ms,
           "roofline": {"kernel": "decode per-token kernels", "bound": "hbm", "achieved": achieved,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                        "traffic": None, "bytes_per_token_step": bytes_per_step, "peak_source": peak_src},
           "device_status": status}
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_cp(args, w: synth.Workload):
    """Context parallelism: the workload's sequences split along T over the N
    ranks (strong scaling: the total work is fixed).  A step is every rank's
    ipttt_cp_begin, one NCCL all-gather of the shard aggregates and ipttt_cp_finish;
    with one rank there is no exchange."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    emulated = world == 1 and args.cp_world > 1
    if emulated:
        # one rank's share of an N-rank split, alone on this GPU: its begin and
        # finish on its own shard, the gathered set filled with copies of its own
        # aggregate (the finish reads N aggregates as it would after the exchange;
        # the values are not a forward's, the bytes and launches are)
        if not 0 <= args.cp_rank < args.cp_world:
            raise ValueError("--cp-rank must lie in [0, --cp-world)")
        world, rank = args.cp_world, args.cp_rank
    if w.T % world or (w.T // world) % w.C:
        raise ValueError(f"T={w.T} does not split into {world} shards of whole {w.C}-token chunks")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1 and not emulated:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
        pg = dist
    TL = w.T // world
    inp = synth.make_inputs(w, seed=0)           # the same sequence and weights on every rank
    sl = slice(rank * TL, (rank + 1) * TL)
    H = inp["H"][:, sl].contiguous().to(dev)
    X0 = inp["X0"][:, sl].contiguous().to(dev)
    wts = {k: inp[k].to(dev) for k in WEIGHTS}
    docs = inp["doc_starts"].to(torch.int32).contiguous()
    del inp
    cfg = ip.LayerConfig(B=w.B, T=TL, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip, dtype=w.dtype)
    ws = torch.empty(ip.cp_workspace_size(cfg), dtype=torch.uint8, device=dev)
    agg = torch.empty(w.B, w.d, w.F, dtype=torch.float32, device=dev)
    # one rank: its own aggregate is the whole gathered set
    gathered = torch.empty(world, w.B, w.d, w.F, dtype=torch.float32, device=dev) if world > 1 else agg.view(1, *agg.shape)
    O = torch.empty(w.B, TL, w.d, dtype=cfg.torch_dtype, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ip.cp_begin(cfg, world, rank, H, X0, wts["Wgate"], wts["Wup"], wts["conv_w"], wts["Wtarget"], docs,
                    agg=agg, workspace=ws)
        if pg:
            ip.cp_exchange(agg, out=gathered)
        ip.cp_finish(cfg, world, rank, H, wts["Wdown0"], gathered, ws, docs, O=O)

    if emulated:
        ip.cp_begin(cfg, world, rank, H, X0, wts["Wgate"], wts["Wup"], wts["conv_w"], wts["Wtarget"], docs,
                    agg=agg, workspace=ws)
        gathered.copy_(agg.unsqueeze(0).expand_as(gathered))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ip.get_status() != 0:
        raise RuntimeError("device status set during warm-up")
    gpu_id = str(local)
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_id.startswith("GPU-"):
            gpu_id = "GPU-" + gpu_id
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    ip.profile_read()
    ip.profile_enable(True)
    launches0 = ip.kernel_launches()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if pg:
        pg.barrier()
    ip.profile_enable(False)
    launches = ip.kernel_launches() - launches0
    phases = ip.profile_read()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, pg, dev)
    status = ip.get_status()
    tokens = w.B * (TL if emulated else w.T)
    peaks, peak_src = load_peaks()
    wl = w.replace(T=TL)
    dom = max(phases, key=lambda k: phases[k][0])
    dom_ms, dom_launches = phases[dom]
    roof = {"kernel": dom, **phase_roofline(wl, dom, dom_ms, dom_launches, args.steps, peaks), "traffic": None,
            "launches": dom_launches, "peak_note": f"sustained bf16 and copy bandwidth ({peak_src}); rank {rank}'s phases"}
    phase_report = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
                    for k, v in phases.items()}
    if rank == 0 or emulated:
        cfgd = config_dict(w, world)
        cfgd.update({"workload": f"cp_{w.name}", "parallelism": f"cp{world}", "shard_tokens": TL, "global_batch": w.B,
                     "exchange": "NCCL all-gather of the fp32 shard aggregates" if pg else "none"})
        if emulated:
            cfgd.update({"emulated_rank": rank, "note": "one rank's share alone on one GPU; value = the rank's "
                         "shard tokens / its step time"})
        out = {"metric": METRIC + " (one sequence split over the GPUs)", "value": tokens / (ms / 1000.0),
               "unit": "tokens/s", "n_gpus": 1 if emulated else world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
               "dtype": "bf16", "data": "synthetic", "config": cfgd,
               "tflops": layer_flops(w) / (ms / 1000.0) / 1e12, "roofline": roof, "phases": phase_report,
               "clocks": clocks, "e2e": None, "gpu_launches": launches, "cpu_baseline": None,
               "device_status": status}
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def backward_flops_per_token(d: int, F: int, dtype: str) -> int:
    """Flops of ipttt_backward per token.  fp32 (CUDA cores): the forward products it
    recomputes (gate, up, target, each chunk's V^T Z: 6dF + 2d^2) and the gradient
    products (gW0, gO W0, per chunk P, gV, gZ from the delta, gZ from the state,
    the state's gradient: 14dF; gH and gWgate, gWup: 8dF; gU, gWtarget: 4d^2).
    bf16 (tensor cores): the whole forward (10dF + 2d^2, its apply included; its
    state update's per-chunk P is kept for the gradients) and then gate and up
    pre-activations 4dF, gO W0 2dF, gW0 2dF, the state gradient's deltas 2dF, Z G^T
    2dF, Z P^T 2dF, three gZ terms 6dF, gH 4dF, gWgate and gWup 4dF, gU and
    gWtarget 4d^2: 38dF + 6d^2."""
    if dtype == "bf16":
        return 38 * d * F + 6 * d * d
    return 28 * d * F + 6 * d * d


def run_backward(args, w: synth.Workload):
    """The backward of one layer (ipttt_backward: fp32 gradients of <gO, O> +
    <gS, S_final> with respect to H, X0 and the five weights) on the workload's
    shapes.  bf16 workloads run it on the tensor cores (roofline: the bf16 peak),
    fp32 ones on the CUDA cores (roofline: the fp32 FMA rate)."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    inp = synth.make_inputs(w, seed=rank)
    cfg = ip.LayerConfig(B=w.B, T=w.T, d=w.d, F=w.F, C=w.C, eta=w.eta, clip=w.clip, dtype=w.dtype)
    t = {k: inp[k].to(dev) for k in ("H", "X0") + WEIGHTS}
    docs = inp["doc_starts"]
    g = torch.Generator().manual_seed(11 + rank)
    gO = torch.randn(w.B, w.T, w.d, generator=g).to(cfg.torch_dtype).to(dev)
    gS = torch.randn(w.B, w.d, w.F, generator=g).to(dev)
    del inp
    ws = torch.empty(ip.backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        return ip.backward(cfg, *(t[k] for k in ("H", "X0") + WEIGHTS), docs, gO, gS, workspace=ws)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    if ip.get_status() != 0:
        raise RuntimeError("device status set during warm-up")
    gpu_id = str(local)
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_id.startswith("GPU-"):
            gpu_id = "GPU-" + gpu_id
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    launches0 = ip.kernel_launches()
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    launches = ip.kernel_launches() - launches0
    ms = e0.elapsed_time(e1) / args.steps
    status = ip.get_status()
    tokens = w.B * w.T
    flops = backward_flops_per_token(w.d, w.F, w.dtype) * tokens
    ach = flops / (ms / 1000.0) / 1e12
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    peaks, peak_src = load_peaks()
    if w.dtype == "bf16":
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        roof = {"kernel": "whole backward (tcgen05 GEMMs on bf16 operands, fp32 accumulators)", "bound": "tensor",
                "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                "peak_note": f"sustained bf16 ({peak_src}); burst {peaks['bf16_tflops']}"}
    else:
        peak = fp32_fma_tflops(sms, mhz)
        roof = {"kernel": "whole backward (fp32 CUDA-core GEMMs and elementwise kernels)", "bound": "alu",
                "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                "peak_note": f"fp32 FMA rate: {sms} SMs x 128 lanes x 2 flops x {mhz:.0f} MHz"}
    cfgd = config_dict(w, 1)
    cfgd.update({"workload": f"backward_{w.name}", "gradients": "H, X0, Wgate, Wup, Wdown0, conv_w, Wtarget (fp32)"})
    out = {"metric": "In-Place TTT MLP layer backward tokens/s (fp32 gradients of O and S_final)",
           "value": tokens / (ms / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
           "config": cfgd, "flops_per_token": backward_flops_per_token(w.d, w.F, w.dtype), "roofline": roof,
           "clocks": clocks, "e2e": None, "gpu_launches": launches, "cpu_baseline": None,
           "device_status": status}
    if rank == 0:
        print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--chunk", type=int, default=None, help="override the chunk size C")
    ap.add_argument("--mode", choices=("prefill", "decode", "cp", "backward"), default="prefill",
                    help="decode: token-by-token decoding of --decode-batch rows instead of the prefill step; "
                         "cp: the sequence split along T over the GPUs (context parallelism); "
                         "backward: the layer's gradients (ipttt_backward)")
    ap.add_argument("--decode-batch", type=int, default=8)
    ap.add_argument("--cp-world", type=int, default=1,
                    help="with --mode cp on one GPU: run one rank's share of a split over this many ranks")
    ap.add_argument("--cp-rank", type=int, default=0, help="the rank that --cp-world runs")
    ap.add_argument("--state-clip", action="store_true",
                    help="the ablation that clips the accumulated state instead of each delta (fp32 workloads)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--piece-tokens", type=int, default=0,
                    help="e2e: tokens per pipelined piece of the host-buffer call (0: about T/8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=16384,
                    help="tokens of row 0 the oracle runs for cpu_baseline (whole chunks, about 10 s)")
    ap.add_argument("--ref-sample-tokens", type=int, default=4096,
                    help="tokens of row 0 per step of the reference arm (whole chunks)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    w = synth.WORKLOADS[args.workload]
    if args.chunk:
        w = w.replace(C=args.chunk)
    if args.impl == "reference":
        run_reference(args, w)
    elif args.mode == "decode":
        run_decode(args, w)
    elif args.mode == "cp":
        run_cp(args, w)
    elif args.mode == "backward":
        run_backward(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
