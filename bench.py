#!/usr/bin/env python3
"""Benchmark of the bidirectional SSD mixer on B200.

One step = one ssd_bidir_fwd call over a whole batch of the 130M-shape mixer
workload (batch 32, L 1024, 24 heads x 64, d_state 128, per-head B/C, bf16
I/O): both scans, the D terms and the output write. Inputs are synthetic
(seeded, ssd_inputs) and already resident in HBM when timing starts; they
total ~1 GB per GPU, well above the 126 MB L2, so no flush is needed between
steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--path auto|simt|chunked|fused|segmented|pair|onetile]
                  [--op bidir|bwd|block]

--op bwd times the backward pass (ssd_bidir_bwd) and --op block the mixer
with its conv1d + SiLU, dt and gated-norm steps (ssd_mixer_block_fwd) at the
same workload's sizes; each prints its own metric.

Under torchrun every rank runs the same per-GPU workload (independent
batches: weak scaling, no collective on the data path); rank 0 prints one
JSON line with the whole-job throughput, timed on the device as the max over
ranks. `--impl reference` times the fp64 CPU oracle on the host cores
instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "bidir SSD tokens/s at 130M shape L=1024 (1×B200) + % roofline"
DEFAULT_WORKLOAD = "mixer130m_b32_L1024"
PATH_IDS = {"auto": 0, "simt": 1, "chunked": 2, "fused": 3, "segmented": 4, "pair": 5, "onetile": 7}
# kernels each path launches per ssd_bidir_fwd call (bf16)
LAUNCHES_PER_CALL = {"simt": 1, "chunked": 3, "fused": 1, "segmented": 4, "pair": 1, "onetile": 1}
# sources each path's kernels compile from (a traffic record is valid only
# while their hash is unchanged)
KERNEL_SOURCE = {
    "simt": ("ssd_simt.cu", "ssd_common.cuh"),
    "chunked": ("ssd_tc.cu", "ssd_mask.cuh", "sm100.cuh", "ssd_tmap.h", "ssd_common.cuh"),
    "fused": ("ssd_fused.cu", "ssd_fused_util.cuh", "ssd_mask.cuh", "sm100.cuh", "ssd_tmap.h", "ssd_common.cuh"),
    "segmented": ("ssd_segments.cu", "ssd_fused.cu", "ssd_pair.cu", "ssd_fused_util.cuh", "ssd_mask.cuh", "sm100.cuh",
                  "ssd_tmap.h", "ssd_common.cuh"),
    "pair": ("ssd_pair.cu", "ssd_fused_util.cuh", "ssd_mask.cuh", "sm100.cuh", "ssd_tmap.h", "ssd_common.cuh"),
    "onetile": ("ssd_onetile.cu", "ssd_fused_util.cuh", "ssd_mask.cuh", "sm100.cuh", "ssd_tmap.h", "ssd_common.cuh"),
}
# kernels one call of each path launches (names as in ncu's "Kernel Name")
KERNEL_NAMES = {"simt": ("scan_simt_pair_kernel",), "chunked": ("tc_state_kernel", "tc_pass_kernel", "tc_out_kernel"),
                "fused": ("tc_fused_kernel",), "segmented": ("tc_fused_kernel", "seg_scan_kernel"),
                "pair": ("tc_pair_kernel",), "onetile": ("onetile_kernel",)}
# kernels a call of the path launches on some shapes only (the segmented
# path's last step runs the two-CTA kernel where the segments suit it; the
# fp32 scan runs one kernel per direction beyond one unit per SM)
KERNEL_OPTIONAL = {"segmented": ("tc_pair_kernel",), "simt": ("scan_simt_seq_kernel",)}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch: independent problems, no shared data."""
    return 1000 + rank


def job_time_ms(local_ms: float, world: int, device=None) -> float:
    """Device time of the whole job: the max over ranks (all-reduce MAX of one
    float; the only collective, outside the timed region)."""
    if world <= 1:
        return local_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, job_ms: float) -> float:
    """Whole-job tokens/s: the units all ranks processed over the max-over-ranks time."""
    return tokens_per_rank_step * world * steps / (job_ms / 1e3)


def algorithmic_bytes(w) -> int:
    """Unavoidable HBM bytes of one bidirectional call: x read once, dt/B/C of
    both directions read once, out written once, A and D (fp32)."""
    io = 4 if w.dtype == "f32" else 2
    tok = w.batch * w.seqlen
    elems = tok * w.nheads * w.headdim * 2 + 2 * tok * w.nheads + 4 * tok * w.ngroups * w.dstate
    return io * elems + 4 * 4 * w.nheads


def intra_chunk_flops(w) -> int:
    """Algorithmic tensor work of one bidirectional call: per direction, head
    and chunk of Q tokens, the causal (lower-triangle, Q(Q+1)/2 entries)
    C.B^T over d_state and the masked matrix times X over headdim, 2 flops per
    multiply-add. Counted per head (the decay mask differs per head even where
    B/C are shared)."""
    q = w.chunk
    chunks = w.batch * -(-w.seqlen // q)
    return 2 * w.nheads * chunks * (q * (q + 1) // 2) * 2 * (w.dstate + w.headdim)


def roofline_bound(w, seconds: float, peaks: dict) -> dict:
    """The metric's roofline: the slower of the algorithmic HBM bytes at the
    measured copy bandwidth and the intra-chunk FLOPs at the measured bf16
    tensor throughput; the fraction is that bound's time over the measured one."""
    nbytes, flops = algorithmic_bytes(w), intra_chunk_flops(w)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        achieved = nbytes / seconds / 1e9
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peaks['source']} STREAM-copy HBM GB/s",
                "algorithmic_bytes_per_launch": nbytes, "intra_chunk_flops_per_launch": flops,
                "other_bound_us": round(1e6 * t_tc, 2)}
    achieved = flops / seconds / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4),
            "peak_source": f"{peaks['source']} cuBLAS bf16 TFLOP/s (burst)",
            "algorithmic_bytes_per_launch": nbytes, "intra_chunk_flops_per_launch": flops,
            "other_bound_us": round(1e6 * t_hbm, 2)}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def kernel_source_sha(path: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCE[path]:
        with open(os.path.join(ROOT, "bidirectional_mamba_ssd_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_record(path: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    if it was taken on the current kernel source (else None)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{path}")
    if not e or e.get("source_sha") != kernel_source_sha(path):
        return None
    return e.get("dram_bytes_per_launch")


def record_traffic(csv_path: str, path: str, workload: str, command: str, scale: float = 1.0,
                   note: str = ""):
    """Store dram__bytes_read.sum + dram__bytes_write.sum of one call of the
    path (summed over one launch of each of its kernels), from
    `ncu -i <report> --page raw --csv` output of a capture of whole calls.
    `scale` converts a smaller captured case to the workload (traffic
    proportional to the tiles processed)."""
    import csv
    with open(csv_path, newline="") as f:
        rows = list(csv.reader(f))
    head, units = rows[0], rows[1]
    unit_scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    col = {m: head.index(m) for m in ("Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum")}
    names = KERNEL_NAMES[path]
    optional = KERNEL_OPTIONAL.get(path, ())
    per = {n: [] for n in names + optional}
    for r in rows[2:]:
        for n in names + optional:
            if n + "<" in r[col["Kernel Name"]] or n + "(" in r[col["Kernel Name"]]:
                per[n].append(sum(float(r[col[m]].replace(",", "")) * unit_scale[units[col[m]]]
                                  for m in ("dram__bytes_read.sum", "dram__bytes_write.sum")))
    if any(not per[n] for n in names):
        raise SystemExit(f"not every kernel of {names} is in {csv_path}")
    per = {n: v for n, v in per.items() if v}
    calls = min(len(v) for v in per.values())
    d = {}
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    # every launch captured, over the calls (the kernel launched fewest times
    # is launched once per call; the segmented path launches the fused kernel thrice)
    per_call = sum(sum(v) for v in per.values()) / calls * scale
    e = {"dram_bytes_per_launch": round(per_call), "calls_captured": calls, "kernels": list(per),
         "source_sha": kernel_source_sha(path), "command": command}
    if scale != 1.0:
        e["scaled"] = {"factor": scale, "note": note}
    d[f"{workload}:{path}"] = e
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(d, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(d[f"{workload}:{path}"]))


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during the timed
    region: an in-process NVML thread polling every millisecond between
    __enter__ and __exit__ (read-only queries), else nvidia-smi every 100 ms."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.rows = []          # (sm MHz, max sm MHz, reason names) from NVML
        self.nvml = None
        self.stop = False

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            props = torch.cuda.get_device_properties(self.index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _sample(self):
        nv, h = self.nvml
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        self.rows.append((float(sm), float(self.max_mhz), [n for b, n in self.REASONS.items() if bits & b]))

    def _poll(self):
        while not self.stop:
            try:
                self._sample()
            except Exception:
                break
            time.sleep(0.001)

    def __enter__(self):
        try:
            self.nvml = self._nvml_handle()
            nv, h = self.nvml
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._sample()            # one sample at the start of the region, whatever its length
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop = True
            self.t.join(timeout=5)
            try:
                self._sample()        # and one at its end
            except Exception:
                pass
            return
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = list(self.rows)
        source = "nvml, 1 ms, during the timed region"
        if not rows:
            source = "nvidia-smi, 100 ms"
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for ln in self.lines:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) != 7:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]),
                                 [names[i] for i, v in enumerate(parts[3:]) if v.lower() == "active"]))
                except ValueError:
                    continue
        if not rows:
            return None
        reasons = sorted({n for _, _, r in rows for n in r})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "source": source}


def cpu_baseline(w, budget_s: float = 12.0):
    """The fp64 oracle, as it stands, on the host cores over a bounded sample of
    the workload: whole batch elements (all heads, both directions), several
    per call so every core has a (batch, head) unit, until ~budget_s of work
    or the workload's batch is used up."""
    import math
    import torch
    import oracle
    import ssd_inputs as si
    cores = oracle.threads(0)
    per_call = max(1, min(w.batch, math.ceil(cores / w.nheads)))
    used = min(cores, per_call * w.nheads)
    done, t_used, calls = 0, 0.0, 0
    while t_used < budget_s and done < w.batch:
        k = min(per_call, w.batch - done)
        inp = si.bidir_inputs(k, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, w.dtype,
                              seed=100 + calls, device="cpu")
        arrs = [inp[n].to(torch.float64).numpy() for n in ("x", "dt", "A", "B", "C", "D")]
        t0 = time.perf_counter()
        oracle.bidir(*arrs)
        t_used += time.perf_counter() - t0
        done += k
        calls += 1
    tokens = done * w.seqlen
    return {"value": tokens / t_used, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{done} of {w.batch} batch elements x {w.seqlen} tokens x {w.nheads} heads, "
                      f"both directions, fp64 sequential recurrence, {t_used:.1f} s on {used} threads"}


def run_reference(args, w):
    """Reference arm: the fp64 CPU oracle timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    vals = []
    info = None
    for i in range(args.warmup + args.steps):
        info = cpu_baseline(w, budget_s=4.0)
        if i >= args.warmup:
            vals.append(info["value"])
    v = statistics.median(vals)
    info["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * w.tokens / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, **{k: getattr(w, k) for k in
                       ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "chunk")},
                       "io_dtype": w.dtype},
            "cpu_baseline": info,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_blockstep(args, w, dev):
    """Block diffusion on one GPU through the library's block-diffusion helper
    (bidirectional_mamba_ssd_b200.blockdiff): prefill of the cached forward
    state over the prefix, then per block `steps` denoising steps (each a block
    step on fresh block inputs, reading the cached state) and the commit of the
    block into the state. One bench step = one block: all its denoising steps
    plus the commit, replayed as one CUDA graph (BlockGraph). value = block
    tokens x denoising steps per second."""
    import torch
    import ssd_inputs as si
    from bidirectional_mamba_ssd_b200.blockdiff import BlockDiffusionCache, BlockGraph
    data = si.blockstep_inputs(w.batch, w.seqlen, w.block, w.steps, w.nheads, w.headdim, w.dstate,
                               w.ngroups, w.dtype, seed=0, device=dev)
    cache = BlockDiffusionCache(1, w.batch, w.nheads, w.headdim, w.dstate, device=dev)
    pre = (data["x_pre"][None], data["dt_pre"][None], data["A"][0][None].contiguous(), data["B_pre"][None])
    # prefill timing (outside the graph)
    for _ in range(2):
        cache.prefill(*pre, chunk=w.chunk)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    cache.prefill(*pre, chunk=w.chunk)
    e1.record()
    torch.cuda.synchronize()
    prefill_ms = e0.elapsed_time(e1)
    bg = BlockGraph(cache, w.steps, w.block, w.nheads, w.headdim, w.dstate, w.ngroups)
    bg.A[0].copy_(data["A"])
    bg.D[0].copy_(data["D"])
    for k, st in enumerate(data["steps"]):
        for n in ("x", "dt", "B", "C"):
            getattr(bg, n)[k, 0].copy_(st[n])
    bg.capture()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        bg.replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        t0.record()
        for _ in range(args.steps):
            bg.replay()
        t1.record()
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    tok = w.batch * w.block * w.steps
    io = 2
    step_bytes = (io * (w.batch * w.block * w.nheads * w.headdim * 2 + 2 * w.batch * w.block * w.nheads
                        + 4 * w.batch * w.block * w.ngroups * w.dstate)
                  + 4 * w.batch * w.nheads * w.headdim * w.dstate)
    prefill_bytes = (io * (w.batch * w.seqlen * (w.nheads * w.headdim + w.nheads + w.ngroups * w.dstate))
                     + 4 * w.batch * w.nheads * w.headdim * w.dstate)
    # the commit: the block's x, forward dt and B read, the state read and written
    commit_bytes = (io * w.batch * w.block * (w.nheads * w.headdim + w.nheads + w.ngroups * w.dstate)
                    + 2 * 4 * w.batch * w.nheads * w.headdim * w.dstate)
    block_bytes = w.steps * step_bytes + commit_bytes
    peaks = measured_peaks()
    achieved = block_bytes / (ms / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4),
            "peak_source": f"{peaks['source']} STREAM-copy HBM GB/s",
            "algorithmic_bytes_per_launch": block_bytes,
            "kernel": "blockstep_kernel (the block steps) + tc_fused_kernel (the commit), one CUDA graph; "
                      "bytes of the whole block",
            "traffic": None}
    line = {"metric": "block-diffusion denoising tokens/s (block x steps), cached prefix state",
            "value": round(tok / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "prefix": w.seqlen, "block": w.block,
                       "denoising_steps": w.steps, "nheads": w.nheads, "headdim": w.headdim,
                       "dstate": w.dstate, "ngroups": w.ngroups,
                       "graph": "one CUDA graph per block (blockdiff.BlockGraph: steps + commit)"},
            "roofline": roof,
            "per_denoising_step_us": round(1e3 * ms / (w.steps + 1), 3),
            "algorithmic_bytes_per_denoising_step": step_bytes,
            "prefill": {"ms": round(prefill_ms, 4), "tokens_per_s": round(w.batch * w.seqlen / (prefill_ms / 1e3), 1),
                        "algorithmic_bytes": prefill_bytes,
                        "hbm_frac": round(prefill_bytes / (prefill_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)},
            # one launch per block step (the one-tile kernel for blocks of at most 64
            # tokens, else the fused kernel from 64 (batch, head) units, else 3
            # chunked kernels) and one per commit (fused kernel; 2 chunked kernels
            # under 64 units)
            "gpu_launches": args.steps * ((w.steps if w.block <= 64 or w.batch * w.nheads >= 64 else 3 * w.steps)
                                          + (1 if w.batch * w.nheads >= 64 else 2)),
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def bench_op(args, w, dev, world, rank):
    """The backward pass (--op bwd, one ssd_bidir_bwd call per step) or the
    mixer block (--op block, one ssd_mixer_block_fwd call per step) at a
    workload's sizes, on inputs resident in HBM, CUDA events on the launching
    stream. roofline: algorithmic HBM bytes (inputs read once, outputs written
    once; intermediates and the backward's saved states are not algorithmic)."""
    import torch
    import bidirectional_mamba_ssd_b200 as ssd
    import ssd_inputs as si
    io = 2 if w.dtype == "bf16" else 4
    tok = w.batch * w.seqlen
    HP, GN, H = w.nheads * w.headdim, w.ngroups * w.dstate, w.nheads
    if args.op == "bwd":
        inp = si.workload_inputs(w, seed=rank_seed(rank), device=dev)
        g = torch.Generator(device=dev).manual_seed(rank_seed(rank) + 1)
        dy = torch.randn(inp["x"].shape, generator=g, device=dev).to(inp["x"].dtype)
        names = ("x", "dt", "A", "B", "C", "D")
        ws = ssd.Workspace(dev)

        def step():
            ssd.ssd_bidir_bwd(*(inp[n] for n in names), dy, workspace=ws)
        metric = "bidir SSD backward tokens/s (fp32 gradients of x, dt, A, B, C, D)"
        nbytes = io * tok * (2 * HP + 2 * H + 4 * GN) + 4 * tok * (HP + 2 * H + 4 * GN) + 4 * 8 * H
        kernel, launches = "bwd_scan_kernel", 1
    else:
        bi = si.block_inputs(w, seed=rank_seed(rank), device=dev)
        ws = ssd.Workspace(dev)

        def step():
            ssd.ssd_mixer_block_fwd(bi["xbc"], bi["z"], bi["dt_raw"], bi["conv_w"], bi["conv_b"], bi["dt_bias"],
                                    bi["A"], bi["D"], bi["norm_w"], w.nheads, w.ngroups, w.dstate,
                                    dt_min=1e-3, dt_max=0.1, workspace=ws)
        metric = "bidir Mamba-2 mixer block tokens/s (conv1d + SiLU, dt, mixer, gated RMS norm)"
        nbytes = io * tok * (HP + 2 * GN + HP + 2 * H + HP) + 4 * (2 * (HP + 2 * GN) * (4 + 1) + 6 * H + HP)
        kernel, launches = "conv_silu_kernel + dt_prep_kernel + tc_pair_kernel + gated_rmsnorm_kernel", 4
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise SystemExit("device status after warm-up")
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = job_time_ms(ev0.elapsed_time(ev1), world, dev)
    if rank != 0:
        return
    ms_step = ms / args.steps
    peaks = measured_peaks()
    achieved = nbytes / (ms_step / 1e3) / 1e9
    line = {"metric": metric, "value": round(job_throughput(w.tokens, args.steps, world, ms), 1), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "op": args.op, **{k: getattr(w, k) for k in
                       ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups")},
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "peak_source": f"{peaks['source']} STREAM-copy HBM GB/s",
                         "algorithmic_bytes_per_launch": nbytes, "kernel": kernel, "traffic": None},
            "gpu_launches": launches * args.steps, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--path", default="auto", choices=list(PATH_IDS))
    ap.add_argument("--op", default="bidir", choices=["bidir", "bwd", "block"],
                    help="bidir: the mixer (default, the headline); bwd: its backward pass (ssd_bidir_bwd); "
                         "block: the mixer with conv, dt and gated norm (ssd_mixer_block_fwd)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--record-traffic", metavar="CSV",
                    help="store the dominant kernel's DRAM bytes per launch from an ncu raw CSV "
                         "(with --path and --workload; --capture-command names the capture) and exit")
    ap.add_argument("--capture-command", default="")
    ap.add_argument("--traffic-scale", type=float, default=1.0)
    ap.add_argument("--traffic-note", default="")
    args = ap.parse_args()
    if args.record_traffic:
        if args.path == "auto":
            ap.error("--record-traffic needs an explicit --path")
        record_traffic(args.record_traffic, args.path, args.workload, args.capture_command,
                       args.traffic_scale, args.traffic_note)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    import ssd_inputs as si
    w = si.WORKLOADS[args.workload]
    if args.impl == "reference":
        if args.op != "bidir":
            ap.error("--impl reference times the mixer (--op bidir) only")
        run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    import bidirectional_mamba_ssd_b200 as ssd
    if w.block:
        bench_blockstep(args, w, dev)
        return
    if args.op != "bidir":
        bench_op(args, w, dev, world, rank)
        return
    path = PATH_IDS[args.path]
    if path == 0:
        path = ssd.lib.ssd_select_path(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                                       w.chunk, 1 if w.dtype == "bf16" else 0)
    path_name = {v: k for k, v in PATH_IDS.items()}[path]

    inp = si.workload_inputs(w, seed=rank_seed(rank), device=dev)
    names = ("x", "dt", "A", "B", "C", "D")
    out = torch.empty_like(inp["x"])
    ws = ssd.Workspace(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssd.ssd_bidir_fwd(*(inp[n] for n in names), out=out, chunk=w.chunk, path=path, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc = ws.status()
    if rc != 0:
        raise SystemExit(f"device status {rc} after warm-up")

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    ms = job_time_ms(ev0.elapsed_time(ev1), world, dev)
    if world > 1:
        dist.barrier()
    ms_step = ms / args.steps
    tokens_job = w.tokens * world
    value = job_throughput(w.tokens, args.steps, world, ms)

    # end to end through the public API: pinned host inputs -> device -> mixer -> host output
    e2e = None
    if not args.no_e2e:
        host = {n: inp[n].cpu().pin_memory() for n in names}
        dev_in = {n: torch.empty_like(inp[n]) for n in names}
        host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = host_out.numel() * host_out.element_size()

        def e2e_step():
            for n in names:
                dev_in[n].copy_(host[n], non_blocking=True)
            ssd.ssd_bidir_fwd(*(dev_in[n] for n in names), out=out, chunk=w.chunk, path=path, workspace=ws)
            host_out.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        k = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = job_time_ms(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_throughput(w.tokens, k, world, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks = measured_peaks()
    launches = LAUNCHES_PER_CALL[path_name]
    roof = roofline_bound(w, ms_step / 1e3, peaks)
    roof.update({"traffic": traffic_record(path_name, w.name),
            "kernel": {"simt": "scan_simt_pair_kernel (both scans side by side; scan_simt_seq_kernel beyond one unit per SM)", "chunked": "tc_state/tc_pass/tc_out kernels (whole step)",
                       "fused": "tc_fused_kernel", "pair": "tc_pair_kernel", "onetile": "onetile_kernel",
                       "segmented": "tc_fused_kernel (forward state, reverse state) + seg_scan_kernel + the "
                                    "segments' kernel (tc_pair_kernel, else tc_fused_kernel) (whole step)"}[path_name]})
    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, **{k: getattr(w, k) for k in
                       ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "chunk")},
                       "io_dtype": w.dtype, "state_dtype": "f32", "path": path_name,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (no flush)"},
            "roofline": roof,
            "e2e": e2e,
            "gpu_launches": launches * args.steps,
            "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
