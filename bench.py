"""Benchmark of the Bi-Level Routing Attention forward on B200.

One step = one pass of the whole path (region pooling, routing, token
attention) over one batch of the BiFormer stage-1 workload: B=64, 56x56 map,
C=64, 2 heads of 32, S=7 (49 regions of 8x8 tokens), topk=1, bf16, seeded
synthetic inputs.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--lce] [--qkv]

``--backward`` times bra_attend_backward (dQ, dK, dV for the routing of a
forward pass made beforehand) on the same workload and reports its own line.
On one GPU the default line also carries ``per_workload`` (stages 2 and 3 and
high-res: step and attention times against their rooflines) and ``extras``
(bra_attend_backward on stages 1 and 2 against its minimal bytes, and the
bra_forward_lce step on stage 1 beside bra_forward), all measured in the same
process; ``--per-workload none --extras none`` leaves them out.

``--qkv`` starts every step from the feature map X instead of Q, K, V: the
fused projection (Q, K, V and their region means in one kernel), routing on
those means and attention (bra_forward_qkv), with seeded linear-layer
weights; the roofline then also reports the projection kernel.

N > 1 runs under torch.distributed.run, one process per GPU, each rank an
independent replica on its own batch (the path has no exchange step), and
the value is all ranks' tokens over the slowest rank's device time.

``--impl reference`` times the float64 CPU oracle on bounded samples of the
same workload, one image per host core per step (the comparison arm; rank 0
only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import bra_inputs as bi  # noqa: E402

WORKLOAD = "stage1"
METRIC = "BRA forward tokens/s on 1 B200 (bf16) and % of tensor/HBM roofline"
L2_BYTES = 126 * 2**20
FALLBACK_HBM_GBS = 6650.0
DATASHEET_HBM_GBS = 7700.0  # B200 HGX nominal HBM3e bandwidth, for context beside the measured copy peak

# DRAM bytes per launch of each workload's attention kernel, from one ncu
# capture, keyed by the sha256 of that kernel's code (kernel_file_hash:
# comments do not count); reported as ``traffic`` only while the code is
# unchanged.  With topk = 1 (stage 1) unrouted K and V regions are never read
# and O is still dirty in L2 when the launch ends, so the figure is below the
# algorithmic bytes.
TRAFFIC_RECORDS: dict[str, dict[str, float]] = {
    # ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch on the full workload
    # (profiles/launches_stage1.md gives the capture command; --workload selects the stage)
    # bra_attend_stack_kernel<4, 1, 0, 0>, stage 1: read 68.26 MB + write 3.34 MB
    "attend_stack.cu": {"de444a53e078031d53e8d08845fa6b9cf4276aaf282a799c863f3bf5acbb37f5": 71.606016e6},
    # bra_attend_warp_kernel<64, 16>, stage 2: read 38.77 MB + write 0.03 MB
    "attend_warp.cu": {"b2601a5bd2bf81174f856102fd86a2efe94baf181481b9015a3669adbf06094b": 38.79296e6},
    # bra_attend_flash_kernel, highres: read 12.64 MB + write 0 MB
    "attend_flash.cu": {"206f6bd5db0df890ea2cd549cf0ed1e6254d335d3084a26e7703259dc62f3106": 12.644352e6},
    # bra_attend_slice_kernel, stage 3: read 20.95 MB + write 0 MB
    "attend_slice.cu": {"03b48fd85e880febd1d5102e078efbdc822eccc63f892d74e0cd1b6921983611": 20.951552e6},
}

# The file holding each workload's attention kernel (the kernel bra_attend
# chooses for that shape).
KERNEL_FILE = {"stage1": "attend_stack.cu", "stage2": "attend_warp.cu", "stage3": "attend_slice.cu",
               "highres": "attend_flash.cu", "detection": "attend_stack.cu", "tiny": "attend_simt.cu"}


# DRAM bytes per launch of the fused projection kernel on the stage-1 workload
# (same rule as above, keyed by kernel_sources_hash("qkv")).  Most of the
# 77 MB of Q, K, V it writes is still dirty in L2 when the launch ends, so the
# figure is below the algorithmic bytes.
QKV_TRAFFIC_RECORDS: dict[str, float] = {
    # ncu capture of bra_qkv_kernel<1> (8 warps, next MMA under the region sums):
    # dram read 25.77 MB + write 19.11 MB
    "672037142a2a077ac0946e1a1c68e35e52673d0180e9b89cde6dbaf09cdc2a17": 44.871424e6,
}


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=WORKLOAD, choices=list(bi.WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=20)
    p.add_argument("--lce", action="store_true",
                   help="add the local context enhancement (seeded 5x5 depthwise weights) to every step: "
                        "bra_forward_lce, the term in the attention kernel's epilogue where it covers the shape")
    p.add_argument("--qkv", action="store_true",
                   help="start every step from the feature map: fused Q/K/V projection + routing + attention")
    p.add_argument("--backward", action="store_true",
                   help="time the attention gradients (bra_attend_backward) instead of the forward")
    p.add_argument("--per-workload", default="stage2,stage3,highres",
                   help="other workloads timed in the same run (comma list; 'none': none)")
    p.add_argument("--extras", default="backward,lce",
                   help="entry points around the path timed in the same one-GPU run, reported under "
                        "'extras' (comma list of backward, lce; 'none': none)")
    return p.parse_args(argv)


def workload_config(shape: bi.BraShape, name: str) -> dict:
    return {"workload": f"{name}: B{shape.B} {shape.H}x{shape.W} C{shape.C} heads{shape.heads} "
                        f"d{shape.d} S{shape.S} topk{shape.topk} {shape.dtype}",
            "B": shape.B, "H": shape.H, "W": shape.W, "C": shape.C, "heads": shape.heads,
            "S": shape.S, "topk": shape.topk, "tokens_per_step": shape.tokens}


def byte_counts(shape: bi.BraShape) -> dict:
    es = 2 if shape.dtype == "bf16" else 4
    m = shape.tokens * shape.C * es
    idx = shape.B * shape.heads * shape.R * shape.topk * 4
    means = shape.B * shape.heads * shape.R * shape.d * 4
    return {
        "map": m,
        "idx": idx,
        # minimal bytes of the whole path: Q, K, V read once, O and I^r written once
        "path_min": 4 * m + idx,
        # attention kernel: Q, K, V read, O written, I^r read
        "attend": 4 * m + idx,
        # pooling kernel: Q, K read, means written
        "pool": 2 * m + 2 * means,
        # fused projection: X and the layer read, Q, K, V and the means written
        "qkv": 4 * m + 2 * means + 3 * shape.C * shape.C * es + 3 * shape.C * 4,
        # attention gradients: Q, K, V, dO and I^r read, dQ, dK, dV written in fp32
        "backward": 4 * m + idx + 3 * shape.tokens * shape.C * 4,
        # the path from X: X read, O and I^r written
        "path_min_qkv": 2 * m + idx,
    }


def attention_flops(shape: bi.BraShape) -> float:
    # QK^T and PV: 2 matmuls x (tokens x topk*n keys x C) multiply-adds x 2 flop
    return 4.0 * shape.tokens * shape.topk * shape.n * shape.C


def measured_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C/C++ source without comments or blank lines: edits to comments do not
    change the code the counters were taken on."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_file_hash(name: str) -> str:
    """sha256 of the code (comments stripped) of one kernel file and the shared
    device headers and TMA host code it builds on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dynamic_sparse_attention_bra_b200", "csrc")
    for f in [name, "common.cuh", "kernels.h", "tc_ptx.cuh", "tma_host.cu", "tma_host.h"]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()


def recorded_traffic(workload: str) -> float | None:
    """ncu DRAM bytes per launch of the workload's attention kernel, if the
    kernel's code is the one they were taken on."""
    name = KERNEL_FILE.get(workload)
    return TRAFFIC_RECORDS.get(name, {}).get(kernel_file_hash(name)) if name else None


def kernel_sources_hash(prefix: str = "attend") -> str:
    """sha256 of the code (comments stripped) of the kernel named by
    ``prefix``: its own files, the TMA host code and the shared device headers."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dynamic_sparse_attention_bra_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith((prefix, "tma_host")) or name in ("common.cuh", "kernels.h", "tc_ptx.cuh"):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int):
        self.samples: list[int] = []
        self.reasons = 0
        self.max_mhz = None
        self.matched_by = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h, self.matched_by = self._handle(pynvml, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report what we could not sample
            self._nvml = None

    @staticmethod
    def _handle(nv, device_index: int):
        """NVML handle of the CUDA device ``device_index``.  NVML numbers the
        GPUs of the machine and ignores CUDA_VISIBLE_DEVICES, so the device is
        found by its UUID (else its PCI bus id), not by its CUDA index."""
        import torch
        props = torch.cuda.get_device_properties(device_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID(f"GPU-{uuid}"), "uuid"
            except Exception:
                pass
        bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        return nv.nvmlDeviceGetHandleByPciBusId(bus), "pci_bus_id"

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                return
            time.sleep(0.0002)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def report(self) -> dict:
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                "nvml_device_matched_by": self.matched_by}


def host_cores() -> int:
    """Cores this process may run on (the affinity mask, not the machine)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# State of one oracle worker process (filled by _oracle_worker_init).
_WORKER: dict = {}


def _oracle_worker_init(shape: bi.BraShape, seed: int, from_feature_map: bool, lce: bool) -> None:
    import oracle
    _WORKER["oracle"] = oracle
    _WORKER["shape"] = shape
    _WORKER["inp"] = bi.make_inputs(shape, seed)
    _WORKER["proj"] = bi.make_projection_inputs(shape, seed) if from_feature_map else None
    if lce:
        rng = np.random.default_rng(seed + 77)
        _WORKER["lce"] = (rng.standard_normal((shape.C, 5, 5)) / 5.0, rng.standard_normal(shape.C))
    else:
        _WORKER["lce"] = None


def _oracle_image(i: int) -> int:
    """The unmodified oracle's forward on image i of the batch (one thread);
    returns the tokens processed."""
    oracle, shape, inp, proj, lce = (_WORKER[k] for k in ("oracle", "shape", "inp", "proj", "lce"))
    b = i % shape.B
    sl = slice(b, b + 1)
    if proj is not None:
        q, k, v = oracle.qkv_projection(proj.x_f64[sl], proj.w_f64, proj.b_f64)
    else:
        q, k, v = inp.q_f64[sl], inp.k_f64[sl], inp.v_f64[sl]
    o, _ = oracle.bra_forward(q, k, v, shape.heads, shape.S, shape.topk)
    if lce is not None:
        o = o + oracle.local_context(v, lce[0], lce[1])
    return shape.H * shape.W


class OraclePool:
    """``cores`` worker processes (spawned, so safe after CUDA is initialised),
    each holding the seeded workload, running the oracle one image per task."""

    def __init__(self, shape: bi.BraShape, seed: int, cores: int, from_feature_map: bool = False,
                 lce: bool = False):
        import multiprocessing as mp
        self.cores = cores
        self.pool = mp.get_context("spawn").Pool(cores, initializer=_oracle_worker_init,
                                                 initargs=(shape, seed, from_feature_map, lce))
        self.pool.map(_oracle_image, range(cores))  # inputs built, oracle loaded in every worker

    def run(self, first_image: int, images: int) -> int:
        return sum(self.pool.map(_oracle_image, range(first_image, first_image + images), chunksize=1))

    def close(self):
        self.pool.close()
        self.pool.join()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def cpu_oracle_throughput(shape: bi.BraShape, seed: int, budget_s: float = 10.0,
                          batches_per_call: int | None = None, from_feature_map: bool = False,
                          all_cores: bool = True) -> dict:
    """The float64 oracle on bounded samples of the workload: one thread, and
    (``all_cores``) one worker process per host core, each running the
    unmodified oracle on its own images."""
    import oracle
    inp = bi.make_inputs(shape, seed)
    proj = bi.make_projection_inputs(shape, seed) if from_feature_map else None
    bpc = batches_per_call or shape.B
    tokens = 0
    t0 = time.perf_counter()
    calls = 0
    while True:
        b0 = (calls * bpc) % shape.B
        sl = slice(b0, b0 + bpc)
        if proj is not None:
            q, k, v = oracle.qkv_projection(proj.x_f64[sl], proj.w_f64, proj.b_f64)
        else:
            q, k, v = inp.q_f64[sl], inp.k_f64[sl], inp.v_f64[sl]
        oracle.bra_forward(q, k, v, shape.heads, shape.S, shape.topk)
        tokens += bpc * shape.H * shape.W
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    one = {"value": tokens / el, "unit": "tokens/s", "cores": 1, "host_cores": host_cores(), "kind": "oracle",
           "sample": f"{calls} oracle calls of {bpc} of {shape.B} images ({tokens} tokens) "
                     f"in {el:.1f} s, float64, one thread"}
    cores = host_cores()
    if not all_cores or cores <= 1:
        return one
    with OraclePool(shape, seed, cores, from_feature_map) as pool:
        done = 0
        t0 = time.perf_counter()
        while True:
            done += pool.run(done // (shape.H * shape.W), cores)
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
    images = done // (shape.H * shape.W)
    return {"value": done / el, "unit": "tokens/s", "cores": cores, "host_cores": cores, "kind": "oracle",
            "sample": f"{images} images of the {shape.B}-image batch ({done} tokens) in {el:.1f} s, float64, "
                      f"one image per task on {cores} worker processes",
            "single_thread": one}


def max_over_ranks(values, world: int, device="cpu") -> list[float]:
    """Element-wise maximum of ``values`` over all ranks (every rank gets it):
    a multi-GPU time is the slowest rank's.  One process: ``values`` itself."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """All ranks' tokens of one step over the (slowest rank's) step time."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


def rank_seed(seed: int, rank: int) -> int:
    """Each replica draws its own batch."""
    return seed + 1000 * rank


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args):
    """The comparison arm: the float64 oracle, unmodified, on the host's cores.
    Each step runs one image per core (a bounded sample of the batch), every
    worker process running the oracle on its own image."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    shape, seed = bi.WORKLOADS[args.workload]
    cores = host_cores()
    with OraclePool(shape, seed, cores, from_feature_map=args.qkv, lce=args.lce) as pool:
        for i in range(args.warmup):
            pool.run(i * cores, cores)
        tokens = 0
        t0 = time.perf_counter()
        for i in range(args.steps):
            tokens += pool.run((args.warmup + i) * cores, cores)
        el = time.perf_counter() - t0
    value = tokens / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(shape, args.workload), "sample_images_per_step": cores,
                   "local_context": bool(args.lce), "from_feature_map": bool(args.qkv)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "host_cores": cores, "kind": "oracle",
                         "sample": f"{cores} of {shape.B} images per step, one per worker process, "
                                   f"float64 oracle"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def measured_peak_tflops() -> float | None:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return None


def roofline_time_s(shape: bi.BraShape, hbm_gbs: float, tflops: float | None) -> tuple[float, str]:
    """The attention kernel's roofline time: the larger of its minimal bytes
    over the HBM peak and its FLOPs over the bf16 tensor peak."""
    t_hbm = byte_counts(shape)["attend"] / (hbm_gbs * 1e9)
    t_tc = attention_flops(shape) / (tflops * 1e12) if tflops else 0.0
    return (t_tc, "tensor") if t_tc > t_hbm else (t_hbm, "hbm")


def time_workload(name: str, steps: int, warmup: int, dev, stream) -> dict:
    """Step time (bra_forward back to back) and the attention kernel's own
    launch time (events around each bra_attend) on another workload, with
    rotating input sets larger than L2, in the same process as the headline."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape, seed = bi.WORKLOADS[name]
    inp = bi.make_inputs(shape, seed)
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    cnt = byte_counts(shape)
    set_bytes = 4 * cnt["map"] + cnt["idx"]
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes))
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    base = [torch.from_numpy(a).view(tdt) if shape.dtype == "bf16" else torch.from_numpy(a)
            for a in (inp.q_store, inp.k_store, inp.v_store)]
    sets = []
    for _ in range(nsets):
        q, k, v = (t.to(dev) for t in base)
        sets.append(dict(q=q, k=k, v=v, o=torch.empty_like(q),
                         idx=torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device=dev),
                         ws=torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device=dev)))
    sp = stream.cuda_stream
    with torch.cuda.stream(stream):
        for i in range(warmup):
            b = sets[i % nsets]
            bra.bra_forward(s, b["q"], b["k"], b["v"], b["o"], b["idx"], b["ws"], sp)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with ClockSampler(dev.index) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(steps):
                b = sets[i % nsets]
                bra.bra_forward(s, b["q"], b["k"], b["v"], b["o"], b["idx"], b["ws"], sp)
            end.record(stream)
            for i in range(steps):
                b = sets[i % nsets]
                bra.bra_route(s, b["q"], b["k"], b["idx"], b["ws"], sp)
                ev[i][0].record(stream)
                bra.bra_attend(s, b["q"], b["k"], b["v"], b["idx"], b["o"], b["ws"], sp)
                ev[i][1].record(stream)
            a0.record(stream)
            for i in range(steps):
                b = sets[i % nsets]
                bra.bra_attend(s, b["q"], b["k"], b["v"], b["idx"], b["o"], b["ws"], sp)
            a1.record(stream)
        torch.cuda.synchronize(dev)
    for b in sets:
        st = bra.bra_device_status(s, b["ws"], sp)
        if st != bra.BRA_OK:
            raise RuntimeError(f"{name}: device status after timing: {bra.bra_status_string(st)}")
    step_ms = start.elapsed_time(end) / steps
    attend_iso_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    attend_ms = a0.elapsed_time(a1) / steps
    peak, peak_kind = measured_peaks()
    t_roof, bound = roofline_time_s(shape, peak, measured_peak_tflops())
    del sets
    torch.cuda.empty_cache()
    return {
        "workload": workload_config(shape, name)["workload"], "tokens_per_step": shape.tokens,
        "step_ms": step_ms, "tokens_per_s": shape.tokens / (step_ms * 1e-3),
        "attend": {"launch_ms": attend_ms, "bound": bound, "roofline_us": t_roof * 1e6,
                   "frac": t_roof / (attend_ms * 1e-3),
                   "launch_ms_isolated": attend_iso_ms, "frac_isolated": t_roof / (attend_iso_ms * 1e-3),
                   "achieved_gbs": cnt["attend"] / (attend_ms * 1e-3) / 1e9,
                   "achieved_tflops": attention_flops(shape) / (attend_ms * 1e-3) / 1e12,
                   "algorithmic_bytes": cnt["attend"], "flops": attention_flops(shape),
                   "peak_kind": peak_kind, "kernel_file": KERNEL_FILE.get(name),
                   "traffic": recorded_traffic(name)},
        "path_frac": cnt["path_min"] / (peak * 1e9) / (step_ms * 1e-3),
        "steps": steps, "l2": f"rotating {nsets} input sets ({nsets * set_bytes / 2**20:.0f} MiB)",
        "clocks": clocks.report(),
    }


def time_backward(name: str, steps: int, warmup: int, dev, stream) -> dict:
    """bra_attend_backward back to back on one workload (a single set of inputs
    and gradients already spans more than L2 on the stage workloads): its time
    per call against the minimal bytes (Q, K, V, dO and I^r read once, dQ, dK,
    dV written once in fp32)."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape, seed = bi.WORKLOADS[name]
    inp = bi.make_inputs(shape, seed)
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    q, k, v = ((torch.from_numpy(a).view(tdt) if shape.dtype == "bf16" else torch.from_numpy(a)).to(dev)
               for a in (inp.q_store, inp.k_store, inp.v_store))
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device=dev)
    idx = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    g = torch.Generator().manual_seed(seed + 100)
    go = torch.randn(q.shape, generator=g).to(tdt).to(dev)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3))
    sp = stream.cuda_stream
    with torch.cuda.stream(stream):
        bra.bra_forward(s, q, k, v, o, idx, ws, sp)
        for _ in range(warmup):
            bra.bra_attend_backward(s, q, k, v, idx, go, dq, dk, dv, ws, sp)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(steps):
                bra.bra_attend_backward(s, q, k, v, idx, go, dq, dk, dv, ws, sp)
            end.record(stream)
        torch.cuda.synchronize(dev)
    st = bra.bra_device_status(s, ws, sp)
    if st != bra.BRA_OK:
        raise RuntimeError(f"backward {name}: device status after timing: {bra.bra_status_string(st)}")
    ms = start.elapsed_time(end) / steps
    cnt = byte_counts(shape)
    min_bytes = cnt["backward"]
    peak, peak_kind = measured_peaks()
    del q, k, v, o, go, dq, dk, dv
    torch.cuda.empty_cache()
    return {"workload": workload_config(shape, name)["workload"], "entry": "bra_attend_backward",
            "kernel": os.environ.get("BRA_BACKWARD_KERNEL") or "auto (tensor cores where covered)",
            "ms_per_call": ms, "tokens_per_s": shape.tokens / (ms * 1e-3), "bound": "hbm",
            "min_bytes": min_bytes, "achieved_gbs": min_bytes / (ms * 1e-3) / 1e9,
            "frac": min_bytes / (ms * 1e-3) / 1e9 / peak, "peak_kind": peak_kind,
            "timing": "one call = clear dK, dV + the kernel; calls back to back", "steps": steps,
            "clocks": clocks.report()}


def time_forward_lce(name: str, steps: int, warmup: int, dev, stream) -> dict:
    """bra_forward_lce (routing, attention and the local context term) back to
    back on rotating input sets larger than L2, against bra_forward on the same
    sets in the same run."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra
    shape, seed = bi.WORKLOADS[name]
    inp = bi.make_inputs(shape, seed)
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    cnt = byte_counts(shape)
    set_bytes = 4 * cnt["map"] + cnt["idx"]
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes))
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    base = [torch.from_numpy(a).view(tdt) if shape.dtype == "bf16" else torch.from_numpy(a)
            for a in (inp.q_store, inp.k_store, inp.v_store)]
    sets = []
    for _ in range(nsets):
        q, k, v = (t.to(dev) for t in base)
        sets.append(dict(q=q, k=k, v=v, o=torch.empty_like(q),
                         idx=torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device=dev),
                         ws=torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device=dev)))
    g = torch.Generator().manual_seed(seed + 77)
    lce_w = (torch.randn(shape.C * 25, generator=g) / 5.0).to(dev)
    lce_b = torch.randn(shape.C, generator=g).to(dev)
    sp = stream.cuda_stream

    def run(i, with_lce):
        b = sets[i % nsets]
        if with_lce:
            bra.bra_forward_lce(s, b["q"], b["k"], b["v"], lce_w, lce_b, b["o"], b["idx"], b["ws"], sp)
        else:
            bra.bra_forward(s, b["q"], b["k"], b["v"], b["o"], b["idx"], b["ws"], sp)

    with torch.cuda.stream(stream):
        for i in range(warmup):
            run(i, True)
            run(i, False)
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with ClockSampler(dev.index) as clocks:
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for i in range(steps):
                run(i, True)
            ev[1].record(stream)
            for i in range(steps):
                run(i, False)
            ev[2].record(stream)
        torch.cuda.synchronize(dev)
    for b in sets:
        st = bra.bra_device_status(s, b["ws"], sp)
        if st != bra.BRA_OK:
            raise RuntimeError(f"forward_lce {name}: device status after timing: {bra.bra_status_string(st)}")
    lce_ms, plain_ms = ev[0].elapsed_time(ev[1]) / steps, ev[1].elapsed_time(ev[2]) / steps
    del sets
    torch.cuda.empty_cache()
    return {"workload": workload_config(shape, name)["workload"], "entry": "bra_forward_lce",
            "step_ms": lce_ms, "tokens_per_s": shape.tokens / (lce_ms * 1e-3),
            "bra_forward_step_ms": plain_ms, "added_ms": lce_ms - plain_ms, "steps": steps,
            "l2": f"rotating {nsets} input sets ({nsets * set_bytes / 2**20:.0f} MiB)", "clocks": clocks.report()}


def run_ours(args):
    import torch
    import dynamic_sparse_attention_bra_b200 as bra

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    shape, seed = bi.WORKLOADS[args.workload]
    inp = bi.make_inputs(shape, rank_seed(seed, rank))
    es = 2 if shape.dtype == "bf16" else 4
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32

    def host(x):
        t = torch.from_numpy(x)
        return t.view(torch.bfloat16) if shape.dtype == "bf16" else t

    host_qkv = [host(a).pin_memory() for a in (inp.q_store, inp.k_store, inp.v_store)]
    cnt = byte_counts(shape)
    set_bytes = (5 if args.qkv else 4) * cnt["map"] + cnt["idx"]
    proj = host_x = w_qkv = b_qkv = None
    if args.qkv:
        proj = bi.make_projection_inputs(shape, rank_seed(seed, rank))
        host_x = host(proj.x_store).pin_memory()
        w_qkv = host(proj.w_store).to(dev)
        b_qkv = torch.from_numpy(proj.b_store).to(dev)
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes))
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    sets = []
    for _ in range(nsets):
        q, k, v = (h.to(dev) for h in host_qkv)
        sets.append(dict(
            q=q, k=k, v=v, o=torch.empty_like(q),
            idx=torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device=dev),
            ws=torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device=dev)))
        if args.qkv:
            sets[-1]["x"] = host_x.to(dev)
            sets[-1]["qr"] = torch.empty((shape.B, shape.heads, shape.R, shape.d), device=dev)
            sets[-1]["kr"] = torch.empty_like(sets[-1]["qr"])
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream

    # local context enhancement parameters (seeded, as a layer's weights would be)
    lce_w = lce_b = None
    if args.lce:
        g = torch.Generator().manual_seed(seed + 77)
        lce_w = (torch.randn(shape.C * 25, generator=g) / 5.0).to(dev)
        lce_b = torch.randn(shape.C, generator=g).to(dev)

    def forward(b):
        if args.qkv:
            bra.bra_forward_qkv(s, b["x"], w_qkv, b_qkv, b["q"], b["k"], b["v"], b["o"], b["idx"], b["ws"], sp)
            if args.lce:
                bra.bra_lce(s, b["v"], lce_w, lce_b, b["o"], sp)
        elif args.lce:
            # the local context term in the attention kernel's epilogue where it covers the shape
            bra.bra_forward_lce(s, b["q"], b["k"], b["v"], lce_w, lce_b, b["o"], b["idx"], b["ws"], sp)
        else:
            bra.bra_forward(s, b["q"], b["k"], b["v"], b["o"], b["idx"], b["ws"], sp)

    def step(i):
        forward(sets[i % nsets])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)

    # Timed region: K steps of the public forward call back to back (pooling,
    # routing and attention per step, chained by programmatic dependent
    # launch), events only at its two ends.  A second pass over the same K
    # steps brackets each attention launch with events on the same stream
    # (``launch_ms_isolated``: each launch alone, its set-up and pipeline fill
    # exposed; an event between two launches ends their overlap, so this pass
    # is not the step time), then times K attention launches back to back
    # (``launch_ms``: the kernel's average launch period, as in a stream of
    # attention calls).
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    ev_qkv = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] if args.qkv else []
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(args.steps):
                step(i)
            end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                b = sets[i % nsets]
                if args.qkv:
                    ev_qkv[i][0].record(stream)
                    bra.bra_qkv_project(s, b["x"], w_qkv, b_qkv, b["q"], b["k"], b["v"], b["qr"], b["kr"],
                                        b["ws"], sp)
                    ev_qkv[i][1].record(stream)
                bra.bra_route(s, b["q"], b["k"], b["idx"], b["ws"], sp)
                ev[i][0].record(stream)
                bra.bra_attend(s, b["q"], b["k"], b["v"], b["idx"], b["o"], b["ws"], sp)
                ev[i][1].record(stream)
            # the attention kernel alone, K launches back to back on the routes of
            # the pass above: its average launch period
            a0.record(stream)
            for i in range(args.steps):
                b = sets[i % nsets]
                bra.bra_attend(s, b["q"], b["k"], b["v"], b["idx"], b["o"], b["ws"], sp)
            a1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    attend_iso_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    attend_ms = a0.elapsed_time(a1) / args.steps
    qkv_ms = sum(a.elapsed_time(b) for a, b in ev_qkv) / args.steps if args.qkv else 0.0
    for b in sets:
        st = bra.bra_device_status(s, b["ws"], sp)
        if st != bra.BRA_OK:
            raise RuntimeError(f"device status after timing: {bra.bra_status_string(st)}")

    # End to end through the public API with host buffers: pinned Q, K, V in,
    # O and I^r out, every step, copies inside the timed region.
    o_host = torch.empty(host_qkv[0].shape, dtype=tdt).pin_memory()
    idx_host = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32).pin_memory()
    b0 = sets[0]
    h2d = (1 if args.qkv else 3) * cnt["map"]
    d2h = cnt["map"] + cnt["idx"]

    def e2e_step():
        with torch.cuda.stream(stream):
            if args.qkv:
                b0["x"].copy_(host_x, non_blocking=True)
            else:
                for dst, src in zip((b0["q"], b0["k"], b0["v"]), host_qkv):
                    dst.copy_(src, non_blocking=True)
            forward(b0)
            o_host.copy_(b0["o"], non_blocking=True)
            idx_host.copy_(b0["idx"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps

    total_ms, attend_ms, attend_iso_ms, e2e_ms, qkv_ms = max_over_ranks(
        [total_ms, attend_ms, attend_iso_ms, e2e_ms, qkv_ms], world, dev)

    # The other workloads' attention and step times, on one GPU (same process).
    per_workload = {}
    if world == 1 and not args.qkv and not args.lce:
        for name in [w for w in args.per_workload.split(",") if w in bi.WORKLOADS and w != args.workload]:
            per_workload[name] = time_workload(name, args.steps, max(args.warmup, 3), dev, stream)
    # Entry points around the path (one GPU): the gradients and the local context term.
    extras = {}
    if world == 1 and not args.qkv and not args.lce:
        wanted = [e for e in args.extras.split(",") if e]
        if "backward" in wanted:
            for name in ("stage1", "stage2"):
                extras[f"backward_{name}"] = time_backward(name, min(args.steps, 100), max(args.warmup, 3), dev,
                                                           stream)
        if "lce" in wanted:
            extras["forward_lce_stage1"] = time_forward_lce("stage1", min(args.steps, 200), max(args.warmup, 3),
                                                            dev, stream)
    ms_per_step = total_ms / args.steps
    tokens = shape.tokens * world
    value = whole_job_tokens_per_s(shape.tokens, world, ms_per_step)

    if rank == 0:
        peak, peak_kind = measured_peaks()
        achieved = cnt["attend"] / (attend_ms * 1e-3) / 1e9
        path_key = "path_min_qkv" if args.qkv else "path_min"
        traffic = recorded_traffic(args.workload)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": shape.dtype, "data": "synthetic",
            "config": {**workload_config(shape, args.workload), "parallelism": f"replicas{world}",
                       "local_context": bool(args.lce), "from_feature_map": bool(args.qkv),
                       "l2": f"rotating {nsets} input sets ({nsets * set_bytes / 2**20:.0f} MiB) > 126 MiB L2"},
            "roofline": {
                "kernel": "bra_attend", "bound": "hbm", "achieved": achieved, "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                "algorithmic_bytes": cnt["attend"], "launch_ms": attend_ms,
                "launch_timing": "CUDA events around K attention launches back to back (average period)",
                "launch_ms_isolated": attend_iso_ms,
                "frac_isolated": cnt["attend"] / (attend_iso_ms * 1e-3) / 1e9 / peak,
                "datasheet_peak": DATASHEET_HBM_GBS, "frac_of_datasheet": achieved / DATASHEET_HBM_GBS,
            },
            "path_roofline": {
                "min_bytes": cnt[path_key], "flops": attention_flops(shape),
                "time_us": ms_per_step * 1e3,
                "frac": cnt[path_key] / peak / 1e9 / (ms_per_step * 1e-3),
            },
            "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": (4 if args.lce and args.qkv else 3) * args.steps,
            "clocks": clocks.report(),
        }
        if per_workload:
            line["per_workload"] = per_workload
        if extras:
            line["extras"] = extras
        if args.qkv:
            qkv_gbs = cnt["qkv"] / (qkv_ms * 1e-3) / 1e9
            line["qkv_roofline"] = {
                "kernel": "bra_qkv_project", "bound": "hbm", "achieved": qkv_gbs, "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": qkv_gbs / peak,
                "traffic": QKV_TRAFFIC_RECORDS.get(kernel_sources_hash("qkv")),
                "algorithmic_bytes": cnt["qkv"], "launch_ms": qkv_ms,
            }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_oracle_throughput(shape, seed, from_feature_map=args.qkv)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def run_backward(args):
    """bra_attend_backward on one GPU: dQ, dK, dV (fp32) for a fixed routing."""
    import torch
    import dynamic_sparse_attention_bra_b200 as bra

    world, rank, local = dist_env()
    if world > 1:
        raise SystemExit("--backward runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    shape, seed = bi.WORKLOADS[args.workload]
    inp = bi.make_inputs(shape, seed)
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32

    def dev_map(x):
        t = torch.from_numpy(x)
        return (t.view(torch.bfloat16) if shape.dtype == "bf16" else t).to(dev)

    q, k, v = (dev_map(a) for a in (inp.q_store, inp.k_store, inp.v_store))
    s = bra.shape_for(shape.B, shape.H, shape.W, shape.C, shape.heads, shape.S, shape.topk, shape.dtype)
    ws = torch.zeros(bra.bra_workspace_bytes(s), dtype=torch.uint8, device=dev)
    idx = torch.empty((shape.B, shape.heads, shape.R, shape.topk), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    stream = torch.cuda.Stream(device=dev)
    sp = stream.cuda_stream
    g = torch.Generator().manual_seed(seed + 100)
    go = torch.randn(q.shape, generator=g).to(tdt).to(dev)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3))
    with torch.cuda.stream(stream):
        bra.bra_forward(s, q, k, v, o, idx, ws, sp)  # the routing the gradients are taken for

    def step():
        bra.bra_attend_backward(s, q, k, v, idx, go, dq, dk, dv, ws, sp)

    # Inputs and gradients (Q, K, V, dO read; dQ, dK, dV cleared and written in fp32)
    # span more than the 126 MB L2 on the stage workloads.
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                step()
            end.record(stream)
        torch.cuda.synchronize(dev)
    st = bra.bra_device_status(s, ws, sp)
    if st != bra.BRA_OK:
        raise RuntimeError(f"device status after timing: {bra.bra_status_string(st)}")
    ms = start.elapsed_time(end) / args.steps
    cnt = byte_counts(shape)
    es = 2 if shape.dtype == "bf16" else 4
    # minimal bytes: Q, K, V, dO and I^r read once, dQ, dK, dV written once in fp32
    min_bytes = cnt["backward"]
    peak, peak_kind = measured_peaks()
    achieved = min_bytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "BRA attention backward tokens/s on 1 B200", "value": shape.tokens / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": shape.dtype,
        "data": "synthetic",
        "config": {**workload_config(shape, args.workload), "gradients": "fp32", "element_bytes": es,
                   "kernel": os.environ.get("BRA_BACKWARD_KERNEL") or "auto (tensor cores where covered)"},
        "roofline": {"kernel": "bra_attend_backward", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                     "algorithmic_bytes": min_bytes, "launch_ms": ms},
        "gpu_launches": args.steps,
        "clocks": clocks.report(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.backward:
        return run_backward(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
