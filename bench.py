"""Benchmark of the MoE-layer forward pass on B200: tokens/s, roofline fraction, oracle baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 3] [--impl ours|reference]

A step is one moe_layer_forward (router, dispatch, expert GEMMs, PR-MoE dense MLP, combine) over
the workload's T tokens of seeded synthetic input already resident in HBM. The default workload
is the largest one that the metric's configurations list: the GPT-1.3B+MoE-128 PR-MoE layer
(T=16384, d=2048, d_ff=8192, E=128, top-1, fixed dense MLP). The other workloads (top-2 E=8,
decode, GPT-350M+MoE-128) are measured in the same process as `per_workload` entries, each stage
against its roofline, and `target_bars` collects the target fractions. L2 is flushed (256 MiB write) between
timed steps; each step is timed with CUDA events on the launching stream; the K-step region is
bracketed by a barrier and device synchronisation on both sides; the max over ranks is taken.
N > 1 (under torchrun) runs N independent replicas, one per GPU: the layer has no exchange step
on one GPU's worth of tokens, so `value` is N * T / (max-over-ranks time per step).

Also measured: each kernel's share (decomposed entry points timed with events), the roofline of
the dominant kernel (algorithmic bytes or FLOPs per launch / its event-timed duration, against
MEASURED_PEAKS.json), the end-to-end throughput through the public API with pinned host buffers
(H2D of x and D2H of the output inside the timed region), SM clocks and throttle reasons sampled
through NVML during the timed region, and the CPU oracle's throughput on a bounded sample.
`train_step` times one training step of the same layer (moe_layer_forward_train keeping the
backward's state, then moe_layer_backward for a fixed output gradient with the load-balance and
z-loss terms) with events, and the backward's algorithmic bytes against the HBM peak.

--impl reference times the CPU oracle (the only reference implementation of this method) on a
bounded sample per step and prints the same JSON line with "impl": "reference".
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer forward tokens/sec on 1 B200; % of bf16 tensor peak / % of HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------- distributed plumbing

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        self.backend = None

    def init(self, device=None, backend: str = "nccl"):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
            self.pg = True
            self.backend = backend

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float, device) -> float:
        if not self.pg:
            return v
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=device if self.backend == "nccl" else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ---------------------------------------------------------------- clocks (NVML, read-only)

class ClockSampler:
    """Samples SM clock, max SM clock, power and clock-event reasons every ~2 ms in a thread."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.h = None
            try:  # the CUDA device's UUID names the same GPU in NVML whatever the visibility mask
                u = str(torch.cuda.get_device_properties(device_index).uuid)
                u = u if u.startswith("GPU-") else "GPU-" + u
                self.h = pynvml.nvmlDeviceGetHandleByUUID(u.encode())
            except Exception:
                self.h = None
            if self.h is None:
                vis = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
                ent = vis[device_index].strip() if device_index < len(vis) else str(device_index)
                self.h = (pynvml.nvmlDeviceGetHandleByUUID(ent.encode()) if ent.startswith("GPU-")
                          else pynvml.nvmlDeviceGetHandleByIndex(int(ent)))
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report no clocks rather than guess
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.time(), sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": getattr(self, "err", "no samples")}
        sms = [s[1] for s in self.samples]
        mask = 0
        for s in self.samples:
            mask |= s[2]
        reasons = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(sms)), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(sms), "source": "NVML during the timed region"}


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def to_dev(a: np.ndarray, device):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def kernel_source_hash() -> str:
    """Hash of the expert GEMM's code (grouped_gemm.cu + common.cuh), `//` comments and blank
    lines left out, so an edit of the comments keeps the committed traffic figures."""
    h = hashlib.sha256()
    for name in ("grouped_gemm.cu", "common.cuh"):
        with open(os.path.join(ROOT, "mixture_experts_layer_57_b200", "csrc", name)) as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if the kernel's source
    is unchanged since it was taken (the summary records the source hash)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.md")
    if not os.path.exists(path):
        return None, None
    src = kernel_source_hash()
    for line in open(path):
        # | workload | kernel | source hash | dram bytes per launch | ...
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[0] == workload and cells[1] == kernel and cells[2] == src:
            try:
                return float(cells[3]), path
            except ValueError:
                return None, None
    return None, None


# ---------------------------------------------------------------- CPU oracle timing

def oracle_sample_rate(w: synth.Workload, inp: dict, n_tokens: int, full_logits=None):
    """Oracle tokens/s on a sample: router logits of n tokens + routing/slots of all T tokens
    (from given logits) + expert FFN and combine of the same n tokens. Single-threaded."""
    import oracle
    if full_logits is None:
        full_logits = np.zeros((w.T, w.E), dtype=np.float32)
    tok = np.arange(n_tokens, dtype=np.int64)
    t0 = time.perf_counter()
    oracle.router_logits(inp["x"][:n_tokens], inp["w_router"], inp.get("router_bias"))
    oracle.layer_forward(inp, w.T, w.d_model, w.d_ff, w.E, w.k, w.capacity_factor,
                         add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                         logits_in=full_logits, tokens=tok)
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt


def run_reference(args, dist: Dist):
    """The reference arm: the CPU oracle, as it stands, on a bounded sample per step."""
    if dist.rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_(T=args.tokens, name=f"{w.name}-T{args.tokens}")
    if args.experts:
        w = w.with_(E=args.experts, name=f"{w.name}-E{args.experts}")
    inp = synth.make_inputs(w)
    # the GPU path's routing is not used here: the logits of all T tokens come from the oracle,
    # computed once (outside the steps); each step then pays the router for its own tokens
    import oracle
    full_logits = oracle.router_logits(inp["x"], inp["w_router"], inp.get("router_bias"))
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    per_token = oracle_sample_rate(w, inp, 2, full_logits)[1] / 2
    n = int(max(2, min(256, budget_s / per_token)))
    times = []
    for i in range(args.warmup + args.steps):
        _, dt = oracle_sample_rate(w, inp, n, full_logits)
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * float(np.mean(times))
    value = n / (ms / 1e3)
    sample = (f"{n} tokens per step (router logits, routing and slots of all {w.T} tokens from "
              f"their logits, expert FFN and combine of the {n}), single-threaded C++ oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "ms_per_step_sample": ms, "tokens_per_step_sample": n,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": sample, "host": host_cpu()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: synth.Workload, n_gpus: int) -> dict:
    return {"workload": f"{w.name}: {w.description}", "T": w.T, "d_model": w.d_model,
            "d_ff": w.d_ff, "E": w.E, "k": w.k, "capacity_factor": w.capacity_factor,
            "dense_branch": w.dense, "global_batch_tokens": w.T * n_gpus,
            "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
            "l2": "flushed between timed steps (256 MiB write)", "seed": w.seed}


# ---------------------------------------------------------------- the GPU arm

def stage_work(w: synth.Workload, R: int, E_t: int, E: int):
    """Algorithmic bytes and FLOPs of each stage of one layer forward, from the run's own routing
    (R kept rows, E_t experts with at least one kept row): every operand read once, every result
    written once."""
    T, k, dm, df = w.T, w.k, w.d_model, w.d_ff
    es = 2 if w.dtype == "bf16" else 4
    res_b = es if w.add_input_residual else 0
    out_b = es
    stage_bytes = {
        "expert_gemm1": E_t * df * dm * es + E_t * df * es + R * dm * es + R * df * es,
        "expert_gemm2": E_t * dm * df * es + E_t * dm * es + R * df * es + R * dm * 4,
        "expert_gemm2_combine": (E_t * dm * df * es + E_t * dm * es + R * df * es + R * 8
                                 + R * dm * (res_b + out_b)),
        "dense_gemm1": df * dm * es + df * es + T * dm * es + T * df * es,
        "dense_gemm2_combine": (dm * df * es + dm * es + T * df * es + T * k * 12 + R * dm * 4
                                + T * dm * (res_b + out_b)),
        "combine": (R * dm * 4 + T * dm * (res_b + out_b) + T * k * 12
                    + (T * dm * 4 if w.dense else 0)),
    }
    stage_flops = {n: 2.0 * (T if n.startswith("dense") else R) * dm * df for n in stage_bytes}
    stage_flops["combine"] = 0.0
    # PR-MoE layers with the expert and dense GEMM layers co-scheduled in one launch per layer
    # (layer 2 writes the dense output in fp32 for the combine kernel)
    dense_gemm2 = dm * df * es + dm * es + T * df * es + T * dm * 4
    stage_bytes["experts_dense_gemm1"] = stage_bytes["expert_gemm1"] + stage_bytes["dense_gemm1"]
    stage_bytes["experts_dense_gemm2"] = stage_bytes["expert_gemm2"] + dense_gemm2
    for n in ("experts_dense_gemm1", "experts_dense_gemm2"):
        stage_flops[n] = 2.0 * (R + T) * dm * df
    # the routing stages: the router's logits are 2 T d E FLOP over x (read once) and W_r, with
    # ids, gates and the dispatch ranks written (the logits are an intermediate that stays on
    # chip); dispatch moves the kept rows (read + write)
    stage_bytes["router"] = T * dm * es + E * dm * 4 + T * k * 12
    stage_flops["router"] = 2.0 * T * dm * E
    stage_bytes["dispatch"] = 2 * R * dm * es + T * k * 12 + 2 * (E + 1) * 4
    stage_flops["dispatch"] = 0.0
    return stage_bytes, stage_flops


def stage_rates(bd: dict, stage_bytes: dict, stage_flops: dict, peaks: dict) -> dict:
    """Per stage: event time, achieved TB/s-class and TFLOP/s rates, and both fractions."""
    out = {}
    for n, ms in bd.items():
        if n not in stage_bytes or ms <= 0:
            continue
        gbs = stage_bytes[n] / (ms / 1e3) / 1e9
        tfs = stage_flops[n] / (ms / 1e3) / 1e12
        out[n] = {"ms": ms, "GB/s": gbs, "TFLOP/s": tfs, "hbm_frac": gbs / peaks["hbm_gbs"],
                  "tensor_frac": tfs / peaks["bf16_tflops"],
                  "algorithmic_bytes": stage_bytes[n], "algorithmic_flops": stage_flops[n]}
    return out


def group_rate(stages: dict, names, peaks: dict) -> dict:
    """Several stages taken together (e.g. both GEMM layers of the experts)."""
    names = [n for n in names if n in stages]
    if not names:
        return None
    ms = sum(stages[n]["ms"] for n in names)
    b = sum(stages[n]["algorithmic_bytes"] for n in names)
    f = sum(stages[n]["algorithmic_flops"] for n in names)
    return {"stages": names, "ms": ms, "TFLOP/s": f / (ms / 1e3) / 1e12,
            "GB/s": b / (ms / 1e3) / 1e9, "tensor_frac": f / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
            "hbm_frac": b / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}


class LayerRun:
    """One workload's inputs resident on the device, its layer arguments and workspace."""

    def __init__(self, moe, w: synth.Workload, device, inp=None):
        self.w = w
        self.inp = synth.make_inputs(w) if inp is None else inp
        self.d = {k: to_dev(v, device) for k, v in self.inp.items()}
        d = self.d
        T, E, k, dm = w.T, w.E, w.k, w.d_model
        dense = (d["dense_w1"], d["dense_b1"], d["dense_w2"], d["dense_b2"]) if w.dense else None
        # the router weight is fixed across inference steps: split once for the tensor-core
        # logits kernel, as a serving caller would (moe_router_prepare)
        self.w_router_prepared = moe.moe_router_prepare(d["w_router"])
        self.args = moe.layer_args(d["x"], d["w_router"], d["w1"], d["b1"], d["w2"], d["b2"], k=k,
                                   capacity_factor=w.capacity_factor,
                                   router_bias=d.get("router_bias"), dense=dense,
                                   add_input_residual=w.add_input_residual, aux_alpha=w.aux_alpha,
                                   w_router_prepared=self.w_router_prepared)
        self.ws = moe.workspace(moe.moe_layer_workspace_bytes(self.args), device)
        self.out = torch.empty(T, dm, dtype=d["x"].dtype, device=device)
        self.aux = dict(expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=device),
                        expert_counts=torch.empty(E, dtype=torch.int32, device=device),
                        lb_stats=torch.empty(2 * E + 1, dtype=torch.float32, device=device))

    def step(self, moe, stream):
        moe.moe_layer_forward(self.args, self.out, aux=self.aux, ws=self.ws, stream=stream)

    def routing(self, moe) -> dict:
        w = self.w
        off = self.aux["expert_offsets"].cpu().numpy()
        counts = self.aux["expert_counts"].cpu().numpy()
        kept = off[1:] - off[:-1]
        R = int(off[-1])
        lb = self.aux["lb_stats"].cpu().numpy()
        return {"kept_rows": R, "pairs": w.T * w.k, "drop_rate": 1.0 - R / (w.T * w.k),
                "experts_touched": int((kept > 0).sum()), "max_expert_demand": int(counts.max()),
                "capacity": moe.moe_capacity(w.T, w.E, w.k, w.capacity_factor),
                "aux_loss": float(lb[-1])}


def time_steps(run: LayerRun, moe, stream, flush_buf, steps: int, warmup: int):
    """Event time (ms) of each of `steps` layer forwards, L2 flushed before each."""
    for _ in range(warmup):
        flush_buf.zero_()
        run.step(moe, stream)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush_buf.zero_()
        evs[i][0].record(stream)
        run.step(moe, stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(run.ws) == 0, "device error during the timed steps"
    return [a.elapsed_time(b) for a, b in evs]


def workload_entry(moe, w: synth.Workload, device, stream, flush_buf, peaks, steps, warmup):
    """A secondary workload measured in the same process: its step time and per-stage rates."""
    run = LayerRun(moe, w, device)
    step_ms = time_steps(run, moe, stream, flush_buf, steps, warmup)
    routing = run.routing(moe)
    bd = stage_breakdown(moe, run.args, run.out, run.aux, run.ws, stream, flush_buf,
                         reps=max(3, min(20, steps)))
    sb, sf = stage_work(w, routing["kept_rows"], routing["experts_touched"], w.E)
    stages = stage_rates(bd, sb, sf, peaks)
    ms = float(np.median(step_ms))
    entry = {"workload": f"{w.name}: {w.description}", "ms_per_step": ms,
             "tokens_per_s": w.T / (ms / 1e3), "steps": steps, "routing": routing,
             "stages": stages,
             "experts": group_rate(stages, ["expert_gemm1", "expert_gemm2",
                                            "expert_gemm2_combine"], peaks),
             "dense_mlp": group_rate(stages, ["dense_gemm1", "dense_gemm2_combine"], peaks)}
    del run
    torch.cuda.empty_cache()
    return entry


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=3, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-train", action="store_true",
                    help="skip the training-step measurement (forward keeping state + backward)")
    ap.add_argument("--skip-others", action="store_true",
                    help="skip the other workloads' per-workload entries")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the workload with T tokens instead of its own (profiling captures)")
    ap.add_argument("--experts", type=int, default=None,
                    help="run the workload with E experts instead of its own (profiling captures "
                         "that must stay small: T / E tokens per expert keeps the capacity)")
    args = ap.parse_args()
    dist = Dist()
    if args.gpus != dist.world and dist.world > 1:
        print(f"--gpus {args.gpus} but WORLD_SIZE {dist.world}", file=sys.stderr)
    if args.gpus > 1 and dist.world == 1:
        print("N > 1 runs one process per GPU: launch with torchrun", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, dist)

    from mixture_experts_layer_57_b200 import moe

    device = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(device)
    dist.init(device)
    w = synth.WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_(T=args.tokens, name=f"{w.name}-T{args.tokens}")
    if args.experts:
        w = w.with_(E=args.experts, name=f"{w.name}-E{args.experts}")
    run = LayerRun(moe, w, device)
    inp, d = run.inp, run.d
    T, E, k, dm, df = w.T, w.E, w.k, w.d_model, w.d_ff
    bf16 = w.dtype == "bf16"
    args_c, out, aux, ws = run.args, run.out, run.aux, run.ws
    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    # ---------------------------------------------------------- timed region
    for _ in range(args.warmup):
        flush_buf.zero_()
        run.step(moe, stream)
    torch.cuda.synchronize()
    launches_per_step = moe.moe_last_launch_count()
    clocks = ClockSampler(dist.local_rank)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush_buf.zero_()
        evs[i][0].record(stream)
        run.step(moe, stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms_local = float(np.mean(step_ms))
    ms = dist.max(ms_local, device)
    assert moe.moe_get_device_error(ws) == 0, "device error during the timed steps"
    value = args.gpus * T / (ms / 1e3)

    # ---------------------------------------------------------- routing statistics
    routing = run.routing(moe)
    R, E_t = routing["kept_rows"], routing["experts_touched"]

    # ---------------------------------------------------------- per-stage breakdown
    bd = stage_breakdown(moe, args_c, out, aux, ws, stream, flush_buf, reps=max(3, min(20, args.steps)))
    stage_bytes, stage_flops = stage_work(w, R, E_t, E)
    peaks, peak_src = load_peaks()
    stages = stage_rates(bd, stage_bytes, stage_flops, peaks)
    if "router" in stages and bf16:
        # the tensor-core router multiplies three bf16 parts of W_r: 3x the algorithmic FLOPs
        r = stages["router"]
        r["tensor_frac_of_three_part_work"] = 3 * r["tensor_frac"]
        r["roofline_ms"] = 1e3 * max(stage_bytes["router"] / (peaks["hbm_gbs"] * 1e9),
                                     3 * stage_flops["router"] / (peaks["bf16_tflops"] * 1e12))
    gemm_stages = [n for n in bd if n in stage_bytes and n.startswith(("expert", "dense"))]
    dom = max(gemm_stages, key=lambda n: bd[n])
    t_dom = bd[dom] / 1e3
    ai = stage_flops[dom] / stage_bytes[dom]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    kernel_name = {"expert_gemm1": "grouped_gemm (expert layer 1, bias+GeLU epilogue)",
                   "expert_gemm2": "grouped_gemm (expert layer 2, bias epilogue)",
                   "expert_gemm2_combine": "grouped_gemm (expert layer 2, bias + fused combine epilogue)",
                   "dense_gemm1": "grouped_gemm (dense MLP layer 1, bias+GeLU epilogue)",
                   "dense_gemm2_combine": "grouped_gemm (dense MLP layer 2, bias + fused combine epilogue)",
                   "experts_dense_gemm1": "co_gemm (expert layer 1 and dense MLP layer 1 in one "
                                          "launch, bias+GeLU epilogues)",
                   "experts_dense_gemm2": "co_gemm (expert layer 2 and dense MLP layer 2 in one "
                                          "launch, bias epilogues, fp32 out)"}[dom]
    traffic, _ = profiled_traffic(w.name, dom)
    if ai < ridge:
        roof = {"kernel": kernel_name, "bound": "hbm", "achieved": stage_bytes[dom] / t_dom / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"kernel": kernel_name, "bound": "tensor",
                "achieved": stage_flops[dom] / t_dom / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["algorithmic_bytes"] = stage_bytes[dom]
    roof["algorithmic_flops"] = stage_flops[dom]
    roof["launch_ms"] = bd[dom]
    roof["peak_source"] = ("measured (MEASURED_PEAKS.json, burst)" if peak_src == "measured"
                           else "fallback")
    roof["tensor_frac"] = stage_flops[dom] / t_dom / 1e12 / peaks["bf16_tflops"]
    roof["hbm_frac"] = stage_bytes[dom] / t_dom / 1e9 / peaks["hbm_gbs"]
    roof["per_stage"] = stages

    # ---------------------------------------------------------- the other workloads
    per_workload = {}
    bars = {}
    own = {"experts": group_rate(stages, ["expert_gemm1", "expert_gemm2", "expert_gemm2_combine"], peaks),
           "dense_mlp": group_rate(stages, ["dense_gemm1", "dense_gemm2_combine"], peaks),
           "experts_and_dense": group_rate(stages, ["experts_dense_gemm1", "experts_dense_gemm2"],
                                           peaks)}
    if w.dense and own["dense_mlp"] is None and not args.skip_others:
        # the dense MLP's own GEMMs, measured with the co-scheduling switched off (the bar on the
        # dense MLP is about its GEMMs alone)
        os.environ["MOE_COSCHEDULE"] = "0"
        try:
            bd_seq = stage_breakdown(moe, args_c, out, aux, ws, stream, flush_buf,
                                     reps=max(3, min(20, args.steps)))
        finally:
            os.environ.pop("MOE_COSCHEDULE", None)
        seq = stage_rates(bd_seq, stage_bytes, stage_flops, peaks)
        own["sequential"] = {"stages": seq, "ms_per_step_sum": float(sum(bd_seq.values()))}
        own["experts"] = group_rate(seq, ["expert_gemm1", "expert_gemm2"], peaks)
        own["dense_mlp"] = group_rate(seq, ["dense_gemm1", "dense_gemm2_combine"], peaks)
    if not args.skip_others and not args.tokens and not args.experts and dist.world == 1:
        for wid in (4, 5, 2):
            if wid == args.workload:
                continue
            ow = synth.WORKLOADS[wid]
            per_workload[ow.name] = workload_entry(moe, ow, device, stream, flush_buf, peaks,
                                                   steps=max(5, min(args.steps, 30)),
                                                   warmup=max(3, min(args.warmup, 5)))
    entries = dict(per_workload)
    entries[w.name] = own
    # the layer's performance targets: >= 60% of dense bf16 tensor peak on the prefill GEMMs that
    # are compute-bound (top-2 experts, PR-MoE dense MLP), >= 70% of HBM bandwidth on decode
    if "top2-e8-zipf" in entries and entries["top2-e8-zipf"]["experts"]:
        bars["top2-e8-zipf experts tensor_frac (>= 0.60)"] = entries["top2-e8-zipf"]["experts"]["tensor_frac"]
    if "gpt1.3b-prmoe128" in entries and entries["gpt1.3b-prmoe128"]["dense_mlp"]:
        bars["gpt1.3b-prmoe128 dense MLP tensor_frac (>= 0.60)"] = entries["gpt1.3b-prmoe128"]["dense_mlp"]["tensor_frac"]
    if "decode-e128" in entries and entries["decode-e128"]["experts"]:
        bars["decode-e128 experts hbm_frac (>= 0.70)"] = entries["decode-e128"]["experts"]["hbm_frac"]
    for name in ("gpt350m-moe128", "gpt1.3b-prmoe128"):
        if name in entries and entries[name]["experts"]:
            bars[f"{name} experts hbm_frac (weight-bound, >= 0.70)"] = entries[name]["experts"]["hbm_frac"]

    # ---------------------------------------------------------- priority overflow, worst case
    prio_collapse = None
    if not args.skip_others and dist.world == 1:
        prio_collapse = priority_collapse(moe, device, stream)

    # ---------------------------------------------------------- end to end through the API
    e2e = None
    if not args.skip_e2e:
        e2e = end_to_end(moe, args_c, d, w, ws, stream, args, dist, device)

    # ---------------------------------------------------------- training step
    train = None
    if not args.skip_train:
        train = train_step(moe, args_c, d, w, stream, flush_buf, args, dist, device, E_t, R)

    # ---------------------------------------------------------- CPU oracle baseline
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.skip_cpu_baseline:
        logits = torch.empty(T, E, dtype=torch.float32, device=device)
        moe.moe_router_topk(d["x"], d["w_router"], k, router_bias=d.get("router_bias"), logits=logits)
        full_logits = logits.cpu().numpy()
        per_tok = oracle_sample_rate(w, inp, 2, full_logits)[1] / 2
        n = int(max(8, min(2048, 12.0 / per_tok)))
        rate, dt = oracle_sample_rate(w, inp, n, full_logits)
        cpu = {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "host": host_cpu(),
               "sample": f"{n} tokens ({dt:.1f} s): their router logits, routing and slots of all "
                         f"{T} tokens from given logits, expert FFN and combine of the {n}; "
                         "single-threaded C++ oracle in double"}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if bf16 else "f32",
            "data": "synthetic (seeded splitmix64 + Box-Muller, shapes and distributions of the workload)",
            "config": workload_config(w, args.gpus), "roofline": roof, "cpu_baseline": cpu,
            "clocks": clocks.summary(), "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "breakdown_ms": bd, "routing": routing, "target_bars": bars,
            "headline_groups": own,
            "per_workload": per_workload, "priority_dispatch_collapse": prio_collapse,
            "train_step": train,
            "step_ms": {"min": float(min(step_ms)), "p10": float(np.percentile(step_ms, 10)),
                        "median": float(np.median(step_ms)),
                        "p90": float(np.percentile(step_ms, 90)), "max": float(max(step_ms))}}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def priority_collapse(moe, device, stream) -> dict:
    """moe_dispatch_priority when every token picks one expert (the ranking's worst case: one
    list of T pairs), event-timed at two batch sizes to show how the time grows with T."""
    out = {}
    gen = torch.Generator(device=device).manual_seed(3)
    for T in (16384, 65536):
        E, d = 128, 1024
        x = torch.randn(T, d, generator=gen, device=device).to(torch.bfloat16)
        ids = torch.full((T, 1), 3, dtype=torch.int32, device=device)
        probs = torch.rand(T, 1, generator=gen, device=device)
        C = moe.moe_capacity(T, E, 1, 1.0)
        r = moe.moe_dispatch(x, ids, E, C, priority_probs=probs)
        for _ in range(3):
            moe.moe_dispatch(x, ids, E, C, priority_probs=probs, **{k: r[k] for k in (
                "slot", "expert_counts", "expert_offsets", "row_token", "x_packed", "ws")})
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(10)]
        for a, b in evs:
            a.record(stream)
            moe.moe_dispatch(x, ids, E, C, priority_probs=probs, stream=stream, **{k: r[k] for k in (
                "slot", "expert_counts", "expert_offsets", "row_token", "x_packed", "ws")})
            b.record(stream)
        torch.cuda.synchronize()
        assert moe.moe_get_device_error(r["ws"]) == 0
        kept = int((r["slot"] >= 0).sum())
        out[str(T)] = {"ms": float(np.median([a.elapsed_time(b) for a, b in evs])),
                       "kept": kept, "capacity": C,
                       "launches": moe.moe_last_launch_count()}
    return out


def host_cpu() -> dict:
    """The host the CPU baseline ran on: logical CPUs and the CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def stage_breakdown(moe, args_c, out, aux, ws, stream, flush_buf, reps: int) -> dict:
    """Median time (ms) of each stage of moe_layer_forward, from CUDA events the library records
    at its stage boundaries (moe_layer_forward_profiled), L2 flushed before each repetition."""
    times = {}
    for _ in range(reps):
        flush_buf.zero_()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(12)]
        names = moe.moe_layer_forward_profiled(args_c, out, evs, aux=aux, ws=ws, stream=stream)
        torch.cuda.synchronize()
        for i in range(1, len(names)):
            times.setdefault(names[i], []).append(evs[i - 1].elapsed_time(evs[i]))
    assert moe.moe_get_device_error(ws) == 0
    return {n: float(np.median(v)) for n, v in times.items()}


def train_step(moe, args_c, d, w, stream, flush_buf, args, dist, device, E_t, R) -> dict:
    """One training step of the layer: moe_layer_forward_train, then moe_layer_backward for a
    fixed output gradient (with the load-balance and z-loss terms), L2 flushed before each step,
    timed with CUDA events around both calls and around each."""
    T, E, k, dm, df = w.T, w.E, w.k, w.d_model, w.d_ff
    dt = d["x"].dtype
    f32 = dict(dtype=torch.float32, device=device)
    ws_t = moe.workspace(moe.moe_layer_train_workspace_bytes(args_c), device)
    out = torch.empty(T, dm, dtype=dt, device=device)
    g = dict(dx=torch.empty(T, dm, dtype=dt, device=device), dw_router=torch.empty(E, dm, **f32),
             db_router=torch.empty(E, **f32), dw1=torch.empty(E, df, dm, **f32),
             db1=torch.empty(E, df, **f32), dw2=torch.empty(E, dm, df, **f32),
             db2=torch.empty(E, dm, **f32))
    if w.dense:
        g.update(dense_dw1=torch.empty(df, dm, **f32), dense_db1=torch.empty(df, **f32),
                 dense_dw2=torch.empty(dm, df, **f32), dense_db2=torch.empty(dm, **f32))
    gen = torch.Generator(device=device).manual_seed(57)
    dout = torch.randn(T, dm, generator=gen, device=device).to(dt)

    def fwd():
        moe.moe_layer_forward_train(args_c, out, ws=ws_t, stream=stream)

    def bwd():
        moe.moe_layer_backward(args_c, dout, g, ws_t, aux_weight=0.01, z_weight=0.001, stream=stream)

    for _ in range(max(3, min(args.warmup, 5))):
        flush_buf.zero_()
        fwd()
        bwd()
    torch.cuda.synchronize()
    launches = moe.moe_last_launch_count()
    n = max(3, min(args.steps, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    dist.barrier()
    torch.cuda.synchronize()
    for i in range(n):
        flush_buf.zero_()
        evs[i][0].record(stream)
        fwd()
        evs[i][1].record(stream)
        bwd()
        evs[i][2].record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    assert moe.moe_get_device_error(ws_t) == 0, "device error during the training steps"
    f_ms = float(np.median([e[0].elapsed_time(e[1]) for e in evs]))
    b_ms = float(np.median([e[1].elapsed_time(e[2]) for e in evs]))
    ms = dist.max(float(np.mean([e[0].elapsed_time(e[2]) for e in evs])), device)
    es = d["x"].element_size()
    # algorithmic bytes of the backward: the weights read by the two data-gradient GEMMs, fp32
    # weight and bias gradients written (every expert's), and the activations it reads/writes
    wbytes = 2 * E_t * dm * df * es + 2 * E * dm * df * 4 + E * (dm + df) * 4
    act = (T * dm * es + R * dm * 4 + R * dm * es          # combine backward
           + R * df * es * 3 + R * dm * es                  # dZ GEMM: g' and dZ, dY in
           + R * df * es + R * dm * 4                       # dX GEMM
           + R * dm * es + R * df * es * 2 + R * dm * es    # weight gradients' operands
           + T * E * 4 * 4 + T * dm * es + T * dm * 4       # router backward
           + T * dm * es + R * dm * 4 + T * dm * 4 + T * dm * es)  # dx gather
    if w.dense:
        wbytes += 2 * dm * df * es + 2 * dm * df * 4
        act += 6 * T * df * es + 4 * T * dm * es + T * dm * 4
    peaks, _ = load_peaks()
    bw_frac = (wbytes + act) / (b_ms / 1e3) / (peaks["hbm_gbs"] * 1e9)
    return {"ms_per_step": ms, "tokens_per_s": args.gpus * T / (ms / 1e3), "fwd_ms": f_ms,
            "bwd_ms": b_ms, "steps": n, "gpu_launches_bwd": launches,
            "bwd_algorithmic_bytes": wbytes + act, "bwd_hbm_frac": bw_frac,
            "objective": "sum(dout * out) + 0.01 aux + 0.001 z_loss, dout ~ N(0, 1)",
            "grads": "dx (bf16) and fp32 dW_r, db_r, dW1, db1, dW2, db2 (+ dense MLP)"}


def end_to_end(moe, args_c, d, w, ws, stream, args, dist, device) -> dict:
    """Same metric through the public call with host buffers, as a serving loop runs it: every
    step copies its x from pinned host memory to the device (copy-in stream), runs
    moe_layer_forward (compute stream) and copies the output back to pinned host memory
    (copy-out stream), all inside the timed region; two device buffers let step i's copies
    overlap steps i - 1 and i + 1 (events order each buffer's reuse). Also reported: the same
    with the three operations serialised on one stream."""
    from mixture_experts_layer_57_b200 import moe as _moe
    T, dm = w.T, w.d_model
    x_dev0 = d["x"]
    x_pin = torch.empty(x_dev0.shape, dtype=x_dev0.dtype, pin_memory=True)
    x_pin.copy_(x_dev0.cpu())
    xs = [torch.empty_like(x_dev0) for _ in range(2)]
    outs = [torch.empty(T, dm, dtype=x_dev0.dtype, device=device) for _ in range(2)]
    out_pins = [torch.empty(T, dm, dtype=x_dev0.dtype, pin_memory=True) for _ in range(2)]
    step_args = []
    for b in range(2):
        a = _moe.LayerArgs()
        ctypes_copy(a, args_c)
        a.x = xs[b].data_ptr()
        step_args.append(a)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    in_done = [ev(), ev()]
    fwd_done = [ev(), ev()]
    out_done = [ev(), ev()]
    started = [False, False]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(fwd_done[b])      # the forward of step i - 2 has read xs[b]
            xs[b].copy_(x_pin, non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if started[b]:
            stream.wait_event(out_done[b])        # step i - 2's output has been copied out
        moe.moe_layer_forward(step_args[b], outs[b], ws=ws, stream=stream)
        fwd_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(fwd_done[b])
            out_pins[b].copy_(outs[b], non_blocking=True)
            out_done[b].record(s_out)
        started[b] = True

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 50))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(n):
        step(i)
    stream.wait_event(out_done[(n - 1) % 2])
    t1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(t0.elapsed_time(t1) / n, device)
    assert torch.equal(out_pins[(n - 1) % 2], outs[(n - 1) % 2].cpu())

    # the serial form: copy in, forward, copy out on one stream, each step waiting for the last
    def serial():
        xs[0].copy_(x_pin, non_blocking=True)
        moe.moe_layer_forward(step_args[0], outs[0], ws=ws, stream=stream)
        out_pins[0].copy_(outs[0], non_blocking=True)

    for _ in range(3):
        serial()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        serial()
        b.record(stream)
    torch.cuda.synchronize()
    ms_serial = dist.max(float(np.mean([a.elapsed_time(b) for a, b in evs])), device)
    es = x_dev0.element_size()
    return {"value": args.gpus * T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": n,
            "h2d_bytes_per_step": T * dm * es, "d2h_bytes_per_step": T * dm * out_pins[0].element_size(),
            "pipeline": "copy-in, compute and copy-out streams, two device buffers",
            "serial": {"value": args.gpus * T / (ms_serial / 1e3), "ms_per_step": ms_serial}}


def ctypes_copy(dst, src):
    """Field-by-field copy of a ctypes structure."""
    for name, _ in src._fields_:
        setattr(dst, name, getattr(src, name))


if __name__ == "__main__":
    sys.exit(main())
