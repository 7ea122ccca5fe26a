"""Benchmark: one MoE layer forward (router -> top-k -> dispatch layout -> permute ->
grouped SwiGLU experts -> combine) per step, on synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wide] [--impl reference]

Default workload: the wide-expert prefill layer (N=8192 tokens, d=7168, 256 routed + 1
shared expert, top-8 of 4 of 8 groups, I=2048, bf16), the largest single-GPU workload and
the one the grouped-GEMM target is stated on.  Each step runs through the library's C
ABI; inputs are resident in HBM when the timed region starts and L2 is flushed (a 256 MiB
write) before every step, outside the step's CUDA-event bracket.  On one GPU the default
run then measures the other workloads (fine, decode, hot, hot_cal, tiny) the same way,
with fewer steps, and reports each one's times, rates and roofline fractions under
"workloads".  Under torchrun each rank runs its own independent batch (weak scaling, no
collective on the data path); the time is the max over ranks.  Prints one JSON line on
rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s; grouped-GEMM TFLOP/s and permute/combine GB/s vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="wide")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload summary of the other workloads (one GPU, default workload)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--movement-sweep", action="store_true",
                    help="permute / combine bandwidth at the workload's row shape for N = 128 .. 16384 "
                         "(one JSON line with the curve)")
    ap.add_argument("--fp8", action="store_true",
                    help="the FP8 (e4m3) expert path: quantised dispatch payload and expert GEMMs")
    ap.add_argument("--mx", action="store_true",
                    help="the block-scaled (MX) e4m3 expert path: E8M0 scales per 32 K values, applied "
                         "by the tensor cores")
    ap.add_argument("--ep", type=int, default=0, metavar="P",
                    help="expert parallelism with P ranks emulated on this GPU (moe_ep_*): per-stage times "
                         "of all ranks, the one-GPU layer beside it, and the NVLink bytes a real P-GPU step moves")
    ap.add_argument("--ep-real", action="store_true",
                    help="under torchrun (2+ GPUs): the expert-parallel layer across the ranks over NVLink "
                         "(moe_ep_layer_forward_overlapped, windows mapped through CUDA IPC)")
    ap.add_argument("--eplb", type=int, default=0, metavar="R",
                    help="run the routed experts over E + R physical slots (redundant copies of the "
                         "hot experts, planned from the batch's own counts)")
    return ap.parse_args()


def describe(cfg):
    return (f"{cfg.name}: N={cfg.N} d={cfg.d} E={cfg.E}+{cfg.S} shared k={cfg.k} I={cfg.I} P={cfg.P} "
            f"{cfg.score}{' renorm' if cfg.renormalize else ''}"
            f"{f' groups {cfg.topk_groups}/{cfg.n_groups}' if cfg.n_groups > 1 else ''} {cfg.dtype}")


def algorithmic(cfg, n_e_touched=None):
    """Algorithmic work of one layer step: FLOPs of the two grouped GEMMs and bytes of the
    movement kernels (each row read or written once)."""
    A, S, N, d, I, E = cfg.N * cfg.k, cfg.S, cfg.N, cfg.d, cfg.I, cfg.E
    b = 2 if cfg.dtype == "bf16" else 4
    rows = A + S * N
    touched = E if n_e_touched is None else n_e_touched
    return dict(
        fc1_flops=2.0 * rows * d * 2 * I,
        fc2_flops=2.0 * rows * I * d,
        ffn_flops=6.0 * rows * d * I,
        fc1_weight_bytes=(touched + S) * 2 * I * d * b,
        permute_bytes=(N + A) * d * b,
        combine_bytes=(A + S * N + N) * d * b,
        router_flops=2.0 * N * d * E,
    )


SPEC_BF16_TFLOPS = 2250.0   # B200 dense bf16 tensor rate (nominal, no sparsity)
SPEC_SM_MHZ = 1965.0        # the SM clock that nominal rate is quoted at (clocks.max.sm)


def config_dict(cfg, world: int) -> dict:
    """The workload description both arms print (identical keys, so the lines compare)."""
    return {"workload": describe(cfg), "tokens_per_gpu": cfg.N,
            "l2": "flushed before every step (256 MiB write, outside the step's event bracket)",
            "parallelism": f"{world} independent replicas (one batch per GPU)"}


def touched_weight_bytes(cfg, touched: int) -> float:
    """W13 and W2 bytes of the experts that received rows plus the shared experts."""
    b = 2 if cfg.dtype == "bf16" else 4
    return (touched + cfg.S) * 3.0 * cfg.d * cfg.I * b


def roofline_layer_ms(cfg, touched: int, hbm_gbs: float, tensor_tflops: float) -> dict:
    """Roofline time of each step of one layer and their sum: the router, permute and
    combine at HBM bandwidth (their algorithmic bytes), the FFN at the slower of its FLOPs
    at the tensor peak and its touched weight bytes at HBM bandwidth."""
    alg = algorithmic(cfg, touched)
    b = 2 if cfg.dtype == "bf16" else 4
    bw = hbm_gbs * 1e9
    router_bytes = (cfg.N * cfg.d + cfg.E * cfg.d) * b + cfg.N * cfg.E * 4 + cfg.N * cfg.k * 8
    ffn_tc = alg["ffn_flops"] / (tensor_tflops * 1e12)
    ffn_hbm = touched_weight_bytes(cfg, touched) / bw
    parts = {"router": max(router_bytes / bw, alg["router_flops"] / (tensor_tflops * 1e12)),
             "permute": alg["permute_bytes"] / bw, "ffn": max(ffn_tc, ffn_hbm),
             "combine": alg["combine_bytes"] / bw}
    return {"ms": 1e3 * sum(parts.values()), "parts_ms": {k: 1e3 * v for k, v in parts.items()},
            "ffn_bound": "tensor" if ffn_tc >= ffn_hbm else "hbm"}


def spec_at_clock(sm_mhz) -> float:
    """The nominal dense bf16 rate scaled to the SM clock the kernels ran at."""
    return SPEC_BF16_TFLOPS * (float(sm_mhz) / SPEC_SM_MHZ if sm_mhz else 1.0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {k: float(j[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, clock_rec):
    """The bf16 peak that matches how the kernel ran: the burst figure when the SM clock
    stayed near its maximum during the timed steps, the sustained (power-capped) figure
    when it did not."""
    if clock_rec and clock_rec.get("sm_mhz") and clock_rec.get("sm_max_mhz") and \
            clock_rec["sm_mhz"] >= 0.95 * clock_rec["sm_max_mhz"]:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


class ClockSampler:
    """Reads the SM clock and the clock-event (throttle) reasons through NVML every 2 ms
    in a background thread while the timed steps run (reading only; no setting is
    changed)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, device_index):
        import threading
        self.samples = []
        self.stop_ev = threading.Event()
        self.thread = None
        self.nvml = None
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            pr = torch.cuda.get_device_properties(device_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.nvml = nv
        except Exception:
            self.nvml = None

    def _run(self):
        nv = self.nvml
        while not self.stop_ev.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
            except Exception:
                pass
            self.stop_ev.wait(0.002)

    def mark_timed(self):
        """Samples from here on belong to the timed steps."""
        self.timed_from = len(self.samples)

    def start(self):
        self.timed_from = 0
        if self.nvml is None:
            return
        import threading
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.nvml is None or self.thread is None:
            return None
        self.stop_ev.set()
        self.thread.join()
        timed = self.samples[getattr(self, "timed_from", 0):] or self.samples
        if not timed:
            return None
        sm = sorted(x for x, _ in timed)
        reasons = set()
        for _, bits in timed:
            for name, const in self.REASONS.items():
                if hasattr(self.nvml, const) and bits & getattr(self.nvml, const):
                    reasons.add(name)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "sm_min_mhz": sm[0],
                "reasons": sorted(reasons), "samples": len(sm), "source": "NVML, every 2 ms, during the timed steps"}


def source_hash(*files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, src_hash):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    r = rec.get(f"{kernel}/{workload}")
    if r and r.get("source_hash") == src_hash:
        return r["bytes_per_launch"]
    return None


# ------------------------------------------------------------------------------ multi-rank aggregation
def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The largest of the ranks' values (each rank passes its own); world == 1: value."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, slowest_ms_per_step: float) -> float:
    """Every rank processes its own batch of tokens_per_rank tokens per step (weak scaling);
    the job's rate is all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (slowest_ms_per_step / 1e3)


# ------------------------------------------------------------------------------ oracle arm
def cpu_slice_tokens(cfg) -> int:
    """Tokens per oracle slice: the oracle converts every touched expert's weights to
    float64 once per slice, which dominates on the 7168-wide experts (about 0.15 s per
    expert), so those workloads take 16-token slices; the others 128."""
    return min(cfg.N, 16 if cfg.d >= 7168 else 128)


def oracle_slice(cfg, inp, s0, n_tok):
    """The float64 oracle (as it stands) on tokens [s0, s0 + n_tok) of the workload, its
    layer steps timed one by one in the pages' order.  Returns (tokens, seconds, seconds
    per step: routing + layout, permute, experts, combine)."""
    from oracle import moe_oracle as O
    xs = inp["x"][s0:s0 + n_tok]
    c = cfg.replace(N=xs.shape[0])
    w13, w2, wg, bias, owner = inp["w13"], inp["w2"], inp["w_gate"], inp["bias"], inp["expert_owner"]
    ta = time.perf_counter()
    ids = O.select_experts(O.router_logits(xs, wg, bias), c.k, c.n_groups, c.topk_groups)
    g = O.gate_weights(O.gate_logits(c, xs, wg, bias), ids, c.score, c.renormalize)
    lay = O.dispatch_layout(ids, c.E, c.P, owner, c.S)
    tb = time.perf_counter()
    xp = O.permute(xs, lay, c.k)
    tc = time.perf_counter()
    o = O.experts_on_rows(xp, lay, w13, w2, c.E)
    shared = [O.swiglu_expert(xs, w13[c.E + s], w2[c.E + s]) for s in range(c.S)]
    td = time.perf_counter()
    O.combine(o, lay, g, c.N, c.k, shared)
    te = time.perf_counter()
    return xs.shape[0], te - ta, (tb - ta, tc - tb, td - tc, te - td)


PHASES = ("routing_layout", "permute", "ffn", "combine")


def cpu_inputs(inp):
    return {k: (t.cpu() if t is not None else None) for k, t in inp.items()}


def oracle_tokens_per_s(cfg, seconds, inputs, slice_tokens=None):
    """Time the oracle on consecutive slices of the workload until about ``seconds`` have
    passed (at least one slice).  Returns (tokens/s, tokens, seconds, threads, seconds spent
    in each step of the layer)."""
    import torch
    threads = len(os.sched_getaffinity(0))
    torch.set_num_threads(threads)
    n_slice = slice_tokens or cpu_slice_tokens(cfg)
    phases = dict.fromkeys(PHASES, 0.0)
    done, el = 0, 0.0
    while True:
        tok, sec, ph = oracle_slice(cfg, inputs, done % cfg.N, n_slice)
        for k_, v_ in zip(PHASES, ph):
            phases[k_] += v_
        done += tok
        el += sec
        if el >= seconds:
            return done / el, done, el, threads, {k_: round(v_, 3) for k_, v_ in phases.items()}


def cpu_baseline_entry(cfg, seconds, inputs):
    v, tok, s, threads, phases = oracle_tokens_per_s(cfg, seconds, inputs)
    return {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{tok} tokens of the workload in {cpu_slice_tokens(cfg)}-token slices, whole layer in "
                      f"float64, {s:.1f} s", "phases_s": phases}


def run_reference(args, cfg, rank):
    """The reference arm: the float64 oracle as it stands, on the host cores.  Each step
    is one slice of the workload (its tokens in order, wrapping around), sized so that
    the W + K steps end within a few minutes; the line reports the steps and tokens that
    actually ran and their measured time."""
    if rank != 0:
        return
    import torch
    from moe_inputs import make_inputs
    threads = len(os.sched_getaffinity(0))
    torch.set_num_threads(threads)
    # the same draw as the GPU arm (its CUDA generators) when a GPU is present
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = cpu_inputs(make_inputs(cfg, device=dev))
    if dev == "cuda":
        torch.cuda.empty_cache()
    # slice size: one trial slice, then scaled so that a step takes about budget seconds
    budget = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    n = cpu_slice_tokens(cfg)
    _, t_trial, _ = oracle_slice(cfg, inp, 0, n)
    n = int(max(1, min(cfg.N, round(n * min(1.0, budget / max(t_trial, 1e-6))))))
    pos = 0
    for _ in range(args.warmup):
        tok, _, _ = oracle_slice(cfg, inp, pos % cfg.N, n)
        pos += tok
    tot_tok, tot_s, phases = 0, 0.0, dict.fromkeys(PHASES, 0.0)
    for _ in range(args.steps):
        tok, sec, ph = oracle_slice(cfg, inp, pos % cfg.N, n)
        pos += tok
        tot_tok += tok
        tot_s += sec
        for k_, v_ in zip(PHASES, ph):
            phases[k_] += v_
    v = tot_tok / tot_s
    sample = (f"{args.steps} steps of {n} tokens each ({tot_tok} tokens, consecutive slices of the workload), "
              f"whole layer in float64, {tot_s:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * tot_s / args.steps,
        "tokens_per_step": n, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded normal inputs, random-init weights)",
        "config": config_dict(cfg, args.gpus),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample,
                         "phases_s": {k: round(x, 3) for k, x in phases.items()}},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "each step is one bounded slice of the workload (tokens_per_step tokens), not the whole batch",
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ our arm
def e2e_pipelined(forward, x, y, flush, steps):
    """End to end through the public call, the way a serving loop runs it: every step
    copies its input from pinned host memory to the device (copy-in stream), runs the
    layer (current stream) and copies its result back to pinned host memory (copy-out
    stream); with two device buffers each way, step i's layer overlaps step i+1's input
    copy and step i-1's result copy.  Returns ms per step, device-timed from the first
    copy-in to the last copy-out (L2 flushed before every layer call, inside the window)."""
    import torch
    dev = x.device
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    comp = torch.cuda.current_stream(dev)
    x_host = x.cpu().pin_memory()
    y_hosts = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    x_devs = [torch.empty_like(x) for _ in range(2)]
    y_devs = [torch.empty_like(y) for _ in range(2)]
    in_done = [torch.cuda.Event() for _ in range(steps)]
    comp_done = [torch.cuda.Event() for _ in range(steps)]
    out_done = [torch.cuda.Event() for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(steps):
        b = i % 2
        if i >= 2:
            s_in.wait_event(comp_done[i - 2])  # the layer of step i-2 has read x_devs[b]
        with torch.cuda.stream(s_in):
            x_devs[b].copy_(x_host, non_blocking=True)
        in_done[i].record(s_in)
        comp.wait_event(in_done[i])
        if i >= 2:
            comp.wait_event(out_done[i - 2])   # y_devs[b] has been copied out
        flush.zero_()
        forward(x_devs[b], y_devs[b])
        comp_done[i].record(comp)
        s_out.wait_event(comp_done[i])
        with torch.cuda.stream(s_out):
            y_hosts[b].copy_(y_devs[b], non_blocking=True)
        out_done[i].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def run_movement_sweep(args, cfg, local):
    """Permute and combine at the workload's shapes (d, k, E, S) for N = 128 .. 16384:
    each kernel timed alone, L2 flushed before every launch, median of 10, at full clock
    (an idle pause before each size)."""
    import torch
    import dispatch_combine_grouped_b200 as moe
    from moe_inputs import make_inputs

    dev = torch.device("cuda", local)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    curve = []
    n = 128
    while n <= 16384:
        c = cfg.replace(N=n)
        inp = make_inputs(c, device=dev, with_experts=False)
        _, ids, w = moe.route(c, inp["x"], inp["w_gate"], inp["bias"])
        lay = moe.dispatch_layout(c, ids, inp["expert_owner"])
        rows = n * c.k + c.S * n
        xp = torch.empty(n * c.k, c.d, dtype=inp["x"].dtype, device=dev)
        out = torch.randn(rows, c.d, device=dev).to(inp["x"].dtype)
        y = torch.empty_like(inp["x"])
        alg = algorithmic(c)
        time.sleep(0.5)
        res = {"N": n}
        for name, fn, byt in [("permute", lambda: moe.permute(c, lay, inp["x"], out=xp), alg["permute_bytes"]),
                              ("combine", lambda: moe.combine(c, lay, out, y=y), alg["combine_bytes"])]:
            ts = []
            for _ in range(10):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            ms = sorted(ts)[5]
            res[f"{name}_us"] = ms * 1e3
            res[f"{name}_gbs"] = byt / (ms / 1e3) / 1e9
        curve.append(res)
        del inp, xp, out, y, lay
        n *= 2
    peaks, src = load_peaks()
    print(json.dumps({"movement_sweep": describe(cfg), "hbm_gbs_measured": peaks["hbm_gbs"], "curve": curve}),
          flush=True)


def run_ep(args, cfg, local):
    """The expert-parallel layer (moe_ep_*) with P ranks emulated on this GPU: P windows,
    each rank's stages issued for all ranks in turn on one stream (every wait finds its
    flags set).  Times each stage summed over the ranks, L2 flushed before every step,
    beside the one-GPU layer on the same batch, and counts the rows a real P-GPU step
    sends across NVLink (assignments whose owner is not their source)."""
    import torch
    import dispatch_combine_grouped_b200 as moe
    from dispatch_combine_grouped_b200 import ep
    from moe_inputs import make_inputs

    P = args.ep
    if cfg.N % P or cfg.E % P:
        raise SystemExit(f"--ep {P}: N and E of {cfg.name} must be multiples of P")
    dev = torch.device("cuda", local)
    gcfg = cfg.replace(P=P)
    inp = make_inputs(gcfg, device=dev)
    n = cfg.N // P
    rc = gcfg.replace(N=n)
    mx = bool(args.mx)
    f8 = bool(args.fp8) and not mx
    E, S, R = cfg.E, cfg.S, args.eplb
    if R and (f8 or mx):
        raise SystemExit("--ep with --eplb runs the bf16 path")
    # the workload's placement (e.g. the hot-spot table), else contiguous; with EPLB the
    # copies are planned from this batch's counts and the slot weights placed once
    # (load-time steps); each rank maps its assignments to slots inside the step
    _, ids0, _ = moe.route(gcfg, inp["x"], inp["w_gate"], inp["bias"])
    n_e0 = torch.bincount(ids0.reshape(-1).long(), minlength=E).cpu().numpy()
    pc, owner_t, w13_ep, w2_ep = rc, inp["expert_owner"], inp["w13"], inp["w2"]
    own0 = owner_t.cpu().numpy() if owner_t is not None else np.arange(E) // (E // P)
    slots_of = [[e for e in range(E) if own0[e] == r] for r in range(P)]
    load = np.bincount(own0, weights=n_e0, minlength=P)
    if R:
        plan = moe.eplb_plan(n_e0, R, P)
        load = np.asarray(plan["owner_load"], dtype=np.float64)
        pc = moe.physical_config(rc, R)
        owner_t = torch.tensor(plan["slot_owner"], dtype=torch.int32, device=dev)
        rep_off = torch.tensor(plan["replica_off"], dtype=torch.int32, device=dev)
        rep_slots = torch.tensor(plan["replica_slots"], dtype=torch.int32, device=dev)
        slots_of = [[q for q in range(E + R) if plan["slot_owner"][q] == r] for r in range(P)]
        w13_ep = moe.eplb_place_weights(plan["slot_expert"], E, S, inp["w13"])
        w2_ep = moe.eplb_place_weights(plan["slot_expert"], E, S, inp["w2"])
        phys = [torch.empty(n, cfg.k, dtype=torch.int32, device=dev) for _ in range(P)]
        eplb_ws = torch.empty(max(moe.eplb_workspace_bytes(rc), 1), dtype=torch.uint8, device=dev)
    E_slots = pc.E
    # receive rows per owner, sized from this batch's counts as the pages size receive
    # buffers from the exchanged counts (+ k*P rows for the per-rank split of copies)
    cap = int(-(-(int(load.max()) + cfg.k * P) // 128) * 128)
    groups, windows = ep.emulated_groups(pc, cap, owner_t)
    ws = [ep.alloc_ws(pc, cap, fp8=f8, mx=mx) for _ in range(P)]
    handles = [ep.Handle(pc, len(slots_of[r])) for r in range(P)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    wts = []
    if f8 or mx:  # weights quantised once (a load-time step), then sliced per owner
        quant = moe.quantize_mx if mx else moe.quantize_fp8
        w13_q, w13_s = quant(inp["w13"])
        w2_q, w2_s = quant(inp["w2"])
        del inp["w13"], inp["w2"]
    for r in range(P):
        idx = torch.tensor(slots_of[r] + list(range(E_slots, E_slots + S)), device=dev)
        if f8 or mx:
            wts.append(tuple(t.index_select(0, idx) for t in (w13_q, w13_s, w2_q, w2_s)))
        else:
            wts.append((w13_ep.index_select(0, idx), w2_ep.index_select(0, idx)))
    xs = [inp["x"][r * n:(r + 1) * n] for r in range(P)]
    qs = None
    if f8:
        qs = [(torch.empty(n, cfg.d, dtype=torch.uint8, device=dev), torch.empty(n, dtype=torch.float32, device=dev))
              for _ in range(P)]
    elif mx:
        qs = [(torch.empty(n, cfg.d, dtype=torch.uint8, device=dev),
               torch.empty(n, cfg.d // 32, dtype=torch.uint8, device=dev)) for _ in range(P)]
    routed = [moe.route(rc, xs[r], inp["w_gate"], inp["bias"]) for r in range(P)]
    ys = [torch.empty(n, cfg.d, dtype=cfg.torch_dtype, device=dev) for _ in range(P)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stages = ["route", "notify", "layout", "dispatch", "ffn", "combine"]

    def step(ev=None, fev=None):
        def mark(i):
            if ev is not None:
                ev[i].record()
        mark(0)
        for r in range(P):
            moe.route(rc, xs[r], inp["w_gate"], inp["bias"], out=routed[r])
            if f8:
                moe.quantize_fp8(xs[r], out=qs[r][0], scale=qs[r][1])
            elif mx:
                moe.quantize_mx(xs[r], out=qs[r][0], sf=qs[r][1])
            if R:
                moe.eplb_assign(rc, routed[r][1], rep_off, rep_slots, E + R, status=status, out=phys[r], ws=eplb_ws)
        ids_ep = phys if R else [rt[1] for rt in routed]
        mark(1)
        for r in range(P):
            ep.notify(pc, groups[r], ids_ep[r], ws[r], status)
        mark(2)
        for r in range(P):
            ep.layout(pc, groups[r], ids_ep[r], handles[r], ws[r], owner_t, status)
        mark(3)
        for r in range(P):
            if f8:
                ep.dispatch_fp8(pc, groups[r], qs[r][0], qs[r][1], routed[r][2], handles[r])
            elif mx:
                ep.dispatch_mx(pc, groups[r], qs[r][0], qs[r][1], routed[r][2], handles[r])
            else:
                ep.dispatch(pc, groups[r], xs[r], routed[r][2], handles[r])
        mark(4)
        for r in range(P):
            if fev is not None:
                fev[r][0].record()
            if f8:
                ep.expert_ffn_fp8(pc, groups[r], qs[r][0], qs[r][1], *wts[r], handles[r], ws[r], status)
            elif mx:
                ep.expert_ffn_mx(pc, groups[r], qs[r][0], qs[r][1], *wts[r], handles[r], ws[r], status)
            else:
                ep.expert_ffn(pc, groups[r], xs[r], wts[r][0], wts[r][1], handles[r], ws[r], status)
            if fev is not None:
                fev[r][1].record()
        mark(5)
        for r in range(P):
            ep.combine(pc, groups[r], handles[r], y=ys[r], status=status)
        mark(6)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise SystemExit(f"EP step reported status {int(status.item())}")
    # per-stage times (eager launches, events between the stages)
    tot = [0.0] * len(stages)
    ffn_owner = [0.0] * P   # each owner's expert FFN (the critical path of a real P-GPU step)
    for _ in range(args.steps):
        flush.zero_()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(P)]
        step(ev, fev)
        torch.cuda.synchronize()
        for i in range(len(stages)):
            tot[i] += ev[i].elapsed_time(ev[i + 1])
        for r in range(P):
            ffn_owner[r] += fev[r][0].elapsed_time(fev[r][1]) / args.steps
    # the whole step as one CUDA graph replay (no host launch gaps); each replay is a new
    # step because the step number lives in the windows
    cs = torch.cuda.Stream(device=dev)
    cs.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        step()
    step_ms = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        step_ms.append(a.elapsed_time(b))
    if int(status.item()) != 0:
        raise SystemExit(f"EP step reported status {int(status.item())}")
    # the one-GPU layer on the same batch (same experts, one owner per E/P block)
    if f8:
        ws1 = torch.empty(moe.workspace_bytes_fp8(gcfg), dtype=torch.uint8, device=dev)

        def one_gpu(y=None):
            return moe.layer_forward_fp8(gcfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], w13_q,
                                         w13_s, w2_q, w2_s, y=y, ws=ws1)
    elif mx:
        ws1 = torch.empty(moe.workspace_bytes_mx(gcfg), dtype=torch.uint8, device=dev)

        def one_gpu(y=None):
            return moe.layer_forward_mx(gcfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], w13_q,
                                        w13_s, w2_q, w2_s, y=y, ws=ws1)
    else:
        ws1 = moe.alloc_workspace(gcfg, dev)

        def one_gpu(y=None):
            return moe.layer_forward(gcfg, inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"],
                                     inp["w2"], y=y, ws=ws1)
    y1 = one_gpu()
    one = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        one_gpu(y1)
        b.record()
        torch.cuda.synchronize()
        one.append(a.elapsed_time(b))
    same = bool(torch.equal(torch.cat(ys), y1))
    # rows a real P-GPU step moves between GPUs (owner != source), per rank and direction
    eb = 2 if cfg.dtype == "bf16" else 4
    cross = []
    for r in range(P):
        dest = handles[r].as_dict()["dest"]
        owner = torch.div(dest[dest >= 0], cap, rounding_mode="floor")
        cross.append(int((owner != r).sum().item()))
    owner_rows = [int(h.as_dict()["owner_off"][-1].item()) for h in handles]
    row_bytes = cfg.d * eb                      # output rows (combine) and bf16 payload rows
    pay_bytes = cfg.d + cfg.d // 32 if mx else cfg.d * (1 if f8 else eb)  # dispatch payload rows (e4m3: d
    #                                                 bytes, plus d/32 scale bytes for MX)
    max_cross = max(cross) * pay_bytes
    med = sorted(step_ms)[len(step_ms) // 2]
    stage_ms = {k: tot[i] / args.steps for i, k in enumerate(stages)}
    x_bytes, rows_bytes = cfg.N * row_bytes, cfg.N * cfg.k * row_bytes
    pay_x, pay_rows = cfg.N * pay_bytes, cfg.N * cfg.k * pay_bytes
    print(json.dumps({
        "metric": "MoE-layer tokens/s, expert-parallel path with P ranks emulated on one GPU"
                  + (" (FP8 dispatch and experts, bf16 combine)" if f8 else "")
                  + (" (MXFP8 dispatch and experts, bf16 combine)" if mx else ""),
        "value": cfg.N / (med / 1e3), "unit": "tokens/s", "n_gpus": 1, "ep_ranks_emulated": P,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": med,
        "dtype": "e4m3 (scaled), bf16 out" if f8 else ("e4m3 + E8M0 per 32, bf16 out" if mx else cfg.dtype),
        "config": {"workload": describe(gcfg), "tokens_per_rank": n, "capacity_rows_per_owner": cap,
                   "l2": "flushed before every step"},
        "how": "ms_per_step: the emulated step of all P ranks as one CUDA graph replay; stages: eager launches "
               "with events between the stages (all ranks of a stage together)",
        "stages_ms_all_ranks": stage_ms,
        "dispatch_gbs_local": (pay_x + pay_rows) / (stage_ms["dispatch"] / 1e3) / 1e9,
        "combine_gbs_local": (rows_bytes + S * x_bytes + x_bytes) / (stage_ms["combine"] / 1e3) / 1e9,
        "one_gpu_layer_ms": sorted(one)[len(one) // 2],
        "y_bit_identical_to_one_gpu_layer": same,
        "nvlink": {"cross_rows_per_rank": cross, "dispatch_bytes_per_rank": max_cross,
                   "combine_bytes_per_rank": max(cross) * row_bytes,
                   "roofline_us_at_770_gbs": (max_cross + max(cross) * row_bytes) / 770e9 * 1e6,
                   "note": "bytes a real P-GPU step sends from (and receives into) each GPU in the dispatch and "
                           "in the combine; the roofline time is their sum at the measured 770 GB/s peer copy; "
                           "not measured here (one GPU)"},
        "owner_receive_rows": owner_rows,
        "ffn_ms_per_owner": [round(v, 4) for v in ffn_owner],
        "ffn_ms_slowest_owner": max(ffn_owner),
        "owner_rows_max_over_mean": max(owner_rows) / (sum(owner_rows) / P) if sum(owner_rows) else None,
        **({"eplb": {"copies": R, "slots": E + R}} if R else {}),
        "status": int(status.item()),
    }), flush=True)


def run_ep_real(args, cfg, world, rank, local):
    """The expert-parallel layer across the torchrun ranks, one GPU each (moe_ep_*): every
    rank holds the workload's N tokens (its own draw) and E / world experts of one shared
    weight draw, maps every other rank's window through CUDA IPC, and runs each step as
    moe_ep_layer_forward_overlapped (shared experts on a side stream).  Timed like the main
    bench: W warm-up steps, K timed steps between a barrier + synchronize on both sides, L2
    flushed before every step, the max over ranks."""
    import torch
    import torch.distributed as dist
    import dispatch_combine_grouped_b200 as moe
    from dispatch_combine_grouped_b200 import ep
    from moe_inputs import make_inputs

    if world < 2 or cfg.E % world:
        raise SystemExit("--ep-real needs torchrun with 2 or more ranks dividing E")
    dev = torch.device("cuda", local)
    rc = cfg.replace(P=world)
    inp = make_inputs(rc, device=dev)                                     # weights: one draw for all ranks
    x = make_inputs(rc, device=dev, seed_offset=rank, with_experts=False)["x"]  # tokens: this rank's own
    E, S = cfg.E, cfg.S
    owner = inp["expert_owner"]
    own = owner.cpu().numpy() if owner is not None else np.arange(E) // (E // world)
    mine = [e for e in range(E) if own[e] == rank]
    idx = torch.tensor(mine + list(range(E, E + S)), device=dev)
    w13, w2 = inp["w13"].index_select(0, idx), inp["w2"].index_select(0, idx)
    del inp["w13"], inp["w2"]
    torch.cuda.empty_cache()
    cap = int(-(-cfg.N * cfg.k * min(world, 4) // 128) * 128)   # receive rows per owner: up to 4x the mean
    window = ep.alloc_window(rc, cap)
    ws = ep.alloc_ws(rc, cap)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    y = torch.empty_like(x)
    side = torch.cuda.Stream(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    dist.barrier()
    grp, close = ep.ipc_group(rc, cap, window, owner)
    dist.barrier()

    def step():
        ep.layer_forward(rc, grp, x, inp["w_gate"], inp["bias"], w13, w2, ws, expert_owner=owner, y=y,
                         status=status, side_stream=side)

    try:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        bad = torch.tensor([int(status.item())], device=dev)
        dist.all_reduce(bad, op=dist.ReduceOp.MAX)
        if int(bad.item()) != 0:
            raise SystemExit(f"EP step reported status {int(bad.item())} on some rank")
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda.synchronize()
            dist.barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            step()
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        dist.barrier()
        med = sorted(ms)[len(ms) // 2]
        slowest = max_over_ranks(med, world, dev)
        st = torch.tensor([int(status.item())], device=dev)
        dist.all_reduce(st, op=dist.ReduceOp.MAX)
        if rank == 0:
            print(json.dumps({
                "metric": "MoE-layer tokens/s, expert-parallel across GPUs (moe_ep_layer_forward_overlapped)",
                "value": whole_job_tokens_per_s(cfg.N, world, slowest), "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": slowest, "higher_is_better": True,
                "scaling": "weak", "dtype": cfg.dtype, "data": "synthetic",
                "config": {"workload": describe(rc), "tokens_per_gpu": cfg.N, "experts_per_gpu": len(mine),
                           "capacity_rows_per_owner": cap, "l2": "flushed before every step"},
                "status": int(st.item()),
            }), flush=True)
    finally:
        torch.cuda.synchronize()
        dist.barrier()
        close()


def run_fp8(args, cfg, world, rank, local):
    """The layer with the FP8 expert path on one stream: route -> layout -> quantise x +
    FP8 permute -> FP8 grouped FFN (FC1, h quantisation, FC2) -> combine.  Weights are
    quantised once, before timing (a load-time step)."""
    import torch
    import torch.distributed  # noqa: F401
    import dispatch_combine_grouped_b200 as moe
    from moe_inputs import make_inputs

    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, device=dev, seed_offset=rank)
    A, S = cfg.N * cfg.k, cfg.S
    rows = A + S * cfg.N
    x, wg, bias, owner = inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"]
    w13_q, w13_s = moe.quantize_fp8(inp["w13"])
    w2_q, w2_s = moe.quantize_fp8(inp["w2"])
    del inp
    logits = torch.empty(cfg.N, cfg.E, dtype=torch.float32, device=dev)
    ids = torch.empty(cfg.N, cfg.k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.N, cfg.k, dtype=torch.float32, device=dev)
    layout = moe.Layout(cfg, dev)
    lay_ws = torch.empty(max(moe.layout_workspace_bytes(cfg), 1), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    x_q = torch.empty(cfg.N, cfg.d, dtype=torch.uint8, device=dev)
    x_s = torch.empty(cfg.N, dtype=torch.float32, device=dev)
    x_perm = torch.empty(A, cfg.d, dtype=torch.uint8, device=dev)
    h = torch.empty(rows, cfg.I, dtype=torch.bfloat16, device=dev)
    h_q = torch.empty(rows, cfg.I, dtype=torch.uint8, device=dev)
    h_s = torch.empty(rows, dtype=torch.float32, device=dev)
    out = torch.empty(rows, cfg.d, dtype=torch.bfloat16, device=dev)
    y = torch.empty(cfg.N, cfg.d, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(moe.workspace_bytes_fp8(cfg), 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step(ev):
        ev[0].record()
        moe.route(cfg, x, wg, bias, out=(logits, ids, w))
        ev[1].record()
        moe.dispatch_layout(cfg, ids, owner, status=status, layout=layout, ws=lay_ws)
        ev[2].record()
        moe.quantize_fp8(x, out=x_q, scale=x_s)
        moe.permute_fp8(cfg, layout, x_q, out=x_perm)
        ev[3].record()
        moe.grouped_ffn_fp8(cfg, layout, x_perm, x_q, x_s, w13_q, w13_s, w2_q, w2_s, topk_w=w, h=h, h_q=h_q,
                            h_scale=h_s, out=out)
        ev[4].record()
        moe.combine(cfg, layout, out, y=y)
        ev[5].record()

    def events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    side = torch.cuda.Stream(device=dev)

    def fused(ev):
        """The product's FP8 layer: one call, shared experts on the side stream."""
        ev[0].record()
        moe.layer_forward_fp8(cfg, x, wg, bias, owner, w13_q, w13_s, w2_q, w2_s, y=y, ws=ws, status=status,
                              side_stream=side)
        ev[1].record()

    clocks = ClockSampler(local)
    evs = [events(2) for _ in range(args.steps)]
    clocks.start()
    for _ in range(args.warmup):
        flush.zero_()
        fused(events(2))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.mark_timed()
    torch.cuda.nvtx.range_push("timed")
    for i in range(args.steps):
        flush.zero_()
        fused(evs[i])
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clock_rec = clocks.stop()
    assert status.item() == 0, f"device status {status.item()}"
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world, dev)
    # per-stage breakdown: the same kernels stage by stage on one stream
    sev = [events(6) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        step(sev[i])
    torch.cuda.synchronize()
    names = ["route", "layout", "quantize_permute", "ffn", "combine"]
    stage_ms = {n: sum(ev[j].elapsed_time(ev[j + 1]) for ev in sev) / args.steps for j, n in enumerate(names)}
    fused_ms = sum(ev[0].elapsed_time(ev[5]) for ev in sev) / args.steps  # one-stream staged step
    e2e_ms = max_over_ranks(e2e_pipelined(
        lambda xd, yd: moe.layer_forward_fp8(cfg, xd, wg, bias, owner, w13_q, w13_s, w2_q, w2_s, y=yd, ws=ws,
                                             status=status, side_stream=side), x, y, flush, max(args.steps, 8)),
        world, dev)

    alg = algorithmic(cfg)
    peaks, peak_src = load_peaks()
    # e4m3 dense rate = 2 x bf16 (4.5 vs 2.25 PFLOP/s nominal)
    bpeak, tkind = tensor_peak(peaks, clock_rec)
    fp8_peak = 2.0 * bpeak
    ffn_tflops = alg["ffn_flops"] / (stage_ms["ffn"] / 1e3) / 1e12
    # launches of one fused step: router 2, x quantisation 1, layout 3, permute 1, combine 1,
    # and per FFN group range FC1 + h quantisation + FC2, once for the routed experts and
    # once for the shared ones
    launches = 2 + 1 + 3 + 1 + 1 + 3 * (2 if S else 1)
    if rank == 0:
        line = {
            "metric": METRIC, "value": whole_job_tokens_per_s(cfg.N, world, step_ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 expert GEMM operands and dispatch payload (fp32 accumulate), bf16 activations",
            "data": "synthetic (seeded normal inputs, random-init weights)",
            "config": {"workload": describe(cfg) + " with the FP8 expert path", "tokens_per_gpu": cfg.N,
                       "l2": "flushed before every step (256 MiB write, outside the step's event bracket)",
                       "parallelism": f"{world} independent replicas (one batch per GPU)"},
            "roofline": {"kernel": "FP8 grouped FFN (FC1 + h quantisation + FC2, tcgen05 kind::f8f6f4)",
                         "bound": "tensor", "achieved": ffn_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": ffn_tflops / fp8_peak,
                         "peak_source": f"{peak_src} bf16 {tkind} x 2 (nominal e4m3 / bf16 ratio)",
                         "traffic": None, "flops_per_launch": alg["ffn_flops"], "ms_per_launch": stage_ms["ffn"]},
            "stages_ms": stage_ms,
            "ffn": {"tflops": ffn_tflops, "frac_of_fp8_peak": ffn_tflops / fp8_peak,
                    "frac_of_bf16_peak": ffn_tflops / bpeak},
            "staged_one_stream_ms_per_step": fused_ms,
            "e2e": {"value": whole_job_tokens_per_s(cfg.N, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size(), "ms_per_step": e2e_ms,
                    "how": "moe_layer_forward* per step, input copied in from pinned host memory and result "
                           "copied out, on their own streams so that step i overlaps the copies of steps "
                           "i+1 and i-1 (two device buffers each way); device-timed from the first copy-in "
                           "to the last copy-out"},
            "gpu_launches": launches * args.steps,
            "clocks": clock_rec,
        }
        print(json.dumps(line), flush=True)


def run_mx(args, cfg, world, rank, local):
    """The layer with the MX (block-scaled e4m3) expert path on one stream: route -> layout
    -> MX quantisation of x + permute of codes and scale rows -> MX grouped FFN (FC1, h
    quantisation, FC2) -> combine.  Weights are quantised once, before timing."""
    import torch
    import dispatch_combine_grouped_b200 as moe
    from moe_inputs import make_inputs

    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, device=dev, seed_offset=rank)
    A, S = cfg.N * cfg.k, cfg.S
    rows = A + S * cfg.N
    x, wg, bias, owner = inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"]
    w13_q, w13_sf = moe.quantize_mx(inp["w13"])
    w2_q, w2_sf = moe.quantize_mx(inp["w2"])
    del inp
    logits = torch.empty(cfg.N, cfg.E, dtype=torch.float32, device=dev)
    ids = torch.empty(cfg.N, cfg.k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.N, cfg.k, dtype=torch.float32, device=dev)
    layout = moe.Layout(cfg, dev)
    lay_ws = torch.empty(max(moe.layout_workspace_bytes(cfg), 1), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    x_q = torch.empty(cfg.N, cfg.d, dtype=torch.uint8, device=dev)
    x_sf = torch.empty(cfg.N, cfg.d // 32, dtype=torch.uint8, device=dev)
    x_perm = torch.empty(A, cfg.d, dtype=torch.uint8, device=dev)
    x_sf_perm = torch.empty(A, cfg.d // 32, dtype=torch.uint8, device=dev)
    h = torch.empty(rows, cfg.I, dtype=torch.bfloat16, device=dev)
    h_q = torch.empty(rows, cfg.I, dtype=torch.uint8, device=dev)
    h_sf = torch.empty(rows, cfg.I // 32, dtype=torch.uint8, device=dev)
    out = torch.empty(rows, cfg.d, dtype=torch.bfloat16, device=dev)
    y = torch.empty(cfg.N, cfg.d, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(moe.workspace_bytes_mx(cfg), 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    def step(ev):
        ev[0].record()
        moe.route(cfg, x, wg, bias, out=(logits, ids, w))
        ev[1].record()
        moe.dispatch_layout(cfg, ids, owner, status=status, layout=layout, ws=lay_ws)
        ev[2].record()
        moe.quantize_mx(x, out=x_q, sf=x_sf)
        moe.permute_mx(cfg, layout, x_q, x_sf, out=x_perm, sf_out=x_sf_perm)
        ev[3].record()
        moe.grouped_ffn_mx(cfg, layout, x_perm, x_sf_perm, x_q, x_sf, w13_q, w13_sf, w2_q, w2_sf, topk_w=w, h=h,
                           h_q=h_q, h_sf=h_sf, out=out)
        ev[4].record()
        moe.combine(cfg, layout, out, y=y)
        ev[5].record()

    side = torch.cuda.Stream(device=dev)

    def fused(ev):
        """The product's MX layer: one call, shared experts on the side stream."""
        ev[0].record()
        moe.layer_forward_mx(cfg, x, wg, bias, owner, w13_q, w13_sf, w2_q, w2_sf, y=y, ws=ws, status=status,
                             side_stream=side)
        ev[1].record()

    clocks = ClockSampler(local)
    evs = [events(2) for _ in range(args.steps)]
    clocks.start()
    for _ in range(args.warmup):
        flush.zero_()
        fused(events(2))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.mark_timed()
    torch.cuda.nvtx.range_push("timed")
    for i in range(args.steps):
        flush.zero_()
        fused(evs[i])
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clock_rec = clocks.stop()
    assert status.item() == 0, f"device status {status.item()}"
    step_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world, dev)
    sev = [events(6) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        step(sev[i])
    torch.cuda.synchronize()
    names = ["route", "layout", "quantize_permute", "ffn", "combine"]
    stage_ms = {n: sum(ev[j].elapsed_time(ev[j + 1]) for ev in sev) / args.steps for j, n in enumerate(names)}
    e2e_ms = max_over_ranks(e2e_pipelined(
        lambda xd, yd: moe.layer_forward_mx(cfg, xd, wg, bias, owner, w13_q, w13_sf, w2_q, w2_sf, y=yd, ws=ws,
                                            status=status, side_stream=side), x, y, flush, max(args.steps, 8)),
        world, dev)
    alg = algorithmic(cfg)
    peaks, peak_src = load_peaks()
    bpeak, tkind = tensor_peak(peaks, clock_rec)
    fp8_peak = 2.0 * bpeak
    ffn_tflops = alg["ffn_flops"] / (stage_ms["ffn"] / 1e3) / 1e12
    # launches of one fused step: router 2, x quantisation 1, layout 3, permute 2 (codes and
    # scale rows), combine 1, and per FFN group range FC1 (which quantises h) + FC2, once
    # for the routed experts and once for the shared ones
    launches = 2 + 1 + 3 + 2 + 1 + 2 * (2 if S else 1)
    if rank == 0:
        line = {
            "metric": METRIC, "value": whole_job_tokens_per_s(cfg.N, world, step_ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "MX e4m3 expert GEMM operands (E8M0 scale per 32 K values) and dispatch payload, "
                     "fp32 accumulate, bf16 activations",
            "data": "synthetic (seeded normal inputs, random-init weights)",
            "config": {"workload": describe(cfg) + " with the MX expert path", "tokens_per_gpu": cfg.N,
                       "l2": "flushed before every step (256 MiB write, outside the step's event bracket)",
                       "parallelism": f"{world} independent replicas (one batch per GPU)"},
            "roofline": {"kernel": "MX grouped FFN (FC1 with h quantised in its epilogue + FC2, tcgen05 kind::mxf8f6f4.block_scale)",
                         "bound": "tensor", "achieved": ffn_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": ffn_tflops / fp8_peak,
                         "peak_source": f"{peak_src} bf16 {tkind} x 2 (nominal e4m3 / bf16 ratio)",
                         "traffic": None, "flops_per_launch": alg["ffn_flops"], "ms_per_launch": stage_ms["ffn"]},
            "stages_ms": stage_ms,
            "ffn": {"tflops": ffn_tflops, "frac_of_fp8_peak": ffn_tflops / fp8_peak,
                    "frac_of_bf16_peak": ffn_tflops / bpeak},
            "e2e": {"value": whole_job_tokens_per_s(cfg.N, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size(), "ms_per_step": e2e_ms},
            "gpu_launches": launches * args.steps,
            "clocks": clock_rec,
        }
        print(json.dumps(line), flush=True)


def bench_layer(args, cfg, world, rank, local, steps, warmup, headline=True):
    """One workload: W warm-up steps, K timed steps (the product's overlapped order, CUDA
    events between the stages), a one-stream pass for the per-stage breakdown, the movement
    kernels timed on their own, the fused entry point and (headline only) the end-to-end
    measurement through the public call; the oracle's CPU baseline on rank 0 at N=1.
    Returns the JSON line (rank 0) or None."""
    import torch
    import torch.distributed as dist
    import dispatch_combine_grouped_b200 as moe
    from moe_inputs import make_inputs

    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, device=dev, seed_offset=rank)
    A, S = cfg.N * cfg.k, cfg.S
    dt = cfg.torch_dtype
    logits = torch.empty(cfg.N, cfg.E, dtype=torch.float32, device=dev)
    ids = torch.empty(cfg.N, cfg.k, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.N, cfg.k, dtype=torch.float32, device=dev)
    layout = moe.Layout(cfg, dev)
    lay_ws = torch.empty(max(moe.layout_workspace_bytes(cfg), 1), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    x_perm = torch.empty(A, cfg.d, dtype=dt, device=dev)
    h = torch.empty(A + S * cfg.N, cfg.I, dtype=dt, device=dev)
    out = torch.empty(A + S * cfg.N, cfg.d, dtype=dt, device=dev)
    y = torch.empty(cfg.N, cfg.d, dtype=dt, device=dev)
    ws = moe.alloc_workspace(cfg, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    x, wg, bias, owner, w13, w2 = inp["x"], inp["w_gate"], inp["bias"], inp["expert_owner"], inp["w13"], inp["w2"]

    side = torch.cuda.Stream(device=dev)
    main = torch.cuda.current_stream(dev)

    # redundant expert slots: plan from this batch's counts, copy the slot weights once
    R = args.eplb
    pcfg, ids_l, w13_l, w2_l, owner_l = cfg, ids, w13, w2, owner
    eplb_info = None
    if R:
        moe.route(cfg, x, wg, bias, out=(logits, ids, w))
        n_e0 = torch.bincount(ids.reshape(-1).long(), minlength=cfg.E).cpu().numpy()
        plan = moe.eplb_plan(n_e0, R, cfg.P)
        rep_off = torch.tensor(plan["replica_off"], dtype=torch.int32, device=dev)
        rep_slots = torch.tensor(plan["replica_slots"], dtype=torch.int32, device=dev)
        eplb_ws = torch.empty(max(moe.eplb_workspace_bytes(cfg), 1), dtype=torch.uint8, device=dev)
        pcfg = moe.physical_config(cfg, R)
        ids_l = torch.empty_like(ids)
        w13_l = moe.eplb_place_weights(plan["slot_expert"], cfg.E, S, w13)
        w2_l = moe.eplb_place_weights(plan["slot_expert"], cfg.E, S, w2)
        owner_l = None
        layout = moe.Layout(pcfg, dev)
        lay_ws = torch.empty(max(moe.layout_workspace_bytes(pcfg), 1), dtype=torch.uint8, device=dev)
        own = owner.long().cpu().numpy() if owner is not None else np.arange(cfg.E) // (cfg.E // cfg.P)
        before = np.bincount(own, weights=n_e0, minlength=cfg.P)
        eplb_info = {"copies": R, "slots": cfg.E + R, "planned_owner_load": plan["owner_load"].tolist(),
                     "owner_max_over_mean_before": float(before.max() / before.mean())}

    def assign():
        if R:
            moe.eplb_assign(cfg, ids, rep_off, rep_slots, cfg.E + R, status=status, out=ids_l, ws=eplb_ws)

    def step(ev):
        """One layer pass as the product runs it (moe_layer_forward_overlapped's order):
        router; then the shared experts on a side stream while layout, permute and the
        routed experts run on the main stream; join; combine."""
        ev[0].record()
        moe.route(cfg, x, wg, bias, out=(logits, ids, w))
        ev[1].record()
        if S:
            fork, join = torch.cuda.Event(), torch.cuda.Event()
            fork.record(main)
            side.wait_event(fork)
            moe.expert_fc1(pcfg, None, None, x, w13_l, h=h, groups="shared", stream=side)
            moe.expert_fc2(pcfg, None, h, w2_l, out=out, groups="shared", stream=side)
            join.record(side)
        assign()
        moe.dispatch_layout(pcfg, ids_l, owner_l, status=status, layout=layout, ws=lay_ws)
        ev[2].record()
        moe.permute(pcfg, layout, x, out=x_perm)
        ev[3].record()
        moe.expert_fc1(pcfg, layout, x_perm, x, w13_l, h=h, groups="routed")
        ev[4].record()
        moe.expert_fc2(pcfg, layout, h, w2_l, topk_w=w, out=out, groups="routed")
        ev[5].record()
        if S:
            main.wait_event(join)
        moe.combine(pcfg, layout, out, y=y)
        ev[6].record()

    def step_sequential(ev):
        """The same kernels one after another on one stream (diagnostic breakdown)."""
        ev[0].record()
        moe.route(cfg, x, wg, bias, out=(logits, ids, w))
        ev[1].record()
        assign()
        moe.dispatch_layout(pcfg, ids_l, owner_l, status=status, layout=layout, ws=lay_ws)
        ev[2].record()
        moe.permute(pcfg, layout, x, out=x_perm)
        ev[3].record()
        moe.expert_fc1(pcfg, layout, x_perm, x, w13_l, h=h)
        ev[4].record()
        moe.expert_fc2(pcfg, layout, h, w2_l, topk_w=w, out=out)
        ev[5].record()
        moe.combine(pcfg, layout, out, y=y)
        ev[6].record()

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(7)]

    clocks = ClockSampler(local)
    evs = [new_events() for _ in range(steps)]
    clocks.start()
    torch.cuda.nvtx.range_push("warmup")
    for _ in range(warmup):
        flush.zero_()
        step(new_events())
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed")
    clocks.mark_timed()
    wall0 = time.perf_counter()
    for i in range(steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clock_rec = clocks.stop()
    assert status.item() == 0, f"device status {status.item()}"

    names = ["route", "layout", "permute", "fc1", "fc2", "combine"]
    stage_ms = {n: 0.0 for n in names}
    step_ms = 0.0
    for ev in evs:
        for j, n in enumerate(names):
            stage_ms[n] += ev[j].elapsed_time(ev[j + 1])
        step_ms += ev[0].elapsed_time(ev[6])
    step_ms_max = max_over_ranks(step_ms, world, dev) / steps
    for n in names:
        stage_ms[n] /= steps

    # diagnostic: the same kernels one after another on one stream (per-stage breakdown)
    seq_evs = [new_events() for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        step_sequential(seq_evs[i])
    torch.cuda.synchronize()
    seq_ms = {n: sum(ev[j].elapsed_time(ev[j + 1]) for ev in seq_evs) / steps for j, n in enumerate(names)}
    seq_step_ms = sum(ev[0].elapsed_time(ev[6]) for ev in seq_evs) / steps

    # the movement kernels timed on their own (L2 flushed, events around the one launch),
    # after an idle pause: in the steps the GPU runs at its power cap and the SM clock sits
    # near 1.44 GHz, which slows these kernels (they are not purely HBM-bound); both are
    # reported
    time.sleep(1.5)

    def kernel_ms(fn):
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(max(steps, 5))]
        for a, b in pairs:
            flush.zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        ts = sorted(a.elapsed_time(b) for a, b in pairs)
        return ts[len(ts) // 2]
    permute_ms = kernel_ms(lambda: moe.permute(pcfg, layout, x, out=x_perm))
    combine_ms = kernel_ms(lambda: moe.combine(pcfg, layout, out, y=y))

    fused_ms, e2e_ms = None, None
    chunked = None
    if headline or cfg.name == "hot_cal":
        # the chunked pipeline (moe_layer_forward_chunked) beside the unchunked overlapped
        # forward, same steps and flushes
        chunked = {}
        for nc in (1, 2, 4):
            cws = torch.empty(max(moe.workspace_bytes_chunked(cfg, nc), 1), dtype=torch.uint8, device=dev)
            moe.layer_forward_chunked(cfg, nc, x, wg, bias, owner, w13, w2, side, y=y, ws=cws, status=status)
            cev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(min(steps, 10))]
            for a, b in cev:
                flush.zero_()
                a.record()
                moe.layer_forward_chunked(cfg, nc, x, wg, bias, owner, w13, w2, side, y=y, ws=cws, status=status)
                b.record()
            torch.cuda.synchronize()
            chunked[str(nc)] = sorted(a.elapsed_time(b) for a, b in cev)[len(cev) // 2]
            del cws
        uev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(min(steps, 10))]
        for a, b in uev:
            flush.zero_()
            a.record()
            moe.layer_forward_overlapped(cfg, x, wg, bias, owner, w13, w2, side, y=y, ws=ws, status=status)
            b.record()
        torch.cuda.synchronize()
        chunked = {"ms_per_step_by_chunks": chunked,
                   "unchunked_overlapped_ms": sorted(a.elapsed_time(b) for a, b in uev)[len(uev) // 2],
                   "how": "moe_layer_forward_chunked with 1, 2, 4 token chunks (layout and permute of chunk c "
                          "beside the experts of chunk c-1 on a side stream) against moe_layer_forward_overlapped, "
                          "median of the steps, L2 flushed before each"}
    if headline:
        # the fused entry point (one C call per step, same kernels and order as the timed step)
        fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            fev[i][0].record()
            moe.layer_forward_overlapped(cfg, x, wg, bias, owner, w13, w2, side, y=y, ws=ws, status=status)
            fev[i][1].record()
        torch.cuda.synchronize()
        fused_ms = sum(a.elapsed_time(b) for a, b in fev) / steps

        # end to end: pinned host input -> device, layer, result -> pinned host, every step
        e2e_ms = max_over_ranks(e2e_pipelined(
            lambda xd, yd: moe.layer_forward_overlapped(cfg, xd, wg, bias, owner, w13, w2, side, y=yd, ws=ws,
                                                        status=status), x, y, flush, max(steps, 8)), world, dev)

    n_e = layout["n_e"].cpu()
    touched = int((n_e > 0).sum())
    R_own = layout["recv_off"].cpu().diff().float()  # rows each virtual owner receives
    owner_imb = float(R_own.max() / R_own.mean()) if float(R_own.mean()) > 0 else None
    alg = algorithmic(cfg, touched)
    peaks, peak_src = load_peaks()
    tpeak, tkind = tensor_peak(peaks, clock_rec)
    sm_mhz = (clock_rec or {}).get("sm_mhz")
    spec = spec_at_clock(sm_mhz)
    A_rows = cfg.N * cfg.k
    routed_fc1_flops = 4.0 * A_rows * cfg.d * cfg.I
    routed_ffn_flops = 6.0 * A_rows * cfg.d * cfg.I
    fc1_tflops = routed_fc1_flops / (stage_ms["fc1"] / 1e3) / 1e12
    ffn_seq_ms = seq_ms["fc1"] + seq_ms["fc2"]
    ffn_seq_tflops = alg["ffn_flops"] / (ffn_seq_ms / 1e3) / 1e12
    ffn_weight_gbs = touched_weight_bytes(cfg, touched) / (ffn_seq_ms / 1e3) / 1e9
    roof = roofline_layer_ms(cfg, touched, peaks["hbm_gbs"], tpeak)
    # movement bandwidth from the kernels timed on their own (median launch, full clock)
    permute_gbs = alg["permute_bytes"] / (permute_ms / 1e3) / 1e9
    combine_gbs = alg["combine_bytes"] / (combine_ms / 1e3) / 1e9
    src = source_hash("dispatch_combine_grouped_b200/csrc/gemm_tc.cu", "dispatch_combine_grouped_b200/csrc/gemm_tc2.cu",
                      "dispatch_combine_grouped_b200/csrc/common.cuh")
    traffic = recorded_traffic("fc1_routed", cfg.name, src)
    value = whole_job_tokens_per_s(cfg.N, world, step_ms_max)
    launches_per_step = kernel_launches_per_step(cfg, R)
    if R:
        R_after = np.diff(layout["recv_off"].cpu().numpy())
        eplb_info["owner_max_over_mean_after"] = float(R_after.max() / R_after.mean())
        eplb_info["note"] = ("stages_ms.layout includes the replica assignment; the fused and e2e "
                             "numbers run the layer without copies")
    graph_ms = None
    if not R and rank == 0:
        if S:
            graph_ms = graph_step_ms(lambda: moe.layer_forward_overlapped(cfg, x, wg, bias, owner, w13, w2, side, y=y,
                                                                          ws=ws, status=status),
                                     flush, min(steps, 20), dev)
        else:
            graph_ms = graph_step_ms(lambda: moe.layer_forward(cfg, x, wg, bias, owner, w13, w2, y=y, ws=ws,
                                                               status=status), flush, min(steps, 20), dev)
    if rank != 0:
        return None
    ffn_rec = {"tflops": ffn_seq_tflops, "ms": ffn_seq_ms, "frac_of_peak": ffn_seq_tflops / tpeak, "peak_kind": tkind,
               "frac_of_burst_peak": ffn_seq_tflops / peaks["bf16_tflops"],
               "frac_of_sustained_peak": ffn_seq_tflops / peaks["bf16_tflops_sustained"],
               "frac_of_spec_at_clock": ffn_seq_tflops / spec,
               "weight_gbs": ffn_weight_gbs, "weight_frac_of_hbm": ffn_weight_gbs / peaks["hbm_gbs"],
               "bound": roof["ffn_bound"],
               "frac_of_roofline": roof["parts_ms"]["ffn"] / ffn_seq_ms,
               "routed_tflops_overlapped": routed_ffn_flops / ((stage_ms["fc1"] + stage_ms["fc2"]) / 1e3) / 1e12}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded normal inputs, random-init weights)",
        "config": config_dict(cfg, world),
        "roofline": {"kernel": "routed grouped FC1 + SwiGLU (tcgen05)",
                     "bound": "tensor", "achieved": fc1_tflops, "peak": tpeak, "unit": "TFLOP/s",
                     "frac": fc1_tflops / tpeak,
                     "peak_source": f"{peak_src} bf16 {tkind} (median SM clock during the timed steps "
                                    f"{sm_mhz} MHz)",
                     "frac_of_burst": fc1_tflops / peaks["bf16_tflops"],
                     "frac_of_sustained": fc1_tflops / peaks["bf16_tflops_sustained"],
                     "frac_of_spec_at_clock": fc1_tflops / spec,
                     "spec_at_clock_tflops": spec,
                     "traffic": traffic, "flops_per_launch": routed_fc1_flops, "ms_per_launch": stage_ms["fc1"],
                     "note": "timed inside the step, with the shared experts running on a side stream; "
                             "frac_of_spec_at_clock divides by 2250 TFLOP/s scaled to the median SM clock"},
        "layer_roofline": {"ms": roof["ms"], "parts_ms": roof["parts_ms"], "frac": roof["ms"] / step_ms_max,
                           "how": "router, permute, combine: algorithmic bytes at the measured HBM copy rate; "
                                  "FFN: max(FLOPs at the tensor peak, touched weight bytes at HBM)"},
        "stages_ms": stage_ms,
        "sequential": {"ms_per_step": seq_step_ms, "stages_ms": seq_ms,
                       "ffn_tflops": ffn_seq_tflops, "ffn_frac_of_peak": ffn_seq_tflops / tpeak},
        "ffn": ffn_rec,
        "permute": {"gbs": permute_gbs, "ms": permute_ms, "frac_of_hbm": permute_gbs / peaks["hbm_gbs"],
                    "frac_of_8tbs": permute_gbs / 8000.0,
                    "gbs_in_step": alg["permute_bytes"] / (seq_ms["permute"] / 1e3) / 1e9},
        "combine": {"gbs": combine_gbs, "ms": combine_ms, "frac_of_hbm": combine_gbs / peaks["hbm_gbs"],
                    "frac_of_8tbs": combine_gbs / 8000.0,
                    "gbs_in_step": alg["combine_bytes"] / (seq_ms["combine"] / 1e3) / 1e9},
        "imbalance": {"max_over_mean_n_e": float(n_e.max()) / float(n_e.float().mean()),
                      "experts_empty": int((n_e == 0).sum()),
                      "max_over_mean_owner_rows": owner_imb},
        "gpu_launches": launches_per_step * steps,
        **({"eplb": eplb_info} if R else {}),
        "clocks": clock_rec,
        "wall_s_timed": wall,
    }
    if chunked is not None:
        line["chunked"] = chunked
    if graph_ms is not None:
        ok = isinstance(graph_ms, float)
        line["graph"] = {"ms_per_step": graph_ms if ok else None,
                         "tokens_per_s": whole_job_tokens_per_s(cfg.N, 1, graph_ms) if ok else None,
                         **({} if ok else {"error": graph_ms}),
                         "how": "moe_layer_forward_overlapped (moe_layer_forward without shared experts) captured once "
                                "in a CUDA graph and replayed, median of the replays, L2 flushed before each outside "
                                "the graph: the step without host launch gaps"}
    if headline:
        line["fused_ms_per_step"] = fused_ms
        line["e2e"] = {"value": whole_job_tokens_per_s(cfg.N, world, e2e_ms), "unit": "tokens/s",
                       "h2d_bytes_per_step": x.numel() * x.element_size(),
                       "d2h_bytes_per_step": y.numel() * y.element_size(), "ms_per_step": e2e_ms,
                       "how": "moe_layer_forward_overlapped per step, input copied in from pinned host memory and "
                              "result copied out, on their own streams so that step i overlaps the copies of "
                              "steps i+1 and i-1 (two device buffers each way); device-timed from the first "
                              "copy-in to the last copy-out"}
    if not args.no_cpu_baseline and world == 1:
        cpu_s = args.cpu_seconds if headline else min(args.cpu_seconds, 6.0)
        line["cpu_baseline"] = cpu_baseline_entry(cfg, cpu_s, cpu_inputs(inp))
    return line


def kernel_launches_per_step(cfg, R=0):
    """This library's kernels in one timed step: router (GEMM + top-k), three layout
    kernels, permute, FC1 and FC2 per group range (routed, then shared), combine, and the
    replica assignment's four with redundant slots."""
    return 2 + 3 + 1 + 2 + (2 if cfg.S else 0) + 1 + (4 if R else 0)


def graph_step_ms(call, flush, n, dev):
    """The product's layer call captured once in a CUDA graph and replayed n times, the
    256 MiB L2 flush before each replay outside the graph; median replay time in ms, or an
    error string when the capture fails."""
    import torch
    try:
        cs = torch.cuda.Stream(device=dev)
        cs.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(cs):
            call()  # warm-up on the capture stream
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            call()
        ts = []
        for _ in range(n):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        del g
        return sorted(ts)[len(ts) // 2]
    except RuntimeError as e:  # capture refused: report it, keep the eager numbers
        torch.cuda.synchronize()
        return f"capture failed: {e}"


def summarize(line) -> dict:
    """The per-workload record of the default run's "workloads" field."""
    keep = {"ms_per_step": line["ms_per_step"], "tokens_per_s": line["value"], "config": line["config"]["workload"],
            "layer_roofline_ms": line["layer_roofline"]["ms"], "frac_of_layer_roofline": line["layer_roofline"]["frac"],
            "ffn": {k: line["ffn"][k] for k in ("tflops", "ms", "bound", "frac_of_roofline", "frac_of_burst_peak",
                                                 "frac_of_sustained_peak", "frac_of_spec_at_clock", "weight_gbs",
                                                 "weight_frac_of_hbm")},
            "routed_fc1": {"tflops": line["roofline"]["achieved"], "frac": line["roofline"]["frac"],
                           "frac_of_burst": line["roofline"]["frac_of_burst"], "traffic": line["roofline"]["traffic"]},
            "permute": {k: line["permute"][k] for k in ("gbs", "frac_of_hbm", "frac_of_8tbs", "gbs_in_step")},
            "combine": {k: line["combine"][k] for k in ("gbs", "frac_of_hbm", "frac_of_8tbs", "gbs_in_step")},
            "imbalance": line["imbalance"], "clocks": line["clocks"], "steps": line["steps"],
            "gpu_launches": line["gpu_launches"],
            "graph_ms_per_step": line.get("graph", {}).get("ms_per_step"),
            "graph_tokens_per_s": line.get("graph", {}).get("tokens_per_s")}
    if "cpu_baseline" in line:
        keep["cpu_baseline"] = line["cpu_baseline"]
    if "chunked" in line:
        keep["chunked"] = line["chunked"]
    return keep


def main():
    args = parse()
    from moe_inputs import CONFIGS, PROFILE_CASES
    cfg = CONFIGS[args.workload] if args.workload in CONFIGS else PROFILE_CASES[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, cfg, rank)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.movement_sweep:
        if rank == 0:
            run_movement_sweep(args, cfg, local)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.ep_real:
        run_ep_real(args, cfg, world, rank, local)
        dist.barrier()
        dist.destroy_process_group()
        return
    if args.ep:
        if rank == 0:
            run_ep(args, cfg, local)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    if args.fp8 or args.mx:
        (run_mx if args.mx else run_fp8)(args, cfg, world, rank, local)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    line = bench_layer(args, cfg, world, rank, local, args.steps, args.warmup, headline=True)
    if line is not None and world == 1 and not args.no_workloads and args.workload == "wide" and not args.eplb:
        # the other workloads, measured the same way with fewer steps (one GPU only: under
        # torchrun the ranks would hold all GPUs for the sweep)
        import torch
        torch.cuda.empty_cache()
        sweep = {"wide": summarize(line)}
        for name in ("fine", "decode", "hot", "hot_cal", "tiny"):
            w_line = bench_layer(args, CONFIGS[name], world, rank, local, min(args.steps, 10), 3, headline=False)
            sweep[name] = summarize(w_line)
            del w_line
            torch.cuda.empty_cache()
        line["workloads"] = sweep
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
