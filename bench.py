"""Benchmark of the sparse-expert MoE FFN decode layer on B200.

One step = one layer call (router, gate, selection, sparse up/down, output cast) on one batch
of synthetic decode tokens.  Default workload: the Llama-4-Maverick-shaped bf16 layer (H5120,
128 routed experts top-1 with a sigmoid gate, one shared expert, I = Ish = 8192; about 32 GB of
expert weights resident) at 16 tokens and 90 % intra-expert sparsity for routed and shared
experts.  ``--sweep`` (on by default on one GPU) adds the metric's grid on every bf16 shape:
Llama-4 at 1..256 tokens, OLMoE at 1..256, DeepSeek-V2-Lite at 1..64 with shared-expert sparsity
0 and 0.5, GPT-OSS-120B at 1..64 in top-K mode and in threshold mode; sparsity 0 / 0.5 / 0.9.
L2 is flushed (a 2x-L2 buffer is written, then another is read) before every timed step and the
token batch rotates through a pool of 32.  The line also reports the same steps replayed from
CUDA graphs (``graph``) and through the host-buffer call with its copies (``e2e``).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                  [--workload llama4|olmoe|dsv2l|gptoss] [--batch B] [--sparsity s]

Multi-GPU: one process per GPU (torchrun); each rank runs the layer on its own token batches
(independent decode streams, no data-path collective), so per-GPU work is fixed: weak scaling.
``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded sample of the
same workload (rank 0 only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer decode tokens/sec and HBM GB/s vs roofline at batch 1–256, sparsity 0/50/90%"
UNIT = "tokens/s"
# B200 HBM3e bandwidth as NVIDIA quotes it (8 TB/s, DGX).  The roofline fraction (`frac`) uses
# the measured copy bandwidth; `frac_spec` is the same figure against this nominal one.
HBM_SPEC_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DEFAULT_DENSE_MIN = -1  # the library's default: automatic path choice per call

# command-line names of the workload shapes
WORKLOADS = {"llama4": "llama4-maverick", "olmoe": "olmoe", "dsv2l": "dsv2-lite",
             "gptoss": "gpt-oss-120b", "tiny": "tiny-fp32"}

# The metric's grid: (shape, batches, [(selection, routed s, shared s)]).  Threshold rows carry
# the target sparsity the threshold is calibrated for.
SWEEP = [
    ("llama4-maverick", [1, 2, 4, 8, 16, 32, 64, 128, 256],
     [("topk", s, s) for s in (0.0, 0.5, 0.9)]),
    ("olmoe", [1, 4, 16, 64, 256], [("topk", s, None) for s in (0.0, 0.5, 0.9)]),
    ("dsv2-lite", [1, 2, 4, 8, 16, 32, 64],
     [("topk", s, sh) for sh in (0.0, 0.5) for s in (0.0, 0.5, 0.9)]),
    ("gpt-oss-120b", [1, 8, 32, 64],
     [("topk", s, None) for s in (0.0, 0.5, 0.9)] +
     [("threshold", s, None) for s in (0.5, 0.9)]),
]
CALIB_TOKENS = 1024  # threshold calibration tokens (seeded apart from the token stream)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="llama4")
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--sparsity", type=float, default=0.9)
    ap.add_argument("--sweep", dest="sweep", action="store_true", default=None)
    ap.add_argument("--no-sweep", dest="sweep", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target host time of the oracle sample")
    ap.add_argument("--crossover", action="store_true",
                    help="time the sparse kernels against the tensor-core path per batch size "
                         "(one GPU) and print the table instead of the benchmark line")
    ap.add_argument("--profile", action="store_true",
                    help="only make warm-up + steps layer calls (L2 flushed before each), for a "
                         "profiler to capture; prints one summary line")
    ap.add_argument("--experts", type=int, default=None,
                    help="routed experts of the layer (default: the workload's); fewer experts "
                         "keep the same kernels and per-item work with less memory resident")
    ap.add_argument("--dense-min", type=int, default=DEFAULT_DENSE_MIN,
                    help="path choice for --profile (see moe_set_dense_min_tokens)")
    ap.add_argument("--fused", dest="fused", action="store_true", default=False,
                    help="run the fused layer kernel instead of the chain of separate kernels "
                         "(see moe_set_fused)")
    ap.add_argument("--no-fused", dest="fused", action="store_false")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    NVML is polled about every millisecond from a background thread (read-only queries; ctypes
    releases the GIL, so the launch loop is not held up), which gives samples even when the
    timed region lasts only milliseconds.  Without NVML, nvidia-smi samples every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_id):
        self.dev = device_id  # "GPU-<uuid>" or an index
        self.proc = None
        self.path = None
        self.thread = None
        self.samples = []

    def _nvml_handle(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            if str(self.dev).startswith("GPU-"):
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID(str(self.dev))
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.dev))
        except Exception:
            return None, None

    def start(self):
        nv, h = self._nvml_handle()
        if h is not None:
            bits = {n: getattr(nv, "nvmlClocksEventReason" + c)
                    for n, c in zip(self.REASONS, ("HwSlowdown", "HwThermalSlowdown",
                                                   "SwThermalSlowdown", "SwPowerCap"))}
            self.stop_flag = threading.Event()

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, mx, [n for n, b in bits.items() if rs & b]))
                    except Exception:
                        break
                    time.sleep(0.001)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = self.samples
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                        "source": "nvml"}
            return {"sm_mhz": statistics.median(r[0] for r in rows),
                    "sm_max_mhz": max(r[1] for r in rows),
                    "reasons": sorted({n for r in rows for n in r[2]}),
                    "samples": len(rows), "source": "nvml"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and parts[1].isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"],
                    "source": "nvidia-smi"}
        reasons = sorted({n for r in rows for n, v in zip(self.REASONS, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(int(r[1]) for r in rows),
                "sm_max_mhz": max(int(r[2]) for r in rows), "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi"}


# ---------------------------------------------------------------------------------------------
def workload_config(shape, B, world, s):
    """The workload keys of `config`, the same in both arms (each arm adds how it ran)."""
    return {"workload": f"{shape.name}-shaped MoE layer", "hidden": shape.hidden,
            "experts": shape.n_routed, "top_k": shape.top_k, "inter": shape.inter,
            "shared": shape.n_shared, "batch_per_gpu": B, "global_batch": B * world,
            "sparsity": s, "selection": "top-K per (token, expert)"
            + (", the same sparsity for the shared experts" if shape.n_shared else "")}


def shape_of(name, experts=None):
    import synth
    shape = synth.SHAPES[WORKLOADS.get(name, name)]
    if experts:
        shape = shape.with_(name=f"{shape.name}-{experts}e", n_routed=experts,
                            top_k=min(shape.top_k, experts))
    return shape


def algorithmic_bytes(shape, dbg, B):
    """Bytes the method must read per stage for one call (each touched expert's gate block
    once, each kept row of the per-expert union once), from the call's kept lists."""
    import numpy as np
    elt, H = shape.elt, shape.hidden
    k, S = shape.top_k, shape.n_shared
    imax = max(shape.inter, shape.inter_shared if S else 0)
    idx = np.asarray(dbg["idx"][:B])
    routed = sorted(set(int(e) for e in idx.ravel()))
    row_of = {e: i for i, e in enumerate(routed)}
    union = np.zeros((len(routed) + S, imax + 1), bool)  # column imax absorbs the -1 padding
    for t in range(B):
        for j in range(k + S):
            u = row_of[int(idx[t][j])] if j < k else len(routed) + j - k
            union[u, dbg["lists"][t][j][: int(dbg["cnt"][t][j])]] = True
    rows = int(union[:, :imax].sum())
    gate = (len(routed) * shape.inter + S * shape.inter_shared) * H * elt
    pairs = B * (k + S)
    return {"router": shape.n_routed * H * elt + B * H * elt, "gate": gate,
            "select": pairs * imax * 4, "updown": rows * 2 * H * elt,
            "finalize": B * H * (8 + elt), "rows": rows}


def traffic_of(key):
    """DRAM bytes (read + write) of one launch from the committed ncu capture of that kernel,
    or None when there is none or the kernel's sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        ent = json.load(f).get(key)
    if not ent:
        return None
    h = hashlib.sha256()
    for name in ent["source_files"]:
        with open(os.path.join(ROOT, "sparse_expert_ffn_logits_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return ent["bytes"] if h.hexdigest()[:16] == ent["source_sha"] else None


def job_time_ms(local_ms, world, device):
    """The job's time: the largest of the ranks' device-timed totals (every rank calls this)."""
    if world == 1:
        return local_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, batch, steps, job_ms):
    """Tokens per second of the whole job: every rank processed `steps` batches of `batch`."""
    return world * batch * steps / (job_ms / 1e3)


def token_stream(rank, i):
    """Index of rank `rank`'s i-th token batch: ranks draw disjoint streams (i < 1000)."""
    return rank * 1000 + i


def make_flush(dev):
    """Writes a 2x-L2 buffer, then reads another one, so that the next timed step starts with
    an L2 that holds none of the layer's data and no dirty lines to write back."""
    import torch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones_like(flush_w)

    def flush():
        flush_w.zero_()
        flush_r.sum()
    return flush


def timed_calls(dl, batches, rule_r, rule_s, steps, warmup, flush, out):
    """Event-timed layer calls (ms each), the L2 flushed before each, batches rotating."""
    import torch
    for i in range(warmup):
        dl.forward(batches[i % len(batches)], rule_r, rule_s, out=out)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush()
        evs[i][0].record()
        dl.forward(batches[i % len(batches)], rule_r, rule_s, out=out)
        evs[i][1].record()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def calibrate_threshold(dl, s, chunk):
    """Threshold t for target sparsity s from the layer's own fp32 activations of the routed
    pairs of CALIB_TOKENS seeded calibration tokens: the scores |SiLU(g)| sorted ascending as
    S[0..N), t = S[m - 1] with m = floor(s N), so that the top N - m scores exceed it (the same
    order statistic as the tests' fp64 calibration; here the scores are the device's)."""
    import torch

    import synth
    shape = dl.shape
    xs = dl.tokens(CALIB_TOKENS, synth.calib_seed(shape))
    scores = []
    for c0 in range(0, CALIB_TOKENS, chunk):
        x = xs[c0:c0 + chunk].contiguous()
        n = x.shape[0]
        dl.forward(x, ("topk", 0.0), ("topk", 0.0))
        d = dl.debug_device(n)
        scores.append(d["act"][:, :shape.top_k, :shape.inter].abs().reshape(-1))
    allv = torch.cat(scores)
    m = int(s * allv.numel())
    if m == 0:
        return float("-inf")
    return float(torch.kthvalue(allv.cpu(), m).values)


def sweep_rows(dl, batches, rules, peak, flush, pool_n, token_stream_of, steps=20):
    """The metric's grid on one shape: per (batch, rule) the median layer time, tokens/s and
    the active-weight bytes over time against the HBM peak; the s = 0.9 / s = 0 speed-up per
    batch and shared-expert sparsity."""
    import torch

    import synth
    shape = dl.shape
    rows = []
    thresholds = {}
    for kind, s, s_sh in rules:
        if kind == "threshold" and s not in thresholds:
            thresholds[s] = calibrate_threshold(dl, s, max(batches))
    for B in batches:
        bx = [dl.tokens(B, synth.token_seed(shape, token_stream_of(i))) for i in range(pool_n)]
        out = torch.empty_like(bx[0])
        times = {}
        for kind, s, s_sh in rules:
            if kind == "threshold":
                r_r = ("threshold", thresholds[s])
                r_s = r_r if shape.n_shared else None
            else:
                r_r = ("topk", s)
                r_s = ("topk", s_sh) if shape.n_shared else None
            ms = statistics.median(timed_calls(dl, bx, r_r, r_s, steps, 3, flush, out))
            nbytes, nrep = 0.0, 2
            for i in range(nrep):
                dl.forward(bx[i], r_r, r_s, out=out)
                ab = algorithmic_bytes(shape, dl.debug(B), B)
                nbytes += (ab["router"] + ab["gate"] + ab["updown"]) / nrep
            gbs = nbytes / (ms / 1e3) / 1e9
            row = {"workload": shape.name, "batch": B, "selection": kind, "sparsity": s}
            if shape.n_shared:
                row["shared_sparsity"] = s_sh
            if kind == "threshold":
                row["threshold"] = thresholds[s]
            row.update({"us": round(ms * 1e3, 1), "tokens_per_s": round(B / (ms / 1e3), 1),
                        "tokens_per_expert": round(B * shape.top_k / shape.n_routed, 3),
                        "launches": dl.last_launches(),
                        "active_bytes": int(nbytes), "gbs": round(gbs, 1),
                        "frac": round(gbs / peak, 4), "frac_spec": round(gbs / HBM_SPEC_GBS, 4)})
            rows.append(row)
            times[(kind, s, s_sh)] = (ms, row)
        for (kind, s, s_sh), (ms, row) in times.items():
            if kind != "topk" or s != 0.9:
                continue
            # against sparsity 0 with the same shared sparsity (DeepSeek-V2-Lite's grid), or with
            # the shared experts dense too where the grid moves both together (Llama-4's)
            base = ("topk", 0.0, s_sh) if ("topk", 0.0, s_sh) in times else ("topk", 0.0, 0.0)
            if base in times:
                row["speedup_s0.9_vs_s0"] = round(times[base][0] / ms, 3)
        del bx, out
    return rows


def run_cuda(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import synth
    from sparse_expert_ffn_logits_b200 import (STAGES, moe_forward_host, moe_profile_stages,
                                               sparsity)
    from sparse_expert_ffn_logits_b200.workload import DeviceLayer

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    shape = shape_of(args.workload)
    B, s = args.batch, args.sparsity
    sweep_on = args.sweep if args.sweep is not None else (world == 1)
    plan = {name: (bs, rules) for name, bs, rules in SWEEP} if sweep_on else {}
    max_tokens = max([B] + (plan[shape.name][0] if shape.name in plan else []))
    rule = ("topk", s)
    rule_s = rule if shape.n_shared else None
    dl = DeviceLayer(shape, max_tokens=max_tokens, device=dev)
    dl.set_fused(args.fused)
    pool_n = 32

    def pool(nb):
        return [dl.tokens(nb, synth.token_seed(shape, token_stream(rank, i)))
                for i in range(pool_n)]

    xs = pool(B)
    out = torch.empty_like(xs[0])
    flush = make_flush(dev)

    # ---- the timed run (warm-up, barrier, K steps, barrier)
    for i in range(args.warmup):
        dl.forward(xs[i % pool_n], rule, rule_s, out=out)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    clocks = ClockSampler(f"GPU-{uuid}" if uuid and not uuid.startswith("GPU-") else
                          (uuid or str(local_rank)))
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        evs[i][0].record()
        dl.forward(xs[i % pool_n], rule, rule_s, out=out)
        evs[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    launches = dl.last_launches()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = job_time_ms(sum(step_ms), world, dev)
    value = job_throughput(world, B, args.steps, total_ms)

    # ---- per-stage durations (kernels launched back to back, events between them).  A call on
    # the fused layer kernel (3 launches) has router, layer and output cast: the layer's events
    # are the gate stage's.  The chain of separate kernels is timed too, for its breakdown.
    fused_call = launches == 3
    nprof = min(args.steps, 20)

    def stage_times(fused):
        dl.set_fused(fused)
        stage_evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)]
        for e in stage_evs:
            e.record()
        torch.cuda.synchronize()
        moe_profile_stages(dl.h, stage_evs)
        stage_ms = {n: [] for n in STAGES}
        for i in range(nprof):
            flush()
            dl.forward(xs[i % pool_n], rule, rule_s, out=out)
            torch.cuda.synchronize()
            for j, n in enumerate(STAGES):
                stage_ms[n].append(stage_evs[j].elapsed_time(stage_evs[j + 1]))
        moe_profile_stages(dl.h, None)
        dl.set_fused(args.fused)
        return {n: statistics.mean(v) for n, v in stage_ms.items()}

    stage_avg = stage_times(args.fused)
    chain_avg = stage_times(False) if fused_call else stage_avg
    abytes = {n: 0.0 for n in STAGES}
    nb = min(pool_n, nprof, 8)
    for i in range(nb):
        dl.forward(xs[i], rule, rule_s, out=out)
        ab = algorithmic_bytes(shape, dl.debug(B), B)
        for n in STAGES:
            abytes[n] += ab[n] / nb
    if fused_call:  # gate, selection and up/down are one kernel
        dom = "layer"
        dom_ms = stage_avg["gate"]
        dom_bytes = abytes["gate"] + abytes["updown"]
    else:
        dom = max(STAGES, key=lambda n: stage_avg[n])
        dom_ms = stage_avg[dom]
        dom_bytes = abytes[dom]
    peak, peak_kind = peaks()
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    layer_bytes = sum(abytes[n] for n in ("router", "gate", "updown"))
    traffic = traffic_of(f"{shape.name}:B{B}:s{s}:{dom}")
    layer_gbs = layer_bytes / (total_ms / args.steps / 1e3) / 1e9
    stage_names = (("router", "router"), ("gate", "layer"), ("finalize", "finalize")) \
        if fused_call else tuple((n, n) for n in STAGES)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peak,
                "peak_source": f"hbm copy, {peak_kind}", "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "frac_spec": round(achieved / HBM_SPEC_GBS, 4), "traffic": traffic,
                "algorithmic_bytes_per_launch": int(dom_bytes),
                "launch_us": round(dom_ms * 1e3, 2),
                "stages_us": {out_n: round(stage_avg[n] * 1e3, 2) for n, out_n in stage_names},
                "chain_stages_us": {n: round(v * 1e3, 2) for n, v in chain_avg.items()},
                "layer": {"algorithmic_bytes": int(layer_bytes), "gbs": round(layer_gbs, 1),
                          "frac": round(layer_gbs / peak, 4),
                          "frac_spec": round(layer_gbs / HBM_SPEC_GBS, 4)}}

    # ---- end to end through the host-buffer C call (pinned host memory, copies inside)
    xh = [x.cpu().pin_memory() for x in xs[:8]]
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    sr = sparsity(rule)
    ss = sparsity(rule) if shape.n_shared else None
    for i in range(args.warmup):
        moe_forward_host(dl.h, xh[i % 8], B, dl.router, dl.routed, dl.shared, sr, ss, oh)
    torch.cuda.synchronize()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        e2e_ev[i][0].record()
        moe_forward_host(dl.h, xh[i % 8], B, dl.router, dl.routed, dl.shared, sr, ss, oh)
        e2e_ev[i][1].record()
    torch.cuda.synchronize()
    e2e_ms = job_time_ms(sum(a.elapsed_time(b) for a, b in e2e_ev), world, dev)
    io_bytes = B * shape.hidden * shape.elt
    e2e = {"value": round(job_throughput(world, B, args.steps, e2e_ms), 1), "unit": UNIT,
           "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes,
           "api": "moe_forward_host"}

    # ---- the same steps replayed from CUDA graphs: one captured layer call per pooled batch
    # (the launches and their programmatic edges are recorded once, replayed per step)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        dl.forward(xs[0], rule, rule_s, out=out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for i in range(pool_n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            dl.forward(xs[i], rule, rule_s, out=out)
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % pool_n].replay()
    torch.cuda.synchronize()
    g_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        g_ev[i][0].record()
        graphs[i % pool_n].replay()
        g_ev[i][1].record()
    torch.cuda.synchronize()
    g_ms = job_time_ms(sum(a.elapsed_time(b) for a, b in g_ev), world, dev)
    graph = {"value": round(job_throughput(world, B, args.steps, g_ms), 1), "unit": UNIT,
             "ms_per_step": round(g_ms / args.steps, 5), "graphs": pool_n}
    del graphs

    # ---- sweep (rank 0, single GPU): the metric's grid on every bf16 shape
    sweep = []
    if sweep_on and rank == 0:
        for name, bs, rules in SWEEP:
            if name == shape.name:
                sdl = dl
            else:
                sdl = DeviceLayer(synth.SHAPES[name], max_tokens=max(bs), device=dev)
                sdl.set_fused(args.fused)
            try:
                sweep += sweep_rows(sdl, bs, rules, peak, flush, pool_n,
                                    lambda i: token_stream(rank, i))
            finally:
                if sdl is not dl:
                    sdl.close()
                    del sdl
                    torch.cuda.empty_cache()

    # ---- CPU baseline: the oracle, as it stands, on a bounded sample (rank 0, N = 1)
    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_baseline(shape, B, rule, args.cpu_seconds)

    dl.close()
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": shape.dtype, "data": "synthetic",
            "config": dict(workload_config(shape, B, world, s),
                           l2="flushed before every step: a 2x-L2 buffer written, then another "
                              "2x-L2 buffer read (clean lines, none of the layer's)",
                           token_pool=pool_n, parallelism=f"replicas x{world}"),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "graph": graph,
            "gpu_launches": launches * args.steps, "clocks": clock_info}
    if sweep:
        line["sweep"] = sweep
    return line


# ---------------------------------------------------------------------------------------------
class OracleSample:
    """Token batches of the benchmark's workload for the fp64 oracle, with their weights.

    Batches hold min(B, 8) tokens of the bench's token streams when the shape's routed weights
    exceed 4 GB (the Llama-4 shape: the oracle then holds a fixed set of 16 routed experts and
    draws only tokens routed among them, so that host memory stays bounded; the oracle's cost
    per token does not depend on which expert it routes to), else B tokens with every expert's
    weights drawn when first needed."""

    def __init__(self, shape, B, stream0=0):
        import oracle
        import synth
        self.shape, self.synth, self.oracle = shape, synth, oracle
        routed_bytes = shape.n_routed * 3 * shape.inter * shape.hidden * shape.elt
        self.limited = routed_bytes > (4 << 30)
        self.nb = min(B, 8) if self.limited else B
        self.router = synth.host_tensor(shape, "router")
        self.rl = oracle.Layer(shape, self.router, {}, [])
        self.shared = [(synth.host_tensor(shape, "sh_gate", j), synth.host_tensor(shape, "sh_up", j),
                        synth.host_tensor(shape, "sh_down", j)) for j in range(shape.n_shared)]
        self.cache = {}
        self.stream = stream0
        self.pending = []

    def _expert(self, e):
        s = self.synth
        if e not in self.cache:
            self.cache[e] = (s.host_tensor(self.shape, "gate", e), s.host_tensor(self.shape, "up", e),
                             s.host_tensor(self.shape, "down", e))
        return self.cache[e]

    def next(self):
        """(layer, x) of the next batch; drawing weights is not part of the oracle's time."""
        import numpy as np
        s = self.synth
        if not self.limited:
            x = s.host_tokens(self.shape, self.nb, s.token_seed(self.shape, self.stream))
            self.stream += 1
            _, idx, _ = self.rl.route(x)
            need = sorted(set(int(e) for e in idx.ravel()))
            return self.oracle.Layer(self.shape, self.router, {e: self._expert(e) for e in need},
                                     self.shared), x
        while len(self.pending) < self.nb:
            x = s.host_tokens(self.shape, 64, s.token_seed(self.shape, self.stream))
            self.stream += 1
            _, idx, _ = self.rl.route(x)
            for t in range(x.shape[0]):
                es = [int(e) for e in idx[t]]
                if len(self.cache) < 16:
                    for e in es:
                        self._expert(e)
                if all(e in self.cache for e in es):
                    self.pending.append(x[t])
        x = np.stack(self.pending[:self.nb])
        self.pending = self.pending[self.nb:]
        return self.oracle.Layer(self.shape, self.router, dict(self.cache), self.shared), x

    def describe(self):
        if self.limited:
            return (f"batches of {self.nb} tokens of the token streams routed among a fixed set "
                    f"of 16 routed experts (host memory bound)")
        return f"batches of {self.nb} tokens of the token streams"


def cpu_baseline(shape, B, rule, seconds):
    """Times the fp64 oracle (all host cores) on batches of the benchmark's token streams,
    batch after batch, until about `seconds` of oracle time has been spent."""
    rule_s = rule if shape.n_shared else None
    smp = OracleSample(shape, B)
    done_tok, spent, nb = 0, 0.0, 0
    while spent < seconds and nb < 4096:
        lay, x = smp.next()
        t0 = time.perf_counter()
        lay.forward(x, rule, rule_s)
        spent += time.perf_counter() - t0
        done_tok += x.shape[0]
        nb += 1
    return {"value": round(done_tok / spent, 3), "unit": UNIT, "cores": smp.oracle.threads(),
            "kind": "oracle",
            "sample": f"{nb} {smp.describe()}, whole layer in fp64, {spent:.1f} s of oracle time"}


def run_reference(args):
    """The benchmark's reference arm: the fp64 CPU oracle, timed on the host cores."""
    shape = shape_of(args.workload)
    B, rule = args.batch, ("topk", args.sparsity)
    rule_s = rule if shape.n_shared else None
    smp = OracleSample(shape, B)
    batches = [smp.next() for _ in range(4)]
    # tokens per step: sized so that the whole run stays within a few minutes
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup) * 4)
    lay0, x0 = batches[0]
    t0 = time.perf_counter()
    lay0.forward(x0[:1], rule, rule_s)
    one = time.perf_counter() - t0
    ntok = int(max(1, min(smp.nb, per_step / max(one, 1e-6))))
    for i in range(args.warmup):
        lay, x = batches[i % 4]
        lay.forward(x[:ntok], rule, rule_s)
    t0 = time.perf_counter()
    for i in range(args.steps):
        lay, x = batches[i % 4]
        lay.forward(x[:ntok], rule, rule_s)
    dt = time.perf_counter() - t0
    value = ntok * args.steps / dt
    sample = f"{ntok} tokens per step from {smp.describe()}, whole layer in fp64"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_config(shape, B, args.gpus, args.sparsity),
                           token_pool=4, parallelism="host cores"),
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT,
                             "cores": smp.oracle.threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_profile(args):
    """Warm-up + steps layer calls of one workload (L2 flushed before each) for a profiler."""
    import torch

    import synth
    from sparse_expert_ffn_logits_b200 import moe_set_dense_min_tokens
    from sparse_expert_ffn_logits_b200.workload import DeviceLayer
    shape = shape_of(args.workload, args.experts)
    B, rule = args.batch, ("topk", args.sparsity)
    rule_s = rule if shape.n_shared else None
    dl = DeviceLayer(shape, max_tokens=B)
    moe_set_dense_min_tokens(dl.h, args.dense_min)
    dl.set_fused(args.fused)
    flush = make_flush(torch.device("cuda", 0))
    xs = [dl.tokens(B, synth.token_seed(shape, i)) for i in range(4)]
    out = torch.empty_like(xs[0])
    ms = timed_calls(dl, xs, rule, rule_s, args.steps, args.warmup, flush, out)
    launches = dl.last_launches()
    # the algorithmic bytes of each token batch (call i used batch i % 4), per stage
    per_batch = []
    for x in xs:
        dl.forward(x, rule, rule_s, out=out)
        ab = algorithmic_bytes(shape, dl.debug(B), B)
        per_batch.append({k: int(v) for k, v in ab.items()})
    print(json.dumps({"profile": shape.name, "batch": B, "sparsity": args.sparsity,
                      "experts": shape.n_routed, "calls": args.warmup + args.steps,
                      "launches_per_call": launches,
                      "median_us": round(statistics.median(ms) * 1e3, 1),
                      "algorithmic_bytes_by_batch": per_batch}))
    dl.close()


def run_crossover(args):
    """Layer time per batch size with the dense tensor-core path off (every expert sparse) and
    forced on (every expert dense), L2 flushed before each call; prints one JSON line per
    (batch, sparsity) and a summary with the smallest batch at which the dense path wins."""
    import torch

    import synth
    from sparse_expert_ffn_logits_b200 import moe_set_dense_min_tokens
    from sparse_expert_ffn_logits_b200.workload import DeviceLayer
    shape = shape_of(args.workload)
    batches = [1, 2, 4, 8, 16, 32, 64, 128, 256]
    dl = DeviceLayer(shape, max_tokens=max(batches))
    flush = make_flush(torch.device("cuda", 0))
    rows = []
    for B in batches:
        xs = [dl.tokens(B, synth.token_seed(shape, 500 + i)) for i in range(8)]
        out = torch.empty_like(xs[0])
        for s in (0.0, 0.5, 0.9):
            rule = ("topk", s)
            rule_s = rule if shape.n_shared else None
            t = {}
            arms = [("sparse", 0), ("dense", 1), ("auto", DEFAULT_DENSE_MIN)]
            if shape.n_shared:
                # the shared experts (every token) on the tensor cores, routed experts sparse
                arms.append(("shared_dense", B))
            for name, dmin in arms:
                moe_set_dense_min_tokens(dl.h, dmin)
                t[name] = statistics.median(
                    timed_calls(dl, xs, rule, rule_s, args.steps, 3, flush, out)) * 1e3
            row = {"workload": shape.name, "batch": B, "sparsity": s,
                   "tokens_per_expert": round(B * shape.top_k / shape.n_routed, 3)}
            row.update({f"{name}_us": round(v, 1) for name, v in t.items()})
            row["faster"] = min((v, name) for name, v in t.items() if name != "auto")[1]
            rows.append(row)
            print(json.dumps(row), flush=True)
    dl.close()
    wins = [r["batch"] for r in rows if r["faster"] != "sparse"]
    print(json.dumps({"workload": shape.name, "crossover_batch": min(wins) if wins else None,
                      "rows": len(rows)}))


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if args.crossover:
        run_crossover(args)
        return 0
    if args.profile:
        run_profile(args)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_cuda(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
