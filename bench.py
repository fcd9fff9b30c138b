"""Benchmark of the gated delta rule library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill4k|prefill256k|varlen]
                    [--path auto|tensor|tensor_pair|tensor_single|tensor_split|simt]
                    [--no-decode] [--no-backward] [--no-front-end] [--no-gr]
                    [--no-cpu-baseline]

One step = one chunked prefill (gdn_chunk_fwd: L2-norm prologue, gate cumsum,
intra-chunk products, triangular solve, state carry, RMSNorm x sigmoid(g)
epilogue) over one batch of the workload (default: B=1, T=4096, 16 QK / 48
value heads, d=128, bf16).  The call gets a preallocated workspace, so small
batches may take the split layout (one kernel, after an asynchronous memset of
the workspace flags).  The JSON line also carries the decode step
(gdn_decode_step, 256 sequences x 64 steps, in place) and the backward of the
model-shape prefill (gdn_chunk_bwd, T=4096) and the conv + SiLU front end
(alone, ahead of the prefill, and fused into a 4-token decode) and the
Gated Residual read / write over an FP8 state as separate objects with their
own timing, roofline and clocks; so are the T=262,144 prefill and the packed
24-sequence prefill (``prefill_configs``).  The line ends with ``summary``:
every headline figure (prefill fractions of the roofline time, decode state
bandwidth fraction, ...) in one short object.

Multi-GPU (torchrun, one process per GPU): every rank runs its own
independent batch (weak scaling; sequences and heads are independent, so the
data path has no collective).  Timing is on the device with CUDA events, the
reported time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle (the only other program that
computes this operation here) on a bounded sample of the same workload, on
rank 0 only.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "GDN prefill tokens/s (48 heads, d=128) and decode state GB/s; % of roofline"
H_QK, H_V, D = 16, 48, 128
CHUNK = 64
L2_BYTES = 126 * 2 ** 20


def flops_per_token(Hqk=H_QK, Hv=H_V, d=D, C=CHUNK):
    """Counted MMA FLOPs per token at the canonical chunk of 64:
    per value head 6 d^2 + 6 C d + C^2 / 3, per QK head 4 C d."""
    return Hv * (6 * d * d + 6 * C * d + C * C / 3.0) + Hqk * 4 * C * d


def prefill_bytes(T, n_seq, epilogue=True, init_state=True, in_bytes=2, Hqk=H_QK, Hv=H_V, d=D):
    """Compulsory HBM bytes of one prefill: every input read once, y and the
    final state written once."""
    per_tok = 2 * Hqk * d * in_bytes + Hv * d * in_bytes + Hv * d * in_bytes + Hv * 8
    if epilogue:
        per_tok += Hv * d * in_bytes
    state = n_seq * Hv * d * d * 4
    return per_tok * T + state * (2 if init_state else 1) + (d * 4 if epilogue else 0)


def bwd_flops_per_token(Hqk=H_QK, Hv=H_V, d=D, C=CHUNK, epilogue=True):
    """Counted contraction FLOPs per token of the chunkwise backward at the
    canonical chunk of 64 (forward recomputation included): per value head
    (18 or 16) d^2 + 24 C d + 13 C^2 / 3, per QK head 4 C d."""
    dd = 18 if epilogue else 16
    return Hv * (dd * d * d + 24 * C * d + 13.0 * C * C / 3.0) + Hqk * 4 * C * d


def bwd_bytes(T, n_seq, epilogue=True, in_bytes=2, Hqk=H_QK, Hv=H_V, d=D):
    """Compulsory HBM bytes of one backward: inputs and dy read once (the
    input dtype), fp32 gradients written once, dS_T read and dS0 written."""
    per_tok_in = 2 * Hqk * d * in_bytes + (3 if epilogue else 2) * Hv * d * in_bytes + Hv * 8
    per_tok_out = 2 * Hqk * d * 4 + (2 if epilogue else 1) * Hv * d * 4 + Hv * 8
    return (per_tok_in + per_tok_out) * T + 2 * n_seq * Hv * d * d * 4 + (d * 4 if epilogue else 0)


def decode_bytes(N, Hqk=H_QK, Hv=H_V, d=D, in_bytes=2):
    """Compulsory HBM bytes of one decode step: the state read and written
    once, plus q/k/v, gates and y."""
    return N * (2 * Hv * d * d * 4 + 2 * Hqk * d * in_bytes + 2 * Hv * d * in_bytes + Hv * 8)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


def code_text(src):
    """The code of a C/C++/CUDA source with its comments removed (string and
    character literals kept as written), trailing blanks stripped and empty
    lines dropped: two sources with the same code text differ only in
    comments and blank lines."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln)


def code_sha(path):
    """sha256[:16] of a source file's code text (comments do not count)."""
    with open(path, encoding="utf-8") as f:
        return hashlib.sha256(code_text(f.read()).encode()).hexdigest()[:16]


def kernel_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the code of
    the kernel source it was taken on is unchanged (comments may differ);
    else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(kernel_key)
        if not d:
            return None
        src = os.path.join(ROOT, d["source"])
        if "code_sha" in d:
            same = code_sha(src) == d["code_sha"]
        else:
            same = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] == d["source_sha"]
        return float(d["bytes_per_launch"]) if same else None
    except Exception:
        return None


class NvmlClockSampler:
    """SM clocks and clock-event reasons read through NVML every ~1 ms from
    start() to stop() (the timed region and its warm-up), for the GPU that
    cuda:`index` is (matched by PCI bus id).  Reads only; changes nothing."""
    NAMES = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
             ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
             ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
             ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap")]

    def __init__(self, index):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(index)
        bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.samples = []
        self.stop_flag = threading.Event()

    def _poll(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.001)

    def start(self):
        self.t = threading.Thread(target=self._poll, daemon=True)
        self.t.start()

    def stop(self):
        self.stop_flag.set()
        self.t.join(timeout=2)
        nv = self.nv
        if not self.samples:
            return None
        mx = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        reasons = set()
        for _, rs in self.samples:
            for nm, const in self.NAMES:
                if rs & getattr(nv, const):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median([sm for sm, _ in self.samples]), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


def clock_sampler(index):
    """NVML sampler (fine-grained), else nvidia-smi."""
    try:
        return NvmlClockSampler(index)
    except Exception:
        return ClockSampler(index)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during a timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x, world, device="cuda"):
    """Max of a host scalar over all ranks (host plumbing, not data path)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms_max):
    """Units all ranks processed divided by the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def rank_seed(name, rank):
    """Each rank draws an independent batch of the same recipe."""
    from gated_deltanet_scan_chunked_b200 import inputs
    return inputs.SEEDS[name] + 100 * rank


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def timed_steps(fn, steps, warmup, world, flush=None, stream=None):
    """Warm up, then time exactly `steps` calls with CUDA events on `stream`
    (flush between steps outside the events).  Returns per-step ms list."""
    stream = stream or torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    barrier(world)
    times = []
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    barrier(world)
    for a, b in ev:
        times.append(a.elapsed_time(b))
    return times


def cpu_baseline(w, target_s=12.0):
    """The fp64 oracle, as it stands, on a bounded prefix of the workload's
    first sequence (all heads), sized for about `target_s` seconds."""
    import oracle
    cores = oracle.max_threads()

    def run(T):
        sub = _prefix(w, T)
        t0 = time.perf_counter()
        oracle.recurrence(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                          g=sub["g"], norm_w=sub["norm_w"], initial_state=sub["s0"])
        return time.perf_counter() - t0

    T_cal = 64
    dt = run(T_cal)
    T_s = int(max(64, min(w.total_T, T_cal * target_s / max(dt, 1e-6))))
    T_s = min(T_s, int(w.cu_seqlens[1].item()))
    # a sequence shorter than the target is run repeatedly (the oracle as it
    # stands; each run is the same work) until about target_s has passed
    reps, total = 0, 0.0
    while reps == 0 or total < 0.5 * target_s:
        total += run(T_s)
        reps += 1
    return {"value": reps * T_s / total, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "first %d tokens of sequence 0, all %d value heads, fp64, OpenMP over "
                      "value heads, %d run(s) (%.1f s)" % (T_s, w.v.shape[1], reps, total)}


def _prefix(w, T):
    cpu = lambda x: None if x is None else x[:T].to("cpu", torch.float32)
    return dict(q=cpu(w.q), k=cpu(w.k), v=cpu(w.v), log_alpha=cpu(w.log_alpha),
                beta=cpu(w.beta), g=cpu(w.g),
                norm_w=None if w.norm_w is None else w.norm_w.to("cpu", torch.float32),
                s0=None if w.initial_state is None else w.initial_state[:1].to("cpu", torch.float32))


def make_workload(name, rank, device="cuda"):
    from gated_deltanet_scan_chunked_b200 import inputs
    w = inputs.workload(name, device=device)
    if rank:
        # an independent batch per rank: same recipe, another seed
        seed = rank_seed(name, rank)
        lengths = w.meta["lengths"]
        w = inputs.make_prefill(lengths, H_QK, H_V, D, D, seed=seed,
                                s0_std=0.01 if w.initial_state is not None else 0.0,
                                device=device)
    return w


def config_of(args, world, n_seq, T):
    """The workload's config object, printed the same way by both arms."""
    return {"workload": args.workload, "global_batch": world * n_seq, "seq_len": T,
            "heads": "16 QK / 48 value", "d": D,
            "parallelism": "replicas%d" % world if world > 1 else "single",
            "l2": "flushed between steps (256 MB write outside the events)"}


def prefill_object(name, args, world, rank, local, peaks, steps, warmup):
    """One prefill workload timed in a region of its own (the same call and
    roofline as the headline), for the configs that are not the headline."""
    from gated_deltanet_scan_chunked_b200 import gdn, gdn_chunk_fwd
    w = make_workload(name, rank)
    T, n_seq = w.total_T, w.n_seq
    has_s0 = w.initial_state is not None
    y = torch.empty_like(w.v)
    fs = torch.empty((n_seq, H_V, D, D), dtype=torch.float32, device="cuda")
    ws_bytes = gdn.workspace_size(n_seq, H_V, D, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda") if ws_bytes > 0 else None
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    clk = clock_sampler(local)
    clk.start()
    times = timed_steps(lambda: gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, g=w.g,
                                              norm_w=w.norm_w, initial_state=w.initial_state,
                                              cu_seqlens=w.cu_seqlens, y=y, final_state=fs,
                                              workspace=ws),
                        steps, warmup, world, flush=lambda: flush_buf.zero_())
    clk_r = clk.stop()
    err = gdn.gdn_check_device_error()
    if err != gdn.GDN_OK:
        raise RuntimeError("device error in %s: %s" % (name, gdn.status_string(err)))
    ms = max_over_ranks(statistics.mean(times), world)
    nbytes = prefill_bytes(T, n_seq, epilogue=w.g is not None, init_state=has_s0)
    nflops = flops_per_token() * T
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = nflops / (peaks["bf16_tflops"] * 1e12)
    out = {"workload": "%s: %d sequence(s), %d tokens, 16 QK / 48 value heads, d=128, bf16, "
                       "epilogue, fp32 initial states" % (name, n_seq, T),
           "ms_per_step": ms, "steps": steps, "tokens_per_s": world * T / (ms * 1e-3),
           "roofline": {"bound": "hbm" if t_hbm >= t_tc else "tensor",
                        "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac_of_roofline_time": max(t_hbm, t_tc) / (ms * 1e-3),
                        "roofline_time_us": max(t_hbm, t_tc) * 1e6, "algorithmic_bytes": nbytes,
                        "counted_flops": nflops,
                        "tensor_frac": nflops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"]},
           "clocks": clk_r,
           "gpu_launches_per_step": 2 if (ws is not None and n_seq * H_V > 64) else 1}
    del w, y, fs, ws, flush_buf
    torch.cuda.empty_cache()
    return out


def run_reference(args, world, rank):
    """The oracle arm: rank 0 only, no process group, no GPU kernels of ours."""
    if rank != 0:
        return
    # the same recipe; generated on the GPU when there is one (as the other
    # arm does), else on the host (a different draw of the same distributions)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if dev == "cuda":
        torch.cuda.set_device(0)
    w = make_workload(args.workload, 0, device=dev)
    times = []
    base = None
    per_step = min(args.ref_seconds, 150.0 / (args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        b = cpu_baseline(w, target_s=per_step)
        if i >= args.warmup:
            times.append(b)
        base = b
    vals = [b["value"] for b in times] or [base["value"]]
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            # a whole step of the workload at the sampled rate
            "ms_per_step": 1e3 * w.total_T / v if v > 0 else None,
            "ms_per_step_basis": "extrapolated from the bounded sample",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(args, world, w.n_seq, w.total_T),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": base["cores"],
                             "kind": "oracle", "sample": base["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    from gated_deltanet_scan_chunked_b200 import gdn, gdn_chunk_fwd, gdn_decode_step, inputs
    gdn.load()
    peaks = load_peaks()
    w = make_workload(args.workload, rank)
    T, n_seq = w.total_T, w.n_seq
    has_s0 = w.initial_state is not None
    stream = torch.cuda.current_stream()
    y = torch.empty_like(w.v)
    fs = torch.empty((n_seq, H_V, D, D), dtype=torch.float32, device="cuda")
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    # caller-owned workspace for the small-batch split layout (allocated once)
    ws = None
    ws_bytes = gdn.workspace_size(n_seq, H_V, D, D) if args.path in gdn._WS_PATHS else 0
    if ws_bytes > 0:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")

    def step():
        gdn_chunk_fwd(w.q, w.k, w.v, w.log_alpha, w.beta, g=w.g, norm_w=w.norm_w,
                      initial_state=w.initial_state, cu_seqlens=w.cu_seqlens, y=y,
                      final_state=fs, path=args.path, workspace=ws)

    def flush():
        flush_buf.zero_()

    clocks = clock_sampler(local)
    clocks.start()
    times = timed_steps(step, args.steps, args.warmup, world, flush=flush, stream=stream)
    clk = clocks.stop()
    # the same steps back to back without the flush (warm L2: the step's
    # ~190 MB of traffic exceed the 126 MB L2, so most of it still comes
    # from HBM); reported beside the headline, which is the flushed figure
    warm_times = timed_steps(step, args.steps, 1, world, stream=stream)
    ms_warm = max_over_ranks(statistics.mean(warm_times), world)
    warm = {"ms_per_step": ms_warm, "value": whole_job_rate(T, world, ms_warm),
            "unit": "tokens/s", "l2": "not flushed between steps"}
    err = gdn.gdn_check_device_error()
    if err != gdn.GDN_OK:
        raise RuntimeError("device error: %s" % gdn.status_string(err))
    ms = statistics.mean(times)
    ms_max = max_over_ranks(ms, world)
    value = whole_job_rate(T, world, ms_max)

    # roofline of the dominant (only) kernel of the step
    nbytes = prefill_bytes(T, n_seq, epilogue=w.g is not None, init_state=has_s0)
    nflops = flops_per_token() * T
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = nflops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        achieved, peak, unit = nbytes / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = nflops / (ms * 1e-3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    # the kernel that runs: the scan layout for at most 64 (sequence, head)
    # items of at least one chunk, the one-CTA layout otherwise
    items = n_seq * H_V
    if args.path == "simt":
        kernel_key = "prefill_simt"
    elif args.path in ("auto", "tensor", "tensor_split") and items <= 64 and T >= 64:
        kernel_key = "prefill_scan"
    else:
        kernel_key = "prefill_tc"
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": kernel_traffic(kernel_key),
                "peak_source": peaks["source"], "roofline_time_us": max(t_hbm, t_tc) * 1e6,
                "frac_of_roofline_time": max(t_hbm, t_tc) / (ms * 1e-3),
                "algorithmic_bytes": nbytes, "counted_flops": nflops,
                "achieved_tflops": nflops / (ms * 1e-3) / 1e12,
                "tensor_frac": nflops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}

    # end to end through the public call with host buffers: every step copies
    # its inputs from pinned host memory and reads its results back.  Steps are
    # pipelined (double-buffered device inputs and outputs, three streams):
    # step i+1's host->device copy runs while step i's kernel runs and step
    # i-1's results are read back.
    e2e = None
    if not args.no_e2e:
        host = {}
        for nm in ("q", "k", "v", "log_alpha", "beta", "g", "norm_w", "initial_state",
                   "cu_seqlens"):
            x = getattr(w, nm)
            host[nm] = None if x is None else x.to("cpu").pin_memory()
        dev = [{nm: (None if x is None else torch.empty_like(x, device="cuda"))
                for nm, x in host.items()} for _ in range(2)]
        yb = [y, torch.empty_like(y)]
        fsb = [fs, torch.empty_like(fs)]
        y_h = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
        fs_h = [torch.empty(fs.shape, dtype=fs.dtype).pin_memory() for _ in range(2)]
        h2d = sum(x.numel() * x.element_size() for x in host.values() if x is not None)
        d2h = y_h[0].numel() * y_h[0].element_size() + fs_h[0].numel() * fs_h[0].element_size()
        cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
        kdone = [None, None]  # kernel of the step that last used buffer b
        read = [None, None]   # read-back of the step that last used buffer b

        def e2e_step(i):
            bi = i % 2
            d = dev[bi]
            with torch.cuda.stream(cin):
                if kdone[bi] is not None:
                    cin.wait_event(kdone[bi])  # step i-2's kernel has read dev[bi]
                for nm, x in host.items():
                    if x is not None:
                        d[nm].copy_(x, non_blocking=True)
                hdone = torch.cuda.Event()
                hdone.record(cin)
            stream.wait_event(hdone)
            if read[bi] is not None:
                stream.wait_event(read[bi])  # step i-2's results have been read back
            gdn_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], g=d["g"],
                          norm_w=d["norm_w"], initial_state=d["initial_state"],
                          cu_seqlens=d["cu_seqlens"], y=yb[bi], final_state=fsb[bi],
                          path=args.path, workspace=ws)
            kd = torch.cuda.Event()
            kd.record(stream)
            kdone[bi] = kd
            with torch.cuda.stream(cout):
                cout.wait_event(kd)
                y_h[bi].copy_(yb[bi], non_blocking=True)
                fs_h[bi].copy_(fsb[bi], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(cout)
            read[bi] = ev

        e_steps, e_warm = max(3, args.steps // 2), 2
        for i in range(e_warm):
            e2e_step(i)
        stream.wait_stream(cout)
        barrier(world)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        cin.wait_event(t0)
        for i in range(e_steps):
            e2e_step(e_warm + i)
        stream.wait_stream(cout)  # the last step's results are read back
        t1.record(stream)
        barrier(world)
        ems = max_over_ranks(t0.elapsed_time(t1) / e_steps, world)
        e2e = {"value": world * T / (ems * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "steps": e_steps,
               "pipelining": "double-buffered: step i+1's host-to-device copy overlaps "
                             "step i's kernel and step i-1's device-to-host read"}
        del dev, host, yb, fsb

    # the other prefill configs (T=262,144 and the 24-sequence packed batch),
    # each in a region of its own, when the headline is the T=4096 workload
    others = None
    launches_others = 0
    if args.workload == "prefill4k" and not args.no_configs:
        del flush_buf
        others = {}
        for nm in ("prefill256k", "varlen"):
            others[nm] = prefill_object(nm, args, world, rank, local, peaks, steps=5, warmup=3)
            launches_others += 5 * others[nm]["gpu_launches_per_step"]
        flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

    # the decode step, timed on its own (256 sequences x 64 steps, in place)
    decode = None
    launches_decode = 0
    if not args.no_decode:
        del flush_buf
        d = inputs.make_decode(device="cuda", seed=inputs.SEEDS["decode"] + 100 * rank)
        state0 = d.state.clone()
        state = d.state
        yd = torch.empty((d.q.shape[1], H_V, D), dtype=torch.bfloat16, device="cuda")
        nsteps = d.q.shape[0]

        def dstep():
            for t in range(nsteps):
                gdn_decode_step(d.q[t], d.k[t], d.v[t], d.log_alpha[t], d.beta[t], state, y=yd)

        def dreset():
            state.copy_(state0)

        dclk = clock_sampler(local)
        dclk.start()
        dt = timed_steps(dstep, max(3, args.steps // 2), 2, world, flush=dreset, stream=stream)
        dclk_r = dclk.stop()
        dms = max_over_ranks(statistics.mean(dt), world) / nsteps
        N = d.q.shape[1]
        sbytes = 2 * N * H_V * D * D * 4
        dbytes = decode_bytes(N)
        decode = {"workload": "decode: 256 sequences x 64 single-token steps, state 48x128x128 "
                              "fp32 per sequence, in place",
                  "us_per_step": dms * 1e3,
                  "state_GBps": world * sbytes / (dms * 1e-3) / 1e9,
                  "tokens_per_s": world * N / (dms * 1e-3),
                  "roofline": {"bound": "hbm",
                               "achieved": dbytes / (dms * 1e-3) / 1e9,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": dbytes / (dms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                               "traffic": kernel_traffic("decode"),
                               "algorithmic_bytes": dbytes},
                  "state_frac_of_8TBps_nominal": sbytes / (dms * 1e-3) / 8e12,
                  "clocks": dclk_r}
        launches_decode = nsteps * max(3, args.steps // 2)

        # multi-token decode: the same 64 tokens as 16 launches of 4 tokens
        # per sequence (speculative verification), state read/written once
        # per launch, in place
        from gated_deltanet_scan_chunked_b200 import gdn_decode_multi
        TS = 4
        tr = lambda x: x.transpose(0, 1).contiguous()
        groups = [dict(q=tr(d.q[c:c + TS]), k=tr(d.k[c:c + TS]), v=tr(d.v[c:c + TS]),
                       la=tr(d.log_alpha[c:c + TS]), b=tr(d.beta[c:c + TS]))
                  for c in range(0, nsteps, TS)]
        ym = torch.empty((N, TS, H_V, D), dtype=torch.bfloat16, device="cuda")

        def mstep():
            for gr in groups:
                gdn_decode_multi(gr["q"], gr["k"], gr["v"], gr["la"], gr["b"], state, y=ym)

        mclk = clock_sampler(local)
        mclk.start()
        mt = timed_steps(mstep, max(3, args.steps // 2), 2, world, flush=dreset, stream=stream)
        mclk_r = mclk.stop()
        mms = max_over_ranks(statistics.mean(mt), world) / len(groups)  # per launch
        mbytes = N * 2 * H_V * D * D * 4 + TS * (decode_bytes(N) - N * 2 * H_V * D * D * 4)
        decode["multi_token"] = {
            "workload": "256 sequences x 4 tokens per launch (16 launches = the same 64 tokens), "
                        "in place",
            "us_per_launch": mms * 1e3,
            "tokens_per_s": world * N * TS / (mms * 1e-3),
            "state_GBps": world * sbytes / (mms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": mbytes / (mms * 1e-3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": mbytes / (mms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": mbytes},
            "clocks": mclk_r}
        launches_decode += len(groups) * max(3, args.steps // 2)

    # the backward (gdn_chunk_bwd) on the model-shape sequence, timed on its own
    backward = None
    launches_bwd = 0
    if not args.no_backward:
        from gated_deltanet_scan_chunked_b200 import gdn_chunk_bwd
        wb = inputs.workload("prefill4k", device="cuda")
        dy, dsT = inputs.make_cotangents(wb, seed=inputs.SEEDS["prefill4k"] + 100 * rank)
        Tb = wb.q.shape[0]
        bws = torch.empty(gdn.bwd_workspace_size(1, Tb, H_QK, H_V, D, D), dtype=torch.uint8,
                          device="cuda")
        bflush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

        def bstep():
            gdn_chunk_bwd(wb.q, wb.k, wb.v, wb.log_alpha, wb.beta, dy, g=wb.g, norm_w=wb.norm_w,
                          d_final_state=dsT, workspace=bws)

        bclk = clock_sampler(local)
        bclk.start()
        bsteps = max(3, args.steps // 4)
        bt = timed_steps(bstep, bsteps, 3, world, flush=lambda: bflush.zero_(), stream=stream)
        bclk_r = bclk.stop()
        err = gdn.gdn_check_device_error()
        if err != gdn.GDN_OK:
            raise RuntimeError("device error in the backward: %s" % gdn.status_string(err))
        bms = max_over_ranks(statistics.mean(bt), world)
        bb = bwd_bytes(Tb, 1)
        bfl = bwd_flops_per_token() * Tb
        alu_peak = 148 * 128 * 2 * 1.965  # fp32 FMA lanes x 2 FLOP x max SM GHz, in GFLOP/s
        backward = {
            "workload": "backward of prefill4k: T=4096, 16 QK / 48 value heads, d=128, bf16 "
                        "inputs and dy, epilogue, dS_T given; fp32 gradients",
            "ms_per_step": bms, "tokens_per_s": world * Tb / (bms * 1e-3),
            "workspace_bytes": bws.numel(),
            "roofline": {"bound": "hbm", "achieved": bb / (bms * 1e-3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": bb / (bms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": bb, "traffic": kernel_traffic("bwd_chunk_b"),
                         "traffic_kernel": "bwd_chunk_b (the largest share of the call)"},
            "tensor": {"achieved_tflops": bfl / (bms * 1e-3) / 1e12,
                       "peak_tflops": peaks["bf16_tflops"],
                       "frac": bfl / (bms * 1e-3) / 1e12 / (peaks["bf16_tflops"])},
            "alu_roofline": {"bound": "alu", "achieved": bfl / (bms * 1e-3) / 1e9,
                             "peak": alu_peak, "unit": "GFLOP/s",
                             "frac": bfl / (bms * 1e-3) / 1e9 / alu_peak,
                             "note": "fp32 CUDA-core arithmetic, the limiter of this kernel set"},
            "clocks": bclk_r}
        launches_bwd = bsteps * (10 if wb.g is not None else 9)
        del bws, bflush

    # the front end (causal conv of kernel 4 + SiLU): alone, in front of the
    # model-shape prefill, and fused into the multi-token decode
    front = None
    launches_front = 0
    if not args.no_front_end:
        from gated_deltanet_scan_chunked_b200 import (gdn_chunk_fwd_conv, gdn_conv_frontend,
                                                      gdn_decode_conv)
        wf = inputs.workload("prefill4k", device="cuda")
        Tf = wf.q.shape[0]
        cw, cst = inputs.make_conv_params(1, H_QK, H_V, D, D, seed=inputs.SEEDS["prefill4k"],
                                          device="cuda")
        cso = torch.empty_like(cst)
        outs = (torch.empty_like(wf.q), torch.empty_like(wf.k), torch.empty_like(wf.v))
        fflush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        fclk = clock_sampler(local)
        fclk.start()
        fsteps = max(3, args.steps // 2)
        # the conv kernel takes less time than the Python call that launches
        # it: time it as a CUDA graph replay so that host overhead stays out
        conv_call = lambda: gdn_conv_frontend(wf.q, wf.k, wf.v, cw, cst, conv_state_out=cso,
                                              out=outs)
        for _ in range(3):
            conv_call()
        torch.cuda.synchronize()
        cgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cgraph):
            conv_call()
        ct = timed_steps(cgraph.replay, fsteps, 3, world, flush=lambda: fflush.zero_(),
                         stream=stream)
        cms = max_over_ranks(statistics.mean(ct), world)
        cbytes = 2 * Tf * (2 * H_QK * D + H_V * D) * 2 + 2 * H_V * 3 * (3 * D) * 4
        cws = torch.empty(gdn.conv_workspace_size(1, Tf, H_QK, H_V, D, D), dtype=torch.uint8,
                          device="cuda")
        yf = torch.empty_like(wf.v)
        fsf = torch.empty((1, H_V, D, D), dtype=torch.float32, device="cuda")
        pt = timed_steps(lambda: gdn_chunk_fwd_conv(wf.q, wf.k, wf.v, cw, wf.log_alpha, wf.beta,
                                                    conv_state_in=cst, conv_state_out=cso,
                                                    g=wf.g, norm_w=wf.norm_w, y=yf,
                                                    final_state=fsf, workspace=cws),
                         fsteps, 3, world, flush=lambda: fflush.zero_(), stream=stream)
        pms = max_over_ranks(statistics.mean(pt), world)
        del cws, fflush, cgraph
        # decode with the front end fused: 256 sequences x 4 tokens per launch, in place
        dd = inputs.make_decode(steps=4, device="cuda", seed=inputs.SEEDS["decode"] + 7)
        Nd = dd.q.shape[1]
        tr = lambda x: x.transpose(0, 1).contiguous()
        dq, dk_, dv_, dla, db = tr(dd.q), tr(dd.k), tr(dd.v), tr(dd.log_alpha), tr(dd.beta)
        dcw, dcst = inputs.make_conv_params(Nd, H_QK, H_V, D, D, seed=3, device="cuda")
        dstate0 = dd.state.clone()
        ydc = torch.empty((Nd, 4, H_V, D), dtype=torch.bfloat16, device="cuda")
        dct = timed_steps(lambda: gdn_decode_conv(dq, dk_, dv_, dcw, dla, db, dd.state, dcst,
                                                  y=ydc),
                          fsteps, 3, world, flush=lambda: dd.state.copy_(dstate0), stream=stream)
        fclk_r = fclk.stop()
        err = gdn.gdn_check_device_error()
        if err != gdn.GDN_OK:
            raise RuntimeError("device error in the front end: %s" % gdn.status_string(err))
        dcms = max_over_ranks(statistics.mean(dct), world)
        dcbytes = (Nd * 2 * H_V * D * D * 4 + 4 * (decode_bytes(Nd) - Nd * 2 * H_V * D * D * 4)
                   + 2 * Nd * H_V * 3 * 3 * D * 4)
        front = {
            "workload": "front end at the model shape: q, k, v of T=4096 (16 QK / 48 value "
                        "heads, d=128, bf16), conv state carried; decode: 256 sequences x 4 "
                        "tokens per launch with the front end fused, in place",
            "conv_us": cms * 1e3, "conv_timing": "CUDA graph replay of one call",
            "conv_roofline": {"bound": "hbm", "achieved": cbytes / (cms * 1e-3) / 1e9,
                              "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": cbytes / (cms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "algorithmic_bytes": cbytes, "traffic": kernel_traffic("conv")},
            "prefill_with_front_end_ms": pms,
            "prefill_with_front_end_tokens_per_s": world * Tf / (pms * 1e-3),
            "decode_conv_us_per_launch": dcms * 1e3,
            "decode_conv_roofline": {"bound": "hbm", "achieved": dcbytes / (dcms * 1e-3) / 1e9,
                                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": dcbytes / (dcms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                     "algorithmic_bytes": dcbytes},
            "clocks": fclk_r}
        launches_front = fsteps * (1 + 2 + 1)

    # Gated Residual read / write around a block, FP8 state, model shape
    # (n_r = 4 branches of d = 2560, router rank 320), 4096 tokens
    grd = None
    launches_gr = 0
    if not args.no_gr:
        from gated_deltanet_scan_chunked_b200 import gdn_gr_read, gdn_gr_write
        Tg, NR, DG, RK = 4096, 4, 2560, 320
        g = inputs.make_gr(Tg, NR, DG, RK, seed=inputs.SEEDS["prefill4k"] + 100 * rank,
                           device="cuda")
        gws = torch.empty(gdn.gr_read_workspace_size(Tg, NR, DG, RK), dtype=torch.uint8,
                          device="cuda")
        xg = torch.empty((Tg, DG), dtype=torch.bfloat16, device="cuda")
        sg = torch.empty((Tg, NR), dtype=torch.float32, device="cuda")
        codes0, scales0 = g["codes"].clone(), g["scales"].clone()
        gflush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        gclk = clock_sampler(local)
        gclk.start()
        gsteps = max(3, args.steps // 2)
        # both calls are shorter than the Python that launches them: time them
        # as CUDA graph replays so that host overhead stays out

        def graph_of(fn):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            gg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gg):
                fn()
            return gg

        rgraph = graph_of(lambda: gdn_gr_read(g["codes"], g["scales"], g["gamma"], g["W_d"],
                                              g["W_u"], g["W_w"], x=xg, s=sg, workspace=gws))
        rt = timed_steps(rgraph.replay, gsteps, 3, world, flush=lambda: gflush.zero_(),
                         stream=stream)

        def wreset():
            g["codes"].copy_(codes0)
            g["scales"].copy_(scales0)
            gflush.zero_()

        wgraph = graph_of(lambda: gdn_gr_write(g["codes"], g["scales"], g["y"], g["s"]))
        wt = timed_steps(wgraph.replay, gsteps, 3, world, flush=wreset, stream=stream)
        gclk_r = gclk.stop()
        err = gdn.gdn_check_device_error()
        if err != gdn.GDN_OK:
            raise RuntimeError("device error in the gated residual: %s" % gdn.status_string(err))
        rms_ = max_over_ranks(statistics.mean(rt), world)
        wms_ = max_over_ranks(statistics.mean(wt), world)
        nd = NR * DG
        rbytes = Tg * (nd + NR * 4 + DG * 2 + NR * 4) + (2 * RK * nd + NR * nd) * 2 + nd * 4
        rflops = 2.0 * 2 * RK * nd * Tg + 2.0 * NR * nd * Tg
        wbytes = Tg * (2 * nd + 2 * NR * 4 + DG * 2 + NR * 4)
        grd = {
            "workload": "Gated Residual, 4096 tokens x 4 branches x d=2560, E4M3 state with a "
                        "scale per row, router rank 320 (bf16 weights)",
            "timing": "CUDA graph replay of one call",
            "read_us": rms_ * 1e3,
            "read_roofline": {"bound": "tensor", "achieved": rflops / (rms_ * 1e-3) / 1e12,
                              "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": rflops / (rms_ * 1e-3) / 1e12 / peaks["bf16_tflops"],
                              "algorithmic_flops": rflops, "algorithmic_bytes": rbytes,
                              "hbm_frac": rbytes / (rms_ * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "write_us": wms_ * 1e3,
            "write_roofline": {"bound": "hbm", "achieved": wbytes / (wms_ * 1e-3) / 1e9,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": wbytes / (wms_ * 1e-3) / 1e9 / peaks["hbm_gbs"],
                               "algorithmic_bytes": wbytes},
            "clocks": gclk_r}
        launches_gr = gsteps * (6 + 1)  # read: norm, GEMM, split-K sum, router, GEMM, gate; write
        del gws, gflush, rgraph, wgraph

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, target_s=args.ref_seconds)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": config_of(args, world, n_seq, T),
                "path": args.path, "workspace_bytes": ws_bytes,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": args.steps, "clocks": clk,
                "warm_l2": warm, "gpu_launches_warm_l2_region": args.steps,
                "backward": backward, "gpu_launches_backward_region": launches_bwd,
                "front_end": front, "gpu_launches_front_end_region": launches_front,
                "gated_residual": grd, "gpu_launches_gated_residual_region": launches_gr,
                "prefill_configs": others, "gpu_launches_prefill_configs_region": launches_others,
                "decode": decode, "gpu_launches_decode_region": launches_decode}
        # last: a compact summary of every figure the targets name, so that a
        # reader of the line's tail has them all
        summ = {"prefill4k_ms": ms_max, "prefill4k_frac": roofline["frac_of_roofline_time"]}
        for nm, o in (others or {}).items():
            summ[nm + "_ms"] = o["ms_per_step"]
            summ[nm + "_frac"] = o["roofline"]["frac_of_roofline_time"]
        if backward:
            summ["backward_ms"] = backward["ms_per_step"]
        if front:
            summ["front_end_prefill_ms"] = front["prefill_with_front_end_ms"]
            summ["conv_frac"] = front["conv_roofline"]["frac"]
        if grd:
            summ["gr_read_us"] = grd["read_us"]
            summ["gr_write_frac"] = grd["write_roofline"]["frac"]
        if decode:
            summ["decode_multi_frac"] = decode["multi_token"]["roofline"]["frac"]
            summ["decode_us_per_step"] = decode["us_per_step"]
            summ["decode_frac"] = decode["roofline"]["frac"]
        line["summary"] = summ
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill4k",
                    choices=["prefill4k", "prefill256k", "varlen"])
    ap.add_argument("--path", default="auto",
                    choices=["auto", "tensor", "simt", "tensor_pair", "tensor_single",
                             "tensor_split"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the T=262,144 and packed-batch prefill objects")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-front-end", action="store_true")
    ap.add_argument("--no-gr", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
