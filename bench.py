"""Benchmark of the fine-grained-scaled FP8 GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step runs every GEMM of the workload once on inputs already resident in
HBM.  The default workload ("all") is the five benchmark configurations in one
step: decode (M=64, N=2112, K=7168), prefill (M=4096 with (N,K) in
{(24576,1536), (7168,16384), (4096,7168)}), contiguous-grouped MoE, masked-
grouped MoE and the small-M decode sweep, 20 GEMMs.  ``value`` is the prefill
throughput (FLOPs of the three prefill GEMMs / their summed device time), the
headline; every GEMM is also reported in ``per_shape`` with the fraction of
its own roofline (tensor for prefill and contiguous, HBM for decode and
masked).  The single-configuration workloads (decode, prefill, contiguous,
masked, decode_sweep, quantize) are for profiling.  Every GEMM keeps several
copies of its operands, together larger than twice the L2 cache, and step s
uses copy s mod copies, so no launch finds its operands in L2.  Each launch is
timed with CUDA events on its launch stream; a short GPU spin before the start
event absorbs the host's launch latency.

N > 1 (under torchrun): every rank runs the same workload on its own GPU
(independent replicas, no collective on the data path; weak scaling); the
time is the max over ranks and ``value`` counts the FLOPs of all ranks.

``--impl reference`` times the CPU oracle (plain C, FP64) on the host cores on
a bounded sample of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "FP8 TFLOPS per shape (device-timed) and % of B200 FP8 tensor / HBM roofline"
UNIT = "TFLOPS"

WORKLOADS = {
    "prefill": {"kind": "normal", "cfg": 1, "M": [4096], "shapes": [(24576, 1536), (7168, 16384), (4096, 7168)],
                "desc": "prefill normal FP8 GEMM, M=4096, (N,K) in {(24576,1536),(7168,16384),(4096,7168)}"},
    "decode": {"kind": "normal", "cfg": 0, "M": [64], "shapes": [(2112, 7168)],
               "desc": "decode normal FP8 GEMM, M=64, N=2112, K=7168"},
    "contiguous": {"kind": "contiguous", "cfg": 2, "G": 8, "shapes": [(4096, 7168), (7168, 2048)],
                   "desc": "contiguous-grouped MoE FP8 GEMM, 8 experts x U[1024,8192] rows (128-aligned), "
                           "(N,K) in {(4096,7168),(7168,2048)}"},
    "masked": {"kind": "masked", "cfg": 3, "G": 32, "M_max": 256, "shapes": [(4096, 7168), (7168, 2048)],
               "desc": "masked-grouped MoE decode FP8 GEMM, 32 experts, M_max=256, masked_m ~ U[0,256], "
                       "(N,K) in {(4096,7168),(7168,2048)}"},
    "decode_sweep": {"kind": "normal", "cfg": 4, "M": [64, 128],
                     "shapes": [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168),
                                (7168, 2048)],
                     "desc": "small-M decode sweep, M in {64,128} x 6 (N,K)"},
    "all": {"kind": "all", "parts": ["decode", "prefill", "contiguous", "masked", "decode_sweep"],
            "headline": "prefill",
            "desc": "the five configurations in one step: decode M=64 N=2112 K=7168; prefill M=4096 (N,K) in "
                    "{(24576,1536),(7168,16384),(4096,7168)}; contiguous-grouped 8 experts (N,K) in "
                    "{(4096,7168),(7168,2048)}; masked-grouped 32 experts M_max=256 (N,K) in "
                    "{(4096,7168),(7168,2048)}; decode sweep M in {64,128} x 6 (N,K); value = prefill TFLOPS"},
    "quantize": {"kind": "quantize", "shapes": [(4096, 7168, "fp32"), (4096, 7168, "bf16"), (64, 7168, "bf16")],
                 "desc": "activation quantiser (1x128 blocks -> E4M3 + MN-major FP32 scales), "
                         "(M,K,dtype) in {(4096,7168,fp32),(4096,7168,bf16),(64,7168,bf16)}"},
}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0          # nominal dense ratio 4.5 / 2.25 PFLOP/s
FP8_SPEC_TFLOPS = 4500.0     # B200 dense FP8 (E4M3) tensor peak, spec
HBM_SPEC_GBS = 8000.0        # B200 HBM3e bandwidth, spec
L2_BYTES = 126 << 20
MAX_COPIES = 32
SPIN_CYCLES = 100_000        # ~50 us at 1.965 GHz: longer than one launch's host latency


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ cases --

class Case:
    """One GEMM call of a workload: device inputs, its launcher, and its
    algorithmic FLOPs and HBM bytes."""

    def __init__(self, name, flops, hbm_bytes, run, host=None, copies=1):
        self.name = name
        self.flops = flops
        self.hbm_bytes = hbm_bytes
        self.run = run            # run(i): one launch on operand copy i % copies
        self.host = host or {}
        self.plan = None          # launch plan (fg.query_plan)
        self.copies = copies
        self.config = None        # workload (configuration) the GEMM belongs to
        self.decode_sized = False  # few rows of A: also timed back to back


def n_copies(footprint_bytes):
    """Operand copies whose total exceeds twice the L2 cache."""
    return int(min(MAX_COPIES, max(1, -(-2 * L2_BYTES // max(1, footprint_bytes)))))


def operand_copies(fg, x, D, n, extra=()):
    """n operand sets for one GEMM (set 0 uses the originals): A, B, sfb, D and
    the named extra tensors are cloned, sfa is laid out again from x.sfa."""
    sets = []
    for i in range(n):
        t = {"A": x.A, "B": x.B, "sfb": x.sfb, "D": D, **{k: getattr(x, k) for k in extra}}
        if i > 0:
            t = {k: v.clone() for k, v in t.items()}
        t["sfa"] = fg.get_col_major_tma_aligned_tensor(x.sfa)
        sets.append(t)
    return sets


def ceil_div(a, b):
    return (a + b - 1) // b


def build_cases(fg, synth, wl, device):
    cases = []
    kind = wl["kind"]
    if kind == "normal":
        si = 0
        for M in wl["M"]:
            for (N, K) in wl["shapes"]:
                x = synth.normal_inputs(M, N, K, seed=synth.seed_for(wl["cfg"], si), device=device)
                si += 1
                D = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                KB = K // 128
                flops = 2.0 * M * N * K
                hbm = M * K + N * K + M * KB * 4 + ceil_div(N, 128) * KB * 4 + 2 * M * N
                sets = operand_copies(fg, x, D, n_copies(hbm))

                def run(i, sets=sets):
                    t = sets[i % len(sets)]
                    fg.fp8_gemm_nt(t["A"], t["sfa"], t["B"], t["sfb"], D=t["D"])

                c = Case(f"M{M}_N{N}_K{K}", flops, hbm, run, host={"x": x, "D": D}, copies=len(sets))
                c.plan = fg.query_plan("normal", M, N, K)
                c.decode_sized = M <= 256
                cases.append(c)
    elif kind == "contiguous":
        for si, (N, K) in enumerate(wl["shapes"]):
            x = synth.contiguous_inputs(wl["G"], N, K, seed=synth.seed_for(wl["cfg"], si), device=device)
            D = torch.empty((x.M_tot, N), dtype=torch.bfloat16, device=device)
            real = sum(x.counts)
            KB = K // 128
            used = sum(1 for c in x.counts if c > 0)
            flops = 2.0 * real * N * K
            hbm = real * K + used * N * K + real * KB * 4 + used * ceil_div(N, 128) * KB * 4 + 2 * real * N \
                + 4 * x.M_tot
            sets = operand_copies(fg, x, D, n_copies(hbm), extra=("m_indices",))

            def run(i, sets=sets):
                t = sets[i % len(sets)]
                fg.m_grouped_fp8_gemm_nt_contiguous(t["A"], t["sfa"], t["B"], t["sfb"], t["m_indices"], D=t["D"])

            c = Case(f"contig_G{wl['G']}_Mtot{x.M_tot}_N{N}_K{K}", flops, hbm, run, host={"x": x, "D": D},
                     copies=len(sets))
            c.plan = fg.query_plan("contiguous", x.M_tot, N, K, wl["G"])
            cases.append(c)
    elif kind == "quantize":
        for si, (M, K, dt) in enumerate(wl["shapes"]):
            g = torch.Generator(device=device)
            g.manual_seed(synth.seed_for(5, si))
            x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
            if dt == "bf16":
                x = x.to(torch.bfloat16)
            hbm = M * K * (x.element_size() + 1) + M * (K // 128) * 4
            sets = [x] + [x.clone() for _ in range(n_copies(hbm) - 1)]

            def run(i, sets=sets):
                fg.quantize_fp8_activations(sets[i % len(sets)])

            cases.append(Case(f"quant_M{M}_K{K}_{dt}", 0.0, hbm, run, host={"xq": x}, copies=len(sets)))
    elif kind == "masked":
        for si, (N, K) in enumerate(wl["shapes"]):
            x = synth.masked_inputs(wl["G"], wl["M_max"], N, K, seed=synth.seed_for(wl["cfg"], si), device=device)
            D = torch.empty((x.G, x.M_max, N), dtype=torch.bfloat16, device=device)
            mm = [min(max(int(v), 0), x.M_max) for v in x.masked_m.cpu().tolist()]
            real = sum(mm)
            used = sum(1 for v in mm if v > 0)
            KB = K // 128
            flops = 2.0 * real * N * K
            hbm = real * K + used * N * K + real * KB * 4 + used * ceil_div(N, 128) * KB * 4 + 2 * real * N + 4 * x.G
            sets = operand_copies(fg, x, D, n_copies(hbm), extra=("masked_m",))

            def run(i, sets=sets):
                t = sets[i % len(sets)]
                fg.m_grouped_fp8_gemm_nt_masked(t["A"], t["sfa"], t["B"], t["sfb"], t["masked_m"], expected_m=128,
                                                D=t["D"])

            c = Case(f"masked_G{x.G}_Mmax{x.M_max}_N{N}_K{K}", flops, hbm, run,
                     host={"x": x, "D": D, "masked": mm}, copies=len(sets))
            c.plan = fg.query_plan("masked", x.M_max, N, K, x.G, 128)
            cases.append(c)
    elif kind == "all":
        for part in wl["parts"]:
            for c in build_cases(fg, synth, WORKLOADS[part], device):
                c.config = part
                cases.append(c)
        return cases
    for c in cases:
        c.config = c.config or next(k for k, v in WORKLOADS.items() if v is wl)
    return cases


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """SM clock, power and clock-event reasons of this GPU, sampled during the
    timed region: through NVML every 5 ms (so even a region of a few tens of
    milliseconds gets a dozen samples), else through ``nvidia-smi -lms 100``.
    Reading only; nothing here changes a GPU setting."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown"}
    SMI_FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, period_s=0.005):
        self.period = period_s
        self.rows = []            # (sm_mhz, max_mhz, power_w, reason bits)
        self.proc = None
        self.thread = None
        self.nvml = None
        self.handle = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid).replace("GPU-", "")
        except Exception:
            self.uuid = None
        try:
            import pynvml
            pynvml.nvmlInit()
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if self.uuid and self.uuid in u:
                    self.handle = h
            if self.handle is None and pynvml.nvmlDeviceGetCount() == 1:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.nvml = pynvml if self.handle is not None else None
        except Exception:
            self.nvml = None

    def _nvml_loop(self):
        nv, h = self.nvml, self.handle
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop:
            try:
                self.rows.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), float(mx),
                                  nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons_fn(h))))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        import threading
        self._stop = False
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def _smi_rows(self):
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        bits = {5: 0x8, 6: 0x40, 7: 0x20, 8: 0x4}
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9 or (self.uuid and self.uuid not in parts[0]):
                continue
            try:
                r = sum(b for i, b in bits.items() if parts[i].lower() == "active")
                self.rows.append((float(parts[1]), float(parts[2]), float(parts[3]), r))
            except ValueError:
                continue

    def stop(self):
        source = "nvml (5 ms)" if self.nvml is not None else "nvidia-smi (100 ms)"
        if self.thread is not None:
            self._stop = True
            self.thread.join()
        elif self.proc is not None:
            self._smi_rows()
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0, "source": source}
        sm = [r[0] for r in self.rows]
        mx = max(r[1] for r in self.rows)
        reasons = sorted({name for r in self.rows for bit, name in self.REASONS.items() if r[3] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(self.rows), "power_w_max": round(max(r[2] for r in self.rows), 1), "source": source}


# ------------------------------------------------------------- oracle leg --

def oracle_sample(cases, budget_s, rng_seed=0):
    """Times the CPU oracle on whole rows of each case (all N columns, full K)
    until about budget_s seconds are spent.  Returns (flops, seconds, threads,
    description)."""
    import oracle
    threads = oracle.num_threads()
    rng = np.random.default_rng(rng_seed)
    flops = 0.0
    secs = 0.0
    done = {}
    t_start = time.perf_counter()
    i = 0
    while True:
        c = cases[i % len(cases)]
        i += 1
        x = c.host["x"]
        kind = type(x).__name__
        if "np" not in c.host:
            c.host["np"] = {k: getattr(x, k).cpu().numpy() for k in ("A", "sfa", "B", "sfb")}
            if kind == "ContiguousInputs":
                c.host["np"]["mi"] = x.m_indices.cpu().numpy()
            if kind == "MaskedInputs":
                c.host["np"]["mm"] = x.masked_m.cpu().numpy()
        h = c.host["np"]
        if kind == "NormalInputs":
            r = int(rng.integers(0, x.M))
            t0 = time.perf_counter()
            oracle.gemm_nt(h["A"], h["sfa"], h["B"], h["sfb"], rows=[r])
            dt = time.perf_counter() - t0
            f = 2.0 * x.N * x.K
        elif kind == "ContiguousInputs":
            real = np.nonzero(h["mi"] >= 0)[0]
            r = int(rng.choice(real))
            t0 = time.perf_counter()
            oracle.m_grouped_contiguous(h["A"], h["sfa"], h["B"], h["sfb"], h["mi"], rows=[r])
            dt = time.perf_counter() - t0
            f = 2.0 * x.N * x.K
        else:
            lim = np.minimum(np.maximum(h["mm"], 0), x.M_max)
            flat = [g * x.M_max + rr for g in range(x.G) for rr in range(lim[g])]
            r = int(rng.choice(flat))
            t0 = time.perf_counter()
            oracle.m_grouped_masked(h["A"], h["sfa"], h["B"], h["sfb"], h["mm"], rows=[r])
            dt = time.perf_counter() - t0
            f = 2.0 * x.N * x.K
        flops += f
        secs += dt
        done[c.name] = done.get(c.name, 0) + 1
        if time.perf_counter() - t_start >= budget_s and i >= len(cases):
            break
    desc = "rows of D computed by the oracle (all N columns, full K): " + ", ".join(
        f"{n}: {k} rows" for n, k in done.items())
    return flops, secs, threads, desc


# ------------------------------------------------------------------- main --

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="all")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chain", action="store_true", help="skip the back-to-back decode timing (profiling)")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0)
    ap.add_argument("--case-index", type=int, default=None,
                    help="time only this GEMM of the workload (profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, wl)

    import fp8_fine_grained_tma_b200 as fg
    import synth

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist

    cases = build_cases(fg, synth, wl, device)
    if args.case_index is not None:
        cases = [cases[args.case_index]]
    stream = torch.cuda.current_stream(device)

    def one_step(s, events=None):
        for ci, c in enumerate(cases):
            torch.cuda._sleep(SPIN_CYCLES)    # the GPU idles here while the host enqueues the launch
            if events is not None:
                events[ci][0].record(stream)
            c.run(s)
            if events is not None:
                events[ci][1].record(stream)

    for s in range(args.warmup):
        one_step(s)
    torch.cuda.synchronize()
    code, detail = fg.get_last_device_status()
    if code != 0:
        raise RuntimeError(f"device status {code} ({detail:#x}) after warm-up")

    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in cases]
           for _ in range(args.steps)]
    clocks = ClockSampler(device)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.start()
    if clocks.nvml is None:
        time.sleep(0.3)                 # nvidia-smi needs a moment before its first sample
    for s in range(args.steps):
        one_step(args.warmup + s, evs[s])
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    clk = clocks.stop()
    per_case_ms = [sum(evs[s][ci][0].elapsed_time(evs[s][ci][1]) for s in range(args.steps))
                   for ci in range(len(cases))]

    # Decode-sized GEMMs (M <= 256) also run as a decode step runs its layers: launches
    # back to back on the stream, each on the next operand copy (the copies
    # total more than twice L2), so programmatic dependent launch overlaps each
    # kernel's set-up with the previous one's tail.  Per-launch time = chain
    # time / launches.  Reported beside the isolated time; the headline does
    # not use it.
    chain_us = {}
    for ci, c in enumerate(cases):
        if args.no_chain or not c.decode_sized:
            continue
        n = max(8, c.copies)
        for i in range(n):
            c.run(i)
        reps = 20
        tot = 0.0
        for r in range(reps):
            torch.cuda._sleep(SPIN_CYCLES)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(n):
                c.run(i)
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1) * 1e3 / n
        chain_us[ci] = max_over_ranks(tot / reps, pg, device)
    total_ms = sum(per_case_ms)
    code, detail = fg.get_last_device_status()
    if code != 0:
        raise RuntimeError(f"device status {code} ({detail:#x}) after the timed steps")

    # The headline: the configuration the metric is quoted on (prefill for the
    # default workload), FLOPs of its GEMMs over their summed device time.
    head_name = wl.get("headline")
    head = [i for i, c in enumerate(cases) if head_name is None or c.config == head_name]
    head_cases = [cases[i] for i in head]
    head_ms = sum(per_case_ms[i] for i in head)
    flops_step = sum(c.flops for c in head_cases)
    bytes_step = sum(c.hbm_bytes for c in head_cases)
    head_ms = max_over_ranks(head_ms, pg, device)
    total_ms = max_over_ranks(total_ms, pg, device)
    value = job_throughput(flops_step, world, args.steps, head_ms)
    unit = UNIT
    if flops_step == 0:   # a bandwidth-bound workload (the quantiser): GB/s
        value = world * bytes_step * args.steps / (head_ms * 1e-3) / 1e9
        unit = "GB/s"

    e2e = None
    if not args.no_e2e and wl["kind"] != "quantize":
        e2e = run_e2e(fg, head_cases, args, device, stream, pg, world)

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return 0

    peaks, peak_src = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    fp8_peak_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP8_OVER_BF16
    ridge = (fp8_peak * 1e12) / (peaks["hbm_gbs"] * 1e9)
    per_shape = []
    for ci, c in enumerate(cases):
        us = per_case_ms[ci] * 1e3 / args.steps
        tf = c.flops / (us * 1e-6) / 1e12
        gbs = c.hbm_bytes / (us * 1e-6) / 1e9
        bound = "tensor" if c.flops / max(1.0, c.hbm_bytes) > ridge else "hbm"
        row = {"config": c.config, "case": c.name, "plan": c.plan, "us": round(us, 3), "tflops": round(tf, 1),
               "hbm_gbs": round(gbs, 1), "bound": bound,
               "frac": round(tf / fp8_peak if bound == "tensor" else gbs / peaks["hbm_gbs"], 4),
               "frac_fp8_peak": round(tf / fp8_peak, 4), "frac_fp8_spec": round(tf / FP8_SPEC_TFLOPS, 4),
               "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "frac_hbm_spec": round(gbs / HBM_SPEC_GBS, 4)}
        if ci in chain_us:
            cu = chain_us[ci]
            row["us_chain"] = round(cu, 3)
            row["hbm_gbs_chain"] = round(c.hbm_bytes / (cu * 1e-6) / 1e9, 1)
            row["frac_hbm_chain"] = round(c.hbm_bytes / (cu * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)
        per_shape.append(row)
    per_config = []
    for name in dict.fromkeys(c.config for c in cases):
        idx = [i for i, c in enumerate(cases) if c.config == name]
        ms = sum(per_case_ms[i] for i in idx) / args.steps
        fl = sum(cases[i].flops for i in idx)
        by = sum(cases[i].hbm_bytes for i in idx)
        tf = fl / (ms * 1e-3) / 1e12
        gbs = by / (ms * 1e-3) / 1e9
        bound = "tensor" if fl / max(1.0, by) > ridge else "hbm"
        per_config.append({"config": name, "gemms": len(idx), "us": round(ms * 1e3, 2), "tflops": round(tf, 1),
                           "hbm_gbs": round(gbs, 1), "bound": bound,
                           "frac": round(tf / fp8_peak if bound == "tensor" else gbs / peaks["hbm_gbs"], 4),
                           "frac_fp8_spec": round(tf / FP8_SPEC_TFLOPS, 4)})
    achieved_tf = flops_step / (head_ms / args.steps * 1e-3) / 1e12
    achieved_gbs = bytes_step / (head_ms / args.steps * 1e-3) / 1e9
    tensor_bound = flops_step / max(1.0, bytes_step) > ridge
    traffic = read_traffic(head_name or args.workload)
    if tensor_bound:
        roof = {"bound": "tensor", "achieved": round(achieved_tf, 1), "peak": round(fp8_peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved_tf / fp8_peak, 4), "traffic": traffic,
                "peak_source": f"{peak_src}: 2 x bf16_tflops (burst) = nominal fp8/bf16 ratio x measured cuBLAS bf16",
                "frac_of_sustained_peak": round(achieved_tf / fp8_peak_sus, 4),
                "frac_of_fp8_spec": round(achieved_tf / FP8_SPEC_TFLOPS, 4), "kernel": "fg8_gemm_kernel"}
    else:
        roof = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": round(peaks["hbm_gbs"], 1),
                "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": f"{peak_src}: hbm_gbs (copy bandwidth)",
                "frac_of_hbm_spec": round(achieved_gbs / HBM_SPEC_GBS, 4)}

    cpu = None
    if not args.no_cpu_baseline and world == 1 and wl["kind"] == "quantize":
        import oracle
        c0 = cases[0]
        xs = c0.host["xq"][:256].float().cpu().numpy()
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < args.cpu_budget_s:
            oracle.quantize_blocks(xs, 1)
            reps += 1
        secs = time.perf_counter() - t0
        cpu = {"value": round(reps * xs.shape[0] * xs.shape[1] * 5 / secs / 1e9, 4), "unit": "GB/s", "cores": 1,
               "kind": "oracle", "sample": f"{reps} x quantize_blocks on 256 rows of {c0.name}",
               "seconds": round(secs, 2)}
    elif not args.no_cpu_baseline and world == 1:
        f, secs, thr, desc = oracle_sample(head_cases, args.cpu_budget_s)
        cpu = {"value": round(f / secs / 1e12, 6), "unit": UNIT, "cores": thr, "kind": "oracle", "sample": desc,
               "seconds": round(secs, 2)}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3 (fp32 accumulate, bf16 out)",
        "data": "synthetic (seeded N(0,1), block-quantised to E4M3)",
        "config": {"workload": wl["desc"], "cases": [c.name for c in cases],
                   "value": (f"{head_name} TFLOPS: FLOPs of its {len(head_cases)} GEMMs / their summed device time; "
                             "ms_per_step = device time of all GEMMs of the step") if head_name else
                            "FLOPs (bytes) of all GEMMs / their summed device time",
                   "l2": "inputs larger than L2: each GEMM rotates over operand copies totalling > 2 x 126 MB "
                         "(copies per GEMM: " + ", ".join(str(c.copies) for c in cases) + "); only GEMM launches "
                         "are timed (CUDA events around each launch, a GPU spin before each start event)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "per_shape": per_shape, "per_config": per_config, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": len(cases) * args.steps, "clocks": clk, "impl": "ours",
    }
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()
    return 0


def run_e2e(fg, cases, args, device, stream, pg, world):
    """Same metric end to end through the public API: every step copies the
    inputs from pinned host memory, lays out sfa with the library's transform
    kernel, runs the GEMM and copies D back to pinned host memory.  As in a
    serving pipeline, consecutive steps overlap on three streams (host-to-device
    copies, compute, device-to-host copies) over two sets of device buffers;
    every byte of every step still crosses PCIe inside the timed region."""
    NSETS = 2
    hosts = []
    h2d = d2h = 0
    for c in cases:
        x = c.host["x"]
        h = {k: getattr(x, k).cpu().pin_memory() for k in ("A", "sfa", "B", "sfb")}
        extra = None
        if hasattr(x, "m_indices"):
            h["mi"] = x.m_indices.cpu().pin_memory()
            extra = "contig"
        if hasattr(x, "masked_m"):
            h["mm"] = x.masked_m.cpu().pin_memory()
            extra = "masked"
        D = c.host["D"]
        devs = [{k: torch.empty_like(h[k], device=device) for k in h} for _ in range(NSETS)]
        Ds = [D] + [torch.empty_like(D) for _ in range(NSETS - 1)]
        out = torch.empty(D.shape, dtype=D.dtype).pin_memory()
        hosts.append((h, devs, Ds, out, extra))
        h2d += sum(t.numel() * t.element_size() for t in h.values())
        d2h += out.numel() * out.element_size()

    s_in = torch.cuda.Stream(device)
    s_cmp = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    # free[j]: set j's inputs and D may be overwritten (its GEMMs and D copies are done)
    free = [torch.cuda.Event() for _ in range(NSETS)]
    for e in free:
        e.record(stream)

    def step(i):
        j = i % NSETS
        loaded = torch.cuda.Event()
        computed = torch.cuda.Event()
        with torch.cuda.stream(s_in):
            s_in.wait_event(free[j])
            for (h, devs, Ds, out, extra) in hosts:
                for k in h:
                    devs[j][k].copy_(h[k], non_blocking=True)
            loaded.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(loaded)
            for c, (h, devs, Ds, out, extra) in zip(cases, hosts):
                dev = devs[j]
                sfa = fg.get_col_major_tma_aligned_tensor(dev["sfa"])
                if extra == "contig":
                    fg.m_grouped_fp8_gemm_nt_contiguous(dev["A"], sfa, dev["B"], dev["sfb"], dev["mi"], D=Ds[j])
                elif extra == "masked":
                    fg.m_grouped_fp8_gemm_nt_masked(dev["A"], sfa, dev["B"], dev["sfb"], dev["mm"], expected_m=128,
                                                   D=Ds[j])
                else:
                    fg.fp8_gemm_nt(dev["A"], sfa, dev["B"], dev["sfb"], D=Ds[j])
            computed.record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed)
            for (h, devs, Ds, out, extra) in hosts:
                out.copy_(Ds[j], non_blocking=True)
            free[j] = torch.cuda.Event()
            free[j].record(s_out)

    steps = max(3, min(args.steps, 20))
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for st in (s_in, s_cmp, s_out):
        st.wait_event(e0)
    for i in range(steps):
        step(3 + i)
    for st in (s_in, s_cmp, s_out):
        stream.wait_stream(st)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), pg, device)
    flops = sum(c.flops for c in cases) * steps * world
    return {"value": round(flops / (ms * 1e-3) / 1e12, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": round(ms / steps, 3),
            "pipeline": "copies in, compute and copies out of consecutive steps overlap on three streams"}


def max_over_ranks(ms, pg, device):
    """The slowest rank's time: every rank takes part, whatever its own value."""
    if pg is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank_step, world, steps, total_ms):
    """Whole-job TFLOPS: the work of all ranks (independent replicas, weak
    scaling) over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (total_ms * 1e-3) / 1e12


def read_traffic(workload):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on the current source of that kernel; else None."""
    import hashlib
    import re
    summ = os.path.join(ROOT, "profiles", f"ncu_traffic_{workload}.txt")
    if not os.path.exists(summ):
        return None
    vals = {}
    for line in open(summ):
        if line.startswith("#") or ":" not in line:
            continue
        k, v = line.split(":", 1)
        vals[k.strip()] = v.strip()
    m = re.search(r"\((csrc/[\w.]+)\)", vals.get("kernel", ""))
    if not m:
        return None
    src = os.path.join(ROOT, "fp8_fine_grained_tma_b200", m.group(1))
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if vals.get("kernel_source_sha256_16") != h:
        return None
    try:
        return float(vals["dram_bytes_per_launch_mean"])
    except (KeyError, ValueError):
        return None


def run_reference(args, wl):
    """The CPU oracle as the reference arm: each step times a bounded sample of
    the workload on the host cores."""
    import oracle
    import synth

    if wl["kind"] == "all":
        # The headline value is the prefill configuration's: time the oracle on it.
        wl = WORKLOADS[wl["headline"]]
    if wl["kind"] == "quantize":
        # The oracle's block quantiser on 256-row samples of each shape.
        g = np.random.default_rng(5)
        samples = [g.standard_normal((256, K)).astype(np.float32) for (_, K, _) in wl["shapes"]]
        per_step = max(0.02, 120.0 / (args.steps + args.warmup))
        for _ in range(args.warmup):
            oracle.quantize_blocks(samples[0], 1)
        nbytes = secs = 0.0
        for _ in range(args.steps):
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < per_step:
                for xs in samples:
                    oracle.quantize_blocks(xs, 1)
                    nbytes += xs.size * 5
            secs += time.perf_counter() - t0
        value = nbytes / secs / 1e9
        line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded N(0,1))", "config": {"workload": wl["desc"]}, "impl": "reference",
                "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                                 "sample": "256-row samples of each shape"},
                "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    # Inputs on the CPU (the reference arm uses no GPU); whole workload shapes.
    cases = []
    for c in build_cpu_cases(synth, wl):
        cases.append(c)
    per_step_budget = max(0.02, 120.0 / (args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(cases, per_step_budget)
    f_tot = s_tot = 0.0
    desc = None
    for s in range(args.steps):
        f, secs, thr, desc = oracle_sample(cases, per_step_budget, rng_seed=s + 1)
        f_tot += f
        s_tot += secs
    value = f_tot / s_tot / 1e12
    cpu = {"value": round(value, 6), "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"per step ~{per_step_budget:.2f} s of " + (desc or "")}
    line = {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s_tot / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1), block-quantised to E4M3)",
            "config": {"workload": wl["desc"], "cases": [c.name for c in cases]},
            "impl": "reference", "cpu_baseline": cpu,
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def build_cpu_cases(synth, wl):
    kind = wl["kind"]
    out = []
    if kind == "normal":
        si = 0
        for M in wl["M"]:
            for (N, K) in wl["shapes"]:
                x = synth.normal_inputs(M, N, K, seed=synth.seed_for(wl["cfg"], si))
                si += 1
                out.append(Case(f"M{M}_N{N}_K{K}", 2.0 * M * N * K, 0, None, host={"x": x}))
    elif kind == "contiguous":
        for si, (N, K) in enumerate(wl["shapes"]):
            x = synth.contiguous_inputs(wl["G"], N, K, seed=synth.seed_for(wl["cfg"], si))
            out.append(Case(f"contig_N{N}_K{K}", 0, 0, None, host={"x": x}))
    else:
        for si, (N, K) in enumerate(wl["shapes"]):
            x = synth.masked_inputs(wl["G"], wl["M_max"], N, K, seed=synth.seed_for(wl["cfg"], si))
            out.append(Case(f"masked_N{N}_K{K}", 0, 0, None, host={"x": x}))
    return out


if __name__ == "__main__":
    sys.exit(main())
