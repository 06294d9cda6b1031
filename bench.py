"""Benchmark: KIVI 2-bit KV cache hot path on B200.

One step = one pass of the whole hot path over the Llama-2-7B layer workload
(batch 8, 32 MHA heads, head_dim 128, 4,096-token context, G=32, R=128, bf16):
prefill quantization, then 64 decode steps each appending one token (the first
append flushes the full residual) and running decode attention, the append fused
into the decode launch (kivi_append_decode) except where it flushes.  The step runs
over `--layers` independent layer caches (default 8) visited round-robin, as a
model's decode does, so the working set (~1.1 GB) is far larger than the
126 MB L2 and every decode streams its cache from HBM.

Metric: decode-attention KV tokens x heads per second (sum over decode calls of
B * H_kv * tokens attended), whole step time in the denominator (prefill and
appends included).  The decode kernel's achieved HBM bandwidth (algorithmic
bytes / CUDA-event duration of each launch) is reported against the measured
copy bandwidth in MEASURED_PEAKS.json.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--batch B] [--decode-steps S] [--layers L]

The default workload is the Llama-2-7B layer above; `--workload` times any
other workload of synth.WORKLOADS the same way (a step being its prefill and
decode steps), `--batch` and `--decode-steps` shrink it.

With N > 1 (torchrun, one process per GPU) every rank runs its own replica
(no data exchange: sequences and heads are independent) and the reported value
is the sum over ranks divided by the slowest rank's time.  `--impl reference`
times the plain CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
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

METRIC = "decode-attn KV tokens·heads/s and achieved HBM GB/s vs 8 TB/s"
UNIT = "KV tokens·heads/s"
WORKLOAD = "llama2_7b_layer"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "decode_llama2_7b_layer_traffic.json")
DECODE_SOURCES = ["bit_asymmetric_kv_prefill_b200/csrc/kivi_decode.cu",
                  "bit_asymmetric_kv_prefill_b200/csrc/kivi_common.cuh"]


# ---- workload arithmetic (bytes and units, no method math) ---------------------

def decode_schedule(w):
    """(n_q, r) seen by each decode call of one layer's step, in order."""
    R, T = w.R, w.T
    n_q = R * ((T - 1) // R)
    r = T - n_q
    out = []
    for _ in range(w.steps):
        if r == R:
            n_q += R
            r = 0
        r += 1
        out.append((n_q, r))
    return out


def get_workload(args):
    from bit_asymmetric_kv_prefill_b200 import synth
    w = synth.WORKLOADS[args.workload]
    over = {}
    if args.batch:
        over["B"] = args.batch
    if args.decode_steps:
        over["steps"] = args.decode_steps
    return synth.scaled(w, **over) if over else w


def is_headline(args):
    return args.workload == WORKLOAD and not args.batch and not args.decode_steps


def flush_steps(w):
    """Per decode step, whether its append flushes the residual (n_q grows)."""
    sched = decode_schedule(w)
    n_q0 = w.R * ((w.T - 1) // w.R)
    return [sched[j][0] != (sched[j - 1][0] if j else n_q0) for j in range(w.steps)]


def decode_bytes(w, n_q, r):
    """Algorithmic HBM bytes of one decode call: per quantized (token, kv head)
    the 2-bit K and V codes plus fp16 scale/zero (D/4 + 4D/G for each of K and
    V), per residual token 2*D*2 bytes, plus q (bf16) and out (fp32)."""
    per_q = 2 * (w.D // 4 + 4 * w.D // w.G)
    per_r = 2 * w.D * 2
    return w.B * w.H_kv * (n_q * per_q + r * per_r) + w.B * w.H_q * w.D * (2 + 4)


def decode_units(w, n_q, r):
    return w.B * w.H_kv * (n_q + r)


def source_hash():
    """sha256 of the decode kernel's sources with comments and blank lines
    removed (an edit of comments leaves the compiled kernel, and so the
    recorded counters, as they were)."""
    import re
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def traffic_per_launch(args):
    """dram read+write bytes per decode launch from the committed ncu summary,
    or None when absent, taken on other kernel sources or on another workload."""
    if not is_headline(args):
        return None
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_source_sha256") != source_hash():
        return None
    return d.get("traffic_bytes_per_launch")


# ---- clocks ----------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi samples of one GPU during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_key: str):
        self.bus = bus_key
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu=pci.bus_id,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    @staticmethod
    def _bus_key(bus: str) -> str:
        # nvidia-smi's "00000000:1B:00.0" -> "1b:00.0"
        return bus.strip().lower().split(":", 1)[-1]

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        want = self.bus
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9 or self._bus_key(parts[0]) != want:
                continue
            parts = parts[1:]
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- multi-rank helpers ------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(x: float, device) -> float:
    """Max of a scalar over ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


# ---- CPU oracle leg ------------------------------------------------------------------

def oracle_stream_rate(w, seconds: float, max_seqs: int = 1 << 30):
    """Time the oracle on whole per-sequence streams (prefill + `steps` x
    (append + decode)) of the workload until `seconds` elapse; returns
    (units/s, sequences done, seconds)."""
    import oracle
    from bit_asymmetric_kv_prefill_b200 import synth
    sched = decode_schedule(w)
    units_seq = sum(n_q + r for n_q, r in sched)
    one = synth.scaled(w, B=1, H_q=w.H_q // w.H_kv, H_kv=1)
    done, t_used = 0, 0.0
    dt = oracle.DTYPE_BF16 if w.dtype == "bf16" else oracle.DTYPE_F16
    while (t_used < seconds or done == 0) and done < max_seqs:
        K, V = synth.prefill_inputs(one, seed=done)
        kb, vb = synth.bits(K), synth.bits(V)
        steps = [tuple(synth.bits(x) for x in synth.step_inputs(one, s, seed=done))
                 for s in range(1, w.steps + 1)]
        c = oracle.OracleCache(1, 1, w.D, w.G, w.R, dt, w.T_max, pre_rope=w.pre_rope,
                               rope_theta=w.rope_theta)
        t0 = time.perf_counter()
        c.prefill(kb, vb)
        for k, v, q in steps:
            c.append(k, v)
            c.decode(q)
        t_used += time.perf_counter() - t0
        done += 1
    return units_seq * done / t_used, done, t_used


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from bit_asymmetric_kv_prefill_b200 import synth
    oracle.build()
    w = get_workload(args)
    for _ in range(args.warmup):
        oracle_stream_rate(w, 0.0, max_seqs=1)
    t_total, units_total = 0.0, 0.0
    units_seq = sum(n_q + r for n_q, r in decode_schedule(w))
    for _ in range(args.steps):
        _, n, t = oracle_stream_rate(w, 0.0, max_seqs=1)
        t_total += t
        units_total += units_seq * n
    value = units_total / t_total
    sample = (f"each step: one (batch, head) sequence of {w.name}: prefill T={w.T} + "
              f"{w.steps} x (append + decode), single thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---- GPU leg ----------------------------------------------------------------------------

def workload_config(w, args):
    heads = f"{w.H_q} MHA heads" if w.H_q == w.H_kv else f"{w.H_q} query heads over {w.H_kv} kv heads"
    title = "Llama-2-7B layer shape, " if w.name == WORKLOAD else ""
    rope = f", keys pre-RoPE (theta {w.rope_theta:g})" if w.pre_rope else ""
    per_layer = w.B * w.H_kv * (w.T_max * 2 * (w.D // 4 + 4 * w.D // w.G) + w.R * 4 * w.D)
    ws_mb = args.layers * per_layer / 1e6
    l2 = (f"inputs larger than L2: {args.layers} layer caches visited round-robin "
          f"(~{ws_mb:.0f} MB working set vs 126 MB L2), no explicit flush") if ws_mb > 126 else \
         f"working set {ws_mb:.0f} MB, not larger than L2 (126 MB)"
    return {"workload": f"{w.name}: {title}batch {w.B}, {heads}, head_dim {w.D}, context {w.T}, "
                        f"G={w.G}, R={w.R}, {w.dtype} input/residual{rope}, "
                        f"prefill + {w.steps} x (append + decode) per layer",
            "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "D": w.D, "T": w.T, "G": w.G, "R": w.R,
            "decode_steps": w.steps, "layers_round_robin": args.layers, "l2": l2,
            "parallelism": f"replicas x{max(1, args.gpus)} (no data-path collective)"}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import bit_asymmetric_kv_prefill_b200 as kivi
    from bit_asymmetric_kv_prefill_b200 import KiviCache, synth
    from bit_asymmetric_kv_prefill_b200 import build as kbuild
    kbuild.build()
    L = kivi.lib()

    w = get_workload(args)
    nl = args.layers
    sched = decode_schedule(w)
    # A fused launch also reads k_t, v_t and writes them to the residual.
    fused_extra = 4 * w.B * w.H_kv * w.D * 2 * (w.steps - sum(flush_steps(w)))
    bytes_step = (sum(decode_bytes(w, n, r) for n, r in sched) + fused_extra) * nl
    units_step = sum(decode_units(w, n, r) for n, r in sched) * nl
    launches_step = nl * (1 + w.steps + sum(flush_steps(w)))

    caches = [KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T_max, pre_rope=w.pre_rope,
                        rope_theta=w.rope_theta) for _ in range(nl)]
    Ks, Vs = [], []
    for l in range(nl):
        K, V = synth.prefill_inputs(w, seed=1000 * rank + l, device=dev)
        Ks.append(K)
        Vs.append(V)
    steps = [[synth.step_inputs(w, s, seed=1000 * rank + l, device=dev) for l in range(nl)]
             for s in range(1, w.steps + 1)]
    outs = [torch.empty(w.B, w.H_q, w.D, dtype=torch.float32, device=dev) for _ in range(nl)]
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    H = [c._h for c in caches]
    Kp = [ctypes.c_void_p(t.data_ptr()) for t in Ks]
    Vp = [ctypes.c_void_p(t.data_ptr()) for t in Vs]
    Sp = [[tuple(ctypes.c_void_p(t.data_ptr()) for t in st) for st in row] for row in steps]
    Op = [ctypes.c_void_p(o.data_ptr()) for o in outs]
    T, Hq = w.T, w.H_q
    reset, prefill, append, decode, fused = (L.kivi_cache_reset, L.kivi_prefill, L.kivi_append,
                                             L.kivi_decode_attn, L.kivi_append_decode)
    # Steps whose append flushes (the quantizer runs): append, then decode;
    # the others fuse the append into the decode launch.  Either way the timed
    # launch is one decode.
    flush = flush_steps(w)

    def one_step(ev=None):
        bad = 0
        for l in range(nl):
            bad |= reset(H[l])
            bad |= prefill(H[l], Kp[l], Vp[l], T, sp)
        i = 0
        for j, row in enumerate(Sp):
            for l in range(nl):
                k, v, q = row[l]
                if flush[j]:
                    bad |= append(H[l], k, v, sp)
                if ev is not None:
                    ev[i][0].record(stream)
                if flush[j]:
                    bad |= decode(H[l], q, Hq, Op[l], sp)
                else:
                    bad |= fused(H[l], k, v, q, Hq, Op[l], sp)
                if ev is not None:
                    ev[i][1].record(stream)
                i += 1
        if bad:
            raise RuntimeError("a KIVI call failed during the benchmark")

    for _ in range(args.warmup):
        one_step()
    n_dec = nl * w.steps
    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in range(n_dec)] for _ in range(args.steps)]
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(f"{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0")
    barrier(dev)
    clocks.start()
    time.sleep(0.3)  # let the sampler attach before the timed region
    t0e.record(stream)
    for k in range(args.steps):
        one_step(events[k])
    t1e.record(stream)
    torch.cuda.synchronize(dev)
    ck = clocks.stop()
    barrier(dev)
    ms_local = t0e.elapsed_time(t1e)
    dec_ms = [a.elapsed_time(b) for ev in events for a, b in ev]
    dec_avg_local = sum(dec_ms) / len(dec_ms)
    status = max(c.device_status() for c in caches)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    ms = reduce_max(ms_local, dev)
    dec_avg = reduce_max(dec_avg_local, dev)
    value = world * units_step * args.steps / (ms / 1e3)
    bytes_per_launch = bytes_step / n_dec
    achieved = bytes_per_launch / (dec_avg / 1e3) / 1e9
    peak, peak_kind = measured_peak()
    traffic = traffic_per_launch(args)

    e2e = run_e2e(args, w, caches, Ks, Vs, steps, dev, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nseq, secs = oracle_stream_rate(w, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{nseq} (batch, head) sequences of {w.name}, each prefill T={w.T} + "
                         f"{w.steps} x (append + decode); {secs:.1f} s single-threaded"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic", "config": workload_config(w, args),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                         "kernel": "decode_kernel (kivi_decode_attn)",
                         "alg_bytes_per_launch": bytes_per_launch,
                         "frac_of_8TBps": achieved / 8000.0},
            "decode_attn": {"avg_us": 1e3 * dec_avg,
                            "median_us": 1e3 * statistics.median(dec_ms),
                            "p90_us": 1e3 * sorted(dec_ms)[int(0.9 * (len(dec_ms) - 1))],
                            "launches_timed": len(dec_ms),
                            "tokens_heads_per_s": units_step / nl / w.steps / (dec_avg / 1e3),
                            "gpu_time_share": sum(dec_ms) / ms_local},
            "e2e": e2e, "gpu_launches": launches_step * args.steps, "clocks": ck,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    for c in caches:
        c.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, w, caches, Ks, Vs, steps, dev, world):
    """Same step through the public API with pinned HOST inputs: the H2D copies
    of every input and the D2H read of every decode output are timed.

    Copies run on their own stream, as a serving loop would run them: step
    k+1's prefill inputs stream in while step k computes (each layer's buffer
    is refilled once that layer's prefill has read it), and each step's decode
    inputs land in one of two buffer sets.  Every timed step's copies happen
    inside the timed region; outputs return on the compute stream."""
    import torch
    nl = len(caches)
    hK = [k.cpu().pin_memory() for k in Ks]
    hV = [v.cpu().pin_memory() for v in Vs]
    hS = [[tuple(t.cpu().pin_memory() for t in st) for st in row] for row in steps]
    dK = [torch.empty_like(Ks[0]) for _ in range(nl)]
    dV = [torch.empty_like(Vs[0]) for _ in range(nl)]
    dS = [[[tuple(torch.empty_like(t) for t in steps[0][0]) for _ in range(nl)] for _ in hS]
          for _ in range(2)]
    hout = [torch.empty(w.B, w.H_q, w.D, dtype=torch.float32).pin_memory() for _ in range(nl)]
    cs = torch.cuda.current_stream(dev)
    xs = torch.cuda.Stream(dev)
    xs2 = torch.cuda.Stream(dev)  # values on a second copy engine
    ev_in = [torch.cuda.Event() for _ in range(nl)]
    ev_in2 = [torch.cuda.Event() for _ in range(nl)]
    ev_used = [torch.cuda.Event() for _ in range(nl)]
    ev_sin = [torch.cuda.Event() for _ in range(2)]
    ev_sused = [torch.cuda.Event() for _ in range(2)]
    for e in ev_used + ev_sused:
        e.record(cs)

    def copies(k):
        b = k % 2
        for l in range(nl):
            xs.wait_event(ev_used[l])
            xs2.wait_event(ev_used[l])
            with torch.cuda.stream(xs):
                dK[l].copy_(hK[l], non_blocking=True)
                ev_in[l].record(xs)
            with torch.cuda.stream(xs2):
                dV[l].copy_(hV[l], non_blocking=True)
                ev_in2[l].record(xs2)
        with torch.cuda.stream(xs):
            xs.wait_event(ev_sused[b])
            for j, row in enumerate(hS):
                for l in range(nl):
                    for d, h in zip(dS[b][j][l], row[l]):
                        d.copy_(h, non_blocking=True)
            ev_sin[b].record(xs)

    def compute(k):
        b = k % 2
        for l in range(nl):
            cs.wait_event(ev_in[l])
            cs.wait_event(ev_in2[l])
            caches[l].reset()
            caches[l].prefill(dK[l], dV[l])
            ev_used[l].record(cs)
        cs.wait_event(ev_sin[b])
        for j in range(len(hS)):
            for l in range(nl):
                k_t, v_t, q = dS[b][j][l]
                out = caches[l].append_decode(k_t, v_t, q)
                hout[l].copy_(out, non_blocking=True)
        ev_sused[b].record(cs)

    def run(n):
        copies(0)
        for k in range(n):
            compute(k)
            if k + 1 < n:
                copies(k + 1)

    n = max(1, min(args.steps, args.e2e_steps))
    run(1)
    torch.cuda.synchronize(dev)
    barrier(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(cs)
    run(n)
    b.record(cs)
    torch.cuda.synchronize(dev)
    barrier(dev)
    ms = reduce_max(a.elapsed_time(b), dev)
    sched = decode_schedule(w)
    units = sum(decode_units(w, nq, r) for nq, r in sched) * nl
    h2d = nl * (2 * Ks[0].numel() * 2 + w.steps * sum(t.numel() * 2 for t in steps[0][0]))
    d2h = nl * w.steps * w.B * w.H_q * w.D * 4
    return {"value": world * units * n / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": ms / n,
            "copies": "H2D on two copy streams (keys, values), step k+1's inputs during step k"}


DIAG_MODES = {
    # mode: ((key axis, symmetric, sparse), (value axis, symmetric, sparse));
    # axis 0 = per channel, sparse 1 = one exactly kept element per group
    "kivi": ((0, False, 0), (1, False, 0)),
    "k_per_token": ((1, False, 0), (1, False, 0)),
    "v_per_channel": ((0, False, 0), (0, False, 0)),
    "naive_symmetric": ((1, True, 0), (1, True, 0)),
    "kivi_sparse": ((0, False, 1), (1, False, 1)),
    "k_per_token_sparse": ((1, False, 1), (1, False, 1)),
}


def run_diag(args):
    """Time kivi_fake_quant over every key and value matrix of one Llama-2-13B
    layer cache (16 x 40 heads, 4,096 tokens, head_dim 128, bf16, heavy-tailed
    keys) under the groupings the KIVI article compares, 2 bits.  Each launch
    reads 2 B and writes 4 B (fp32 x_hat) per element; the inputs (1.3 GB)
    exceed L2.  Reports per-mode launch times, achieved HBM GB/s and the
    relative Frobenius errors ||X - X_hat|| / ||X|| from the kernel's own sums."""
    import torch
    import bit_asymmetric_kv_prefill_b200 as kivi
    from bit_asymmetric_kv_prefill_b200 import synth
    from bit_asymmetric_kv_prefill_b200 import build as kbuild
    kbuild.build()
    L = kivi.lib()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS["llama2_13b_cache"]
    if args.batch:
        w = synth.scaled(w, B=args.batch)
    K, V = synth.prefill_inputs(w, seed=0, device=dev)
    N, T, D = w.B * w.H_kv, w.T, w.D
    xh = torch.empty((N, T, D), dtype=torch.float32, device=dev)
    err = torch.empty(N, dtype=torch.float64, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    dt = kivi.KIVI_BF16
    norms = {"K": float(K.double().pow(2).sum()), "V": float(V.double().pow(2).sum())}
    src = {"K": ctypes.c_void_p(K.data_ptr()), "V": ctypes.c_void_p(V.data_ptr())}
    xhp, errp = ctypes.c_void_p(xh.data_ptr()), ctypes.c_void_p(err.data_ptr())
    elems = N * T * D

    def launch(which, axis, sym, sparse, values=True):
        rc = L.kivi_fake_quant(src[which], dt, N, T, D, axis, 32, 2, int(sym), sparse,
                               xhp if values else None, errp, sp)
        if rc:
            raise RuntimeError(f"kivi_fake_quant failed: {kivi.status_string(rc)}")

    plan = []
    for mode, ((ka, ks, ko), (va, vs, vo)) in DIAG_MODES.items():
        plan.append((mode, "K", ka, ks, ko, True))
        plan.append((mode, "V", va, vs, vo, True))
    plan.append(("kivi_error_only", "K", 0, False, 0, False))
    plan.append(("kivi_error_only", "V", 1, False, 0, False))
    for _ in range(args.warmup):
        for _, which, axis, sym, sparse, values in plan:
            launch(which, axis, sym, sparse, values)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in plan] for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(f"{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0")
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0e.record(stream)
    for k in range(args.steps):
        for i, (_, which, axis, sym, sparse, values) in enumerate(plan):
            ev[k][i][0].record(stream)
            launch(which, axis, sym, sparse, values)
            ev[k][i][1].record(stream)
    t1e.record(stream)
    torch.cuda.synchronize(dev)
    ck = clocks.stop()
    ms = t0e.elapsed_time(t1e)
    peak, peak_kind = measured_peak()
    modes = {}
    for i, (mode, which, axis, sym, sparse, values) in enumerate(plan):
        us = 1e3 * sum(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps)) / args.steps
        nbytes = elems * (6 if values else 2)
        m = modes.setdefault(mode, {})
        m[f"{which}_us"] = us
        m[f"{which}_gbs"] = nbytes / (us / 1e6) / 1e9
    # errors of each mode (one more untimed pass, read back)
    for mode, ((ka, ks, ko), (va, vs, vo)) in DIAG_MODES.items():
        for which, axis, sym, sparse in (("K", ka, ks, ko), ("V", va, vs, vo)):
            launch(which, axis, sym, sparse, values=False)
            modes[mode][f"{which}_rel_err"] = (float(err.sum()) / norms[which]) ** 0.5
    launches = len(plan) * args.steps
    cpu = None
    if not args.no_cpu_baseline:
        # the oracle as it stands, single-threaded, on whole key matrices of
        # the same cache (keys per channel, 2 bits), for about cpu_seconds
        import oracle
        Kh = K.reshape(N, T, D)
        done, t0 = 0, time.perf_counter()
        while done < N and (done == 0 or time.perf_counter() - t0 < args.cpu_seconds):
            oracle.fake_quant(Kh[done].float().cpu().numpy(), 0, 32, 2, False)
            done += 1
        secs = time.perf_counter() - t0
        cpu = {"value": done * T * D / secs, "unit": "elements/s", "cores": 1, "kind": "oracle",
               "sample": f"{done} key matrices ({T} x {D}) of the same cache, per channel, "
                         f"{secs:.1f} s single-threaded"}
    dom = modes["kivi"]
    achieved = elems * 6 / (dom["K_us"] / 1e6) / 1e9
    print(json.dumps({
        "metric": "fake-quant elements/s", "value": launches * elems / (ms / 1e3),
        "unit": "elements/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
        "config": {"workload": "llama2_13b_layer_cache fake quantization, 6 groupings + error-only",
                   "batch": w.B, "matrices": N, "T": T, "D": D, "G": 32, "bits": 2, "input": "bf16",
                   "l2": f"inputs {2 * K.numel() * 2 / 1e9:.2f} GB vs 0.126 GB L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "kernel": "fq_channel_kernel (kivi_fake_quant, keys per channel)",
                     "alg_bytes_per_launch": elems * 6},
        "modes": modes, "gpu_launches": launches, "clocks": ck, "cpu_baseline": cpu,
    }), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kivi", "reference"], default="kivi")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--e2e-steps", dest="e2e_steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", dest="cpu_seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", dest="no_cpu_baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["tiny", "llama2_7b_layer", "llama2_13b_cache", "mistral_gqa", "long_context"])
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch")
    ap.add_argument("--decode-steps", dest="decode_steps", type=int, default=0,
                    help="override the workload's decode steps")
    ap.add_argument("--diag", action="store_true",
                    help="time the diagnostic grouping modes (kivi_fake_quant) instead")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.diag:
        return run_diag(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
