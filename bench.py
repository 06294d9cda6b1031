"""Benchmark: KIVI 2-bit KV cache hot path on B200.

The reported line is the largest single-GPU workload, the GQA Mistral-7B-like
stream: batch 64, 32 query heads over 8 kv heads, head_dim 128, a 32,768-token
context, G=32, R=128, bf16.  One step is one pass of the whole hot path over
it: prefill quantization of the context, then 256 decode steps, each appending
one token (the full residual flushes at steps 1 and 129) and running decode
attention; the append is fused into the decode launch (kivi_append_decode)
except where it flushes.  The packed cache (1.6 GB) is far larger than the
126 MB L2, so every decode streams it from HBM.

Metric: decode-attention KV tokens x heads per second (sum over decode calls
of B * H_kv * tokens attended), whole step time in the denominator (prefill
and appends included).  The decode kernel's achieved HBM bandwidth
(algorithmic bytes / CUDA-event duration of each launch) is reported against
the measured copy bandwidth in MEASURED_PEAKS.json.

`per_config` in the same line measures the other workloads the same way:
  llama2_7b_layer   batch 8, 32 MHA heads, 4,096 tokens, prefill + 64 steps,
                    8 layer caches visited round-robin;
  llama2_13b_cache  40 layers of batch 16 x 40 MHA heads at 4,096 tokens:
                    each layer's prefill and one decode over it, with the
                    cache bytes checked against the record's 128,000 B/token;
  long_context      batch 1, 32/8 heads, 131,072 tokens, keys pre-RoPE:
                    the timed 128K-token prefill and 32 decode steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--batch B] [--decode-steps S] [--layers L]
                    [--no-per-config] [--no-cpu-baseline] [--diag]

With N > 1 (torchrun, one process per GPU) every rank runs its own replica
(no data exchange: sequences and heads are independent) and the reported value
is the sum over ranks divided by the slowest rank's time.  `--impl reference`
times the plain CPU oracle on a bounded sample of the same workload, on the
host's cores.
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
WORKLOAD = "mistral_gqa"
PER_CONFIG = ("llama2_7b_layer", "llama2_13b_cache", "long_context")
WORKLOAD_NAMES = ["tiny", "llama2_7b_layer", "llama2_13b_cache", "mistral_gqa", "long_context"]
# Layer caches per step (visited round-robin) and distinct prefill inputs they
# share: the Llama-2-13B cache has 40 layers; four input sets keep its inputs
# at 11 GB while every layer keeps its own cache.
LAYERS = {"tiny": 8, "llama2_7b_layer": 8, "llama2_13b_cache": 40, "mistral_gqa": 1,
          "long_context": 8}
INPUT_SETS = {"llama2_13b_cache": 4}
# Decode steps per sequence the CPU oracle runs in its bounded sample.
ORACLE_STEPS = {"mistral_gqa": 8, "long_context": 2}
PROFILE_TRAFFIC = {
    "llama2_7b_layer": os.path.join(ROOT, "profiles", "decode_llama2_7b_layer_traffic.json"),
    "mistral_gqa": os.path.join(ROOT, "profiles", "decode_mistral_gqa_traffic.json"),
}
DECODE_SOURCES = ["bit_asymmetric_kv_prefill_b200/csrc/kivi_decode.cu",
                  "bit_asymmetric_kv_prefill_b200/csrc/kivi_decode_ops.cuh",
                  "bit_asymmetric_kv_prefill_b200/csrc/kivi_common.cuh"]


# ---- workload arithmetic (bytes and units, no method math) ---------------------

def decode_calls(w):
    """Decode calls of one layer's step, in order: (n_q, r, kind) seen by each,
    kind "flush" (its append quantizes the full residual first, a separate
    launch), "fused" (append fused into the decode launch) or "none" (a
    workload without decode steps: one decode over the prefilled cache)."""
    R, T = w.R, w.T
    n_q = R * ((T - 1) // R)
    r = T - n_q
    if w.steps == 0:
        return [(n_q, r, "none")]
    out = []
    for _ in range(w.steps):
        kind = "fused"
        if r == R:
            n_q += R
            r = 0
            kind = "flush"
        r += 1
        out.append((n_q, r, kind))
    return out


def decode_schedule(w):
    """(n_q, r) seen by each decode call of one layer's step, in order."""
    return [(n_q, r) for n_q, r, _ in decode_calls(w)]


def flush_steps(w):
    """Per decode call, whether its append flushes the residual."""
    return [kind == "flush" for _, _, kind in decode_calls(w)]


def get_workload(args, name=None):
    from bit_asymmetric_kv_prefill_b200 import synth
    w = synth.WORKLOADS[name or args.workload]
    over = {}
    if name is None and args.batch:
        over["B"] = args.batch
    if name is None and args.decode_steps:
        over["steps"] = args.decode_steps
    return synth.scaled(w, **over) if over else w


def is_headline(args):
    return args.workload == WORKLOAD and not args.batch and not args.decode_steps


def decode_bytes(w, n_q, r):
    """Algorithmic HBM bytes of one decode call: per quantized (token, kv head)
    the 2-bit K and V codes plus fp16 scale/zero (D/4 + 4D/G for each of K and
    V), per residual token 2*D*2 bytes, plus q (bf16) and out (fp32)."""
    per_q = 2 * (w.D // 4 + 4 * w.D // w.G)
    per_r = 2 * w.D * 2
    return w.B * w.H_kv * (n_q * per_q + r * per_r) + w.B * w.H_q * w.D * (2 + 4)


def decode_flops(w, n_q, r):
    """Algorithmic flops of one decode call: per (token, query head) a D-long
    dot product with the key and a D-long weighted sum of the value, 2 flops
    per multiply-add each."""
    return 4 * w.D * w.B * w.H_q * (n_q + r)


def fma_peak_tflops(sms, sm_mhz):
    """fp32 FMA peak of the CUDA cores: 4 schedulers per SM, each issuing one
    32-lane FMA instruction per clock (2 flops per lane)."""
    return sms * 4 * 32 * 2 * sm_mhz * 1e6 / 1e12


def fused_append_bytes(w):
    """A fused launch also reads k_t, v_t and writes them to the residual."""
    return 4 * w.B * w.H_kv * w.D * 2


def prefill_bytes(w):
    """Algorithmic HBM bytes of a prefill: K and V read once (2 B per element),
    the packed groups written (24*D bytes per 32 quantized tokens of a
    sequence: codes and fp16 scale/zero of keys and values) and the r residual
    rows of K and V written."""
    n_q = w.R * ((w.T - 1) // w.R)
    r = w.T - n_q
    seqs = w.B * w.H_kv
    return seqs * (2 * w.T * w.D * 2 + (n_q // w.G) * 24 * w.D + 2 * r * w.D * 2)


def decode_units(w, n_q, r):
    return w.B * w.H_kv * (n_q + r)


def cache_record_bytes(w, layers):
    """Per-token bytes of `layers` layer caches of capacity w.T, as the record
    counts them: every context token's 2-bit codes plus a full R-slot residual
    (and, separately, the fp16 scale/zero metadata)."""
    per_layer_codes = w.B * w.H_kv * w.T * w.D * 2 * 2 // 8
    per_layer_res = w.B * w.H_kv * w.R * w.D * 2 * 2
    per_layer_meta = w.B * w.H_kv * w.T * 2 * (4 * w.D // w.G)
    return (layers * (per_layer_codes + per_layer_res) / (w.B * w.T),
            layers * per_layer_meta / (w.B * w.T))


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


def traffic_per_launch(w, full_size):
    """dram read+write bytes per decode launch from the committed ncu summary
    of this workload, or None when absent, taken on other kernel sources or
    when the workload was shrunk."""
    path = PROFILE_TRAFFIC.get(w.name)
    if not full_size or path is None:
        return None
    try:
        with open(path) as f:
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


def clock_sampler(dev):
    import torch
    props = torch.cuda.get_device_properties(dev)
    return ClockSampler(f"{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0")


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

def oracle_sample(w, steps=None):
    """The oracle's unit of work: one (batch, kv head) sequence of the workload,
    prefill of w.T tokens then its first `steps` decode calls (all by
    default), each appending its token first.  Returns the one-sequence
    workload, its calls and their KV token x head units."""
    from bit_asymmetric_kv_prefill_b200 import synth
    calls = decode_calls(w)
    if steps is not None:
        calls = calls[:max(1, steps)]
    one = synth.scaled(w, B=1, H_q=w.H_q // w.H_kv, H_kv=1)
    return one, calls, sum(n_q + r for n_q, r, _ in calls)


def _oracle_inputs(one, calls, seed):
    from bit_asymmetric_kv_prefill_b200 import synth
    K, V = synth.prefill_inputs(one, seed=seed)
    steps = [tuple(synth.bits(x) for x in synth.step_inputs(one, s, seed=seed))
             for s in range(1, len(calls) + 1)]
    return synth.bits(K), synth.bits(V), steps


def _oracle_sequence(one, w, calls, inp):
    import oracle
    kb, vb, steps = inp
    dt = oracle.DTYPE_BF16 if w.dtype == "bf16" else oracle.DTYPE_F16
    c = oracle.OracleCache(1, 1, w.D, w.G, w.R, dt, w.T_max, pre_rope=w.pre_rope,
                           rope_theta=w.rope_theta)
    c.prefill(kb, vb)
    for (_, _, kind), (k, v, q) in zip(calls, steps):
        if kind != "none":
            c.append(k, v)
        c.decode(q)


def oracle_rate(w, seconds: float, threads: int, steps=None, waves: int = 0):
    """Time the oracle on whole sequence samples (see oracle_sample) on
    `threads` threads at once (each C call releases the GIL).  Threads loop
    over samples until `seconds` have passed (at least one each), or run
    exactly `waves` samples each.  Returns (units/s, samples done, wall s)."""
    one, calls, units = oracle_sample(w, steps)
    n_inputs = min(threads, 4)
    inputs = [_oracle_inputs(one, calls, seed=i) for i in range(n_inputs)]
    start = threading.Barrier(threads + 1)
    done = [0] * threads
    ends = [0.0] * threads
    t0 = [0.0]

    def worker(i):
        start.wait()
        n = 0
        while True:
            _oracle_sequence(one, w, calls, inputs[(i + n) % n_inputs])
            n += 1
            now = time.perf_counter()
            if (waves and n >= waves) or (not waves and now - t0[0] >= seconds):
                break
        done[i] = n
        ends[i] = now

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(threads)]
    for t in ts:
        t.start()
    t0[0] = time.perf_counter()
    start.wait()
    for t in ts:
        t.join()
    wall = max(ends) - t0[0]
    return units * sum(done) / wall, sum(done), wall


def oracle_threads():
    import oracle
    return oracle.workers()


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = get_workload(args)
    threads = oracle_threads()
    k = ORACLE_STEPS.get(w.name)
    _, calls, units = oracle_sample(w, k)
    for _ in range(args.warmup):
        oracle_rate(w, 0.0, threads, k, waves=1)
    t_total, units_total = 0.0, 0.0
    for _ in range(args.steps):
        _, n, t = oracle_rate(w, 0.0, threads, k, waves=1)
        t_total += t
        units_total += units * n
    value = units_total / t_total
    sample = (f"each step: {threads} threads, each one (batch, kv head) sequence of {w.name}: "
              f"prefill T={w.T} + {len(calls)} of its {len(decode_calls(w))} decode calls "
              f"(append + decode)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args, LAYERS[w.name], world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(w, seconds):
    """The oracle on the host's cores (and on one thread) over bounded samples
    of the workload."""
    threads = oracle_threads()
    k = ORACLE_STEPS.get(w.name)
    _, calls, _ = oracle_sample(w, k)
    rate, n, wall = oracle_rate(w, seconds, threads, k)
    rate1, n1, wall1 = oracle_rate(w, seconds / 3, 1, k)
    what = (f"(batch, kv head) sequences of {w.name}, each prefill T={w.T} + the first "
            f"{len(calls)} of its {len(decode_calls(w))} decode calls (append + decode)")
    return {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} {what} on {threads} threads in {wall:.1f} s",
            "single_thread": {"value": rate1, "unit": UNIT,
                              "sample": f"{n1} such sequences on one thread in {wall1:.1f} s"}}


# ---- GPU leg ----------------------------------------------------------------------------

def workload_config(w, args, layers, world, sets=None):
    heads = f"{w.H_q} MHA heads" if w.H_q == w.H_kv else f"{w.H_q} query heads over {w.H_kv} kv heads"
    rope = f", keys pre-RoPE (theta {w.rope_theta:g})" if w.pre_rope else ""
    per_layer = w.B * w.H_kv * (w.T_max * 2 * (w.D // 4 + 4 * w.D // w.G) + w.R * 4 * w.D)
    ws_mb = layers * per_layer / 1e6
    steps = (f"prefill + {w.steps} x (append + decode)" if w.steps else "prefill + one decode")
    l2 = (f"inputs larger than L2: {layers} layer cache(s) of {per_layer / 1e6:.0f} MB visited "
          f"round-robin (~{ws_mb:.0f} MB working set vs 126 MB L2), no explicit flush") \
        if ws_mb > 126 else f"working set {ws_mb:.0f} MB, not larger than L2 (126 MB)"
    cfg = {"workload": f"{w.name}: batch {w.B}, {heads}, head_dim {w.D}, context {w.T}, "
                       f"G={w.G}, R={w.R}, {w.dtype} input/residual{rope}, {steps} per layer",
           "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "D": w.D, "T": w.T, "G": w.G, "R": w.R,
           "decode_steps": w.steps, "layers_round_robin": layers, "l2": l2,
           "parallelism": f"replicas x{max(1, world)} (no data-path collective)"}
    if sets and sets < layers:
        cfg["prefill_input_sets"] = sets
    return cfg


class Workbench:
    """Caches and device-resident inputs of one workload, and its timed step."""

    def __init__(self, w, layers, sets, rank, dev):
        import torch
        import bit_asymmetric_kv_prefill_b200 as kivi
        from bit_asymmetric_kv_prefill_b200 import KiviCache, synth
        self.w, self.nl, self.dev = w, layers, dev
        self.sets = min(sets, layers)
        self.L = kivi.lib()
        self.calls = decode_calls(w)
        self.caches = [KiviCache(w.B, w.H_kv, w.D, w.G, w.R, w.torch_dtype, w.T_max,
                                 pre_rope=w.pre_rope, rope_theta=w.rope_theta)
                       for _ in range(layers)]
        self.Ks, self.Vs = [], []
        for l in range(self.sets):
            K, V = synth.prefill_inputs(w, seed=1000 * rank + l, device=dev)
            self.Ks.append(K)
            self.Vs.append(V)
        # per call, per input set: (k_t, v_t, q)
        self.steps = [[synth.step_inputs(w, max(s, 1), seed=1000 * rank + l, device=dev)
                       for l in range(self.sets)] for s in range(1, len(self.calls) + 1)]
        self.outs = [torch.empty(w.B, w.H_q, w.D, dtype=torch.float32, device=dev)
                     for _ in range(layers)]
        self.stream = torch.cuda.current_stream(dev)
        self.sp = ctypes.c_void_p(self.stream.cuda_stream)
        self.H = [c._h for c in self.caches]
        self.Kp = [ctypes.c_void_p(t.data_ptr()) for t in self.Ks]
        self.Vp = [ctypes.c_void_p(t.data_ptr()) for t in self.Vs]
        self.Sp = [[tuple(ctypes.c_void_p(t.data_ptr()) for t in st) for st in row]
                   for row in self.steps]
        self.Op = [ctypes.c_void_p(o.data_ptr()) for o in self.outs]
        self.units_step = sum(decode_units(w, n, r) for n, r, _ in self.calls) * layers
        self.flops_step = sum(decode_flops(w, n, r) for n, r, _ in self.calls) * layers
        self.sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.bytes_step = (sum(decode_bytes(w, n, r) for n, r, _ in self.calls)
                           + fused_append_bytes(w) * sum(k == "fused" for _, _, k in self.calls)) * layers
        self.n_dec = layers * len(self.calls)
        self.launches_step = layers * (1 + len(self.calls) + sum(k == "flush" for _, _, k in self.calls))

    def step(self, runs=None, pre_ev=None, pool=None):
        """One step: every layer's reset and prefill, then the decode calls.
        When timing, events (CUDA, on the launching stream) bracket each
        prefill and each run of back-to-back decode launches (a flush's
        quantizer launch ends a run): `runs` receives (start, end, launches)
        per run, events drawn from `pool`."""
        L, H, sp, w = self.L, self.H, self.sp, self.w
        bad = 0
        for l in range(self.nl):
            i = l % self.sets
            bad |= L.kivi_cache_reset(H[l])
            if pre_ev is not None:
                pre_ev[l][0].record(self.stream)
            bad |= L.kivi_prefill(H[l], self.Kp[i], self.Vp[i], w.T, sp)
            if pre_ev is not None:
                pre_ev[l][1].record(self.stream)
        run = None   # [start event, launches] of the open run

        def close_run():
            nonlocal run
            if run is not None:
                e = pool.pop()
                e.record(self.stream)
                runs.append((run[0], e, run[1]))
                run = None

        for c, (_, _, kind) in enumerate(self.calls):
            row = self.Sp[c]
            for l in range(self.nl):
                k, v, q = row[l % self.sets]
                if kind == "flush":
                    if runs is not None:
                        close_run()
                    bad |= L.kivi_append(H[l], k, v, sp)
                if runs is not None and run is None:
                    e = pool.pop()
                    e.record(self.stream)
                    run = [e, 0]
                if kind == "fused":
                    bad |= L.kivi_append_decode(H[l], k, v, q, w.H_q, self.Op[l], sp)
                else:
                    bad |= L.kivi_decode_attn(H[l], q, w.H_q, self.Op[l], sp)
                if runs is not None:
                    run[1] += 1
        if runs is not None:
            close_run()
        if bad:
            raise RuntimeError("a KIVI call failed during the benchmark")

    def measure(self, steps, warmup, clocks=True):
        """Warm up, then time `steps` steps: device time of the whole region,
        of every prefill, and of every run of back-to-back decode launches
        (per-launch duration = the runs' total over their launches; an event
        between every two launches would add its own gap to each).  Returns
        a dict of timings."""
        import torch
        for _ in range(warmup):
            self.step()
        ev = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        flush_launches = self.nl * sum(k == "flush" for _, _, k in self.calls)
        pool = [torch.cuda.Event(enable_timing=True) for _ in range(steps * 2 * (flush_launches + 2))]
        runs = []
        pre_ev = [[ev() for _ in range(self.nl)] for _ in range(steps)]
        t0e, t1e = ev()
        ck = clock_sampler(self.dev) if clocks else None
        barrier(self.dev)
        if ck:
            ck.start()
            time.sleep(0.3)  # let the sampler attach before the timed region
        t0e.record(self.stream)
        for k in range(steps):
            self.step(runs, pre_ev[k], pool)
        t1e.record(self.stream)
        torch.cuda.synchronize(self.dev)
        cks = ck.stop() if ck else None
        barrier(self.dev)
        status = max(c.device_status() for c in self.caches)
        if status != 0:
            raise RuntimeError(f"device status {status} after the timed region")
        run_ms = [(a.elapsed_time(b), n) for a, b, n in runs]
        pre_ms = [a.elapsed_time(b) for row in pre_ev for a, b in row]
        return {"ms": t0e.elapsed_time(t1e), "runs": run_ms, "pre_ms": pre_ms, "clocks": cks}

    def close(self):
        for c in self.caches:
            c.close()


def sm_clock(t):
    """Median SM clock sampled during the timed region (MHz), else the B200's
    maximum."""
    ck = t.get("clocks") or {}
    return ck.get("sm_mhz") or ck.get("sm_max_mhz") or 1965.0


def roofline(wb, dec_avg_ms, t, peak, peak_kind, traffic):
    """The decode kernel against both ceilings that can bind it: HBM (its
    algorithmic bytes per launch over the measured copy bandwidth) and the
    CUDA cores' fp32 FMA peak (its algorithmic flops per launch).  `bound`
    names the one it is closer to; the other is reported beside it."""
    bpl = wb.bytes_step / wb.n_dec
    fpl = wb.flops_step / wb.n_dec
    gbs = bpl / (dec_avg_ms / 1e3) / 1e9
    tfs = fpl / (dec_avg_ms / 1e3) / 1e12
    mhz = sm_clock(t)
    fpk = fma_peak_tflops(wb.sms, mhz)
    hbm = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
           "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
           "alg_bytes_per_launch": bpl, "frac_of_8TBps": gbs / 8000.0}
    alu = {"bound": "alu", "achieved": tfs, "peak": fpk, "unit": "TFLOP/s", "frac": tfs / fpk,
           "peak_source": (f"fp32 FMA peak of the CUDA cores: {wb.sms} SMs x 128 FMA/clk x 2 flops "
                           f"x {mhz:.0f} MHz (median SM clock sampled in the timed region)"),
           "alg_flops_per_launch": fpl}
    main, other = (alu, hbm) if alu["frac"] > hbm["frac"] else (hbm, alu)
    out = dict(main)
    out["traffic"] = traffic
    out["kernel"] = "decode_kernel (kivi_decode_attn / kivi_append_decode)"
    out["other_bound"] = other
    return out


def summarize(wb, t, steps, world, peak):
    """Per-workload figures from a Workbench measurement."""
    w = wb.w
    launches = sum(n for _, n in t["runs"])
    dec_total = sum(ms for ms, _ in t["runs"])
    dec_avg = dec_total / launches
    pre_avg = sum(t["pre_ms"]) / len(t["pre_ms"])
    bpl = wb.bytes_step / wb.n_dec
    achieved = bpl / (dec_avg / 1e3) / 1e9
    fpl = wb.flops_step / wb.n_dec
    tfs = fpl / (dec_avg / 1e3) / 1e12
    fpk = fma_peak_tflops(wb.sms, sm_clock(t))
    pb = prefill_bytes(w)
    return {
        "value": world * wb.units_step * steps / (t["ms"] / 1e3), "unit": UNIT,
        "ms_per_step": t["ms"] / steps, "steps": steps,
        "decode": {"avg_us": 1e3 * dec_avg,
                   "timing": "CUDA events around each run of back-to-back decode launches",
                   "runs_timed": len(t["runs"]), "launches_timed": launches,
                   "alg_bytes_per_launch": bpl,
                   "achieved_gbs": achieved, "frac_of_measured_hbm": achieved / peak,
                   "frac_of_8TBps": achieved / 8000.0,
                   "alg_flops_per_launch": fpl, "achieved_tflops": tfs,
                   "frac_of_fma_peak": tfs / fpk,
                   "tokens_heads_per_s": wb.units_step / wb.n_dec / (dec_avg / 1e3),
                   "gpu_time_share": dec_total / t["ms"]},
        "prefill": {"avg_us": 1e3 * pre_avg, "alg_bytes": pb,
                    "achieved_gbs": pb / (pre_avg / 1e3) / 1e9,
                    "frac_of_measured_hbm": pb / (pre_avg / 1e3) / 1e9 / peak,
                    "launches_timed": len(t["pre_ms"])},
        "clocks": t["clocks"],
    }


def graph_decode(wb, steps, warmup):
    """One decode per layer cache (the caches as the last step left them),
    captured once into a CUDA graph and replayed: the launch overhead of the
    whole stack amortised.  Device time per replay (CUDA events)."""
    import torch
    w, L = wb.w, wb.L
    qp = [row[l % wb.sets][2] for row in wb.Sp[:1] for l in range(wb.nl)]
    s = torch.cuda.Stream(wb.dev)
    s.wait_stream(wb.stream)
    sp = ctypes.c_void_p(s.cuda_stream)

    def run():
        bad = 0
        for l in range(wb.nl):
            bad |= L.kivi_decode_attn(wb.H[l], qp[l], w.H_q, wb.Op[l], sp)
        if bad:
            raise RuntimeError("a KIVI call failed during graph capture")

    with torch.cuda.stream(s):
        run()
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize(wb.dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        g.replay()
    b.record()
    torch.cuda.synchronize(wb.dev)
    ms = a.elapsed_time(b) / steps
    n_q, r, _ = wb.calls[0]
    per = decode_bytes(w, n_q, r)
    del g
    return {"layers": wb.nl, "us_per_replay": 1e3 * ms, "us_per_layer": 1e3 * ms / wb.nl,
            "achieved_gbs": per * wb.nl / (ms / 1e3) / 1e9, "launches_per_replay": wb.nl}


def per_config_entry(args, name, dev, peak):
    """Measure one of the other workloads at full size (rank 0, N = 1)."""
    import torch
    w = get_workload(args, name)
    layers, sets = LAYERS[name], INPUT_SETS.get(name, LAYERS[name])
    wb = Workbench(w, layers, sets, 0, dev)
    try:
        t = wb.measure(args.steps, args.warmup)
        s = summarize(wb, t, args.steps, 1, peak)
        s["config"] = workload_config(w, args, layers, 1, sets)
        s["gpu_launches"] = wb.launches_step * args.steps
        tr = traffic_per_launch(w, True)
        s["decode"]["traffic"] = tr
        if name == "llama2_13b_cache":
            s["decode_graph"] = graph_decode(wb, args.steps, args.warmup)
            nb = wb.caches[0].nbytes()
            per_tok = lambda x: x * layers / (w.B * w.T)
            rec, meta = cache_record_bytes(w, layers)
            s["cache_bytes"] = {
                "codes_plus_residual_per_token": per_tok(nb["codes"] + nb["residual"]),
                "metadata_per_token": per_tok(nb["meta"]),
                "record_per_token": 128000, "record_basis_closed_form": rec,
                "matches_record": per_tok(nb["codes"] + nb["residual"]) == 128000 == rec,
                "source": "kivi_cache_bytes of the allocated caches (capacity 4,096 tokens)"}
        return s
    finally:
        wb.close()
        del wb
        torch.cuda.empty_cache()


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from bit_asymmetric_kv_prefill_b200 import build as kbuild
    kbuild.build()

    w = get_workload(args)
    layers = args.layers or LAYERS[w.name]
    sets = min(INPUT_SETS.get(w.name, layers), layers)
    peak, peak_kind = measured_peak()
    wb = Workbench(w, layers, sets, rank, dev)
    t = wb.measure(args.steps, args.warmup)
    ms = reduce_max(t["ms"], dev)
    dec_avg = reduce_max(sum(ms_ for ms_, _ in t["runs"]) / sum(n for _, n in t["runs"]), dev)
    t["ms"] = ms
    s = summarize(wb, t, args.steps, world, peak)
    roof = roofline(wb, dec_avg, t, peak, peak_kind,
                    traffic_per_launch(w, not (args.batch or args.decode_steps)))
    e2e = run_e2e(args, wb, world) if sets == layers else None
    launches = wb.launches_step * args.steps
    wb.close()
    del wb
    torch.cuda.empty_cache()

    per_config, cpu = None, None
    if world == 1 and is_headline(args) and not args.no_per_config:
        per_config = {name: per_config_entry(args, name, dev, peak) for name in PER_CONFIG}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": s["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
            "data": "synthetic", "config": workload_config(w, args, layers, world, sets),
            "roofline": roof,
            "decode_attn": s["decode"], "prefill": s["prefill"],
            "e2e": e2e, "gpu_launches": launches, "clocks": s["clocks"],
            "cpu_baseline": cpu, "per_config": per_config,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, wb, world):
    """Same step through the public API with pinned HOST inputs: the H2D copies
    of every input and the D2H read of every decode output are timed.

    Copies run on their own streams, as a serving loop would run them: step
    k+1's prefill inputs stream in while step k computes (each layer's buffer
    is refilled once that layer's prefill has read it), and each step's decode
    inputs land in one of two buffer sets; every decode's output goes back to
    the host on a third stream.  Every timed step's copies happen inside the
    timed region (the first step's with nothing to overlap them)."""
    import torch
    w, dev, nl, caches = wb.w, wb.dev, wb.nl, wb.caches
    Ks, Vs, steps = wb.Ks, wb.Vs, [[row[l] for l in range(nl)] for row in wb.steps]
    def pinned(t):   # a pinned host copy, with no pageable copy in between
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    hK = [pinned(k) for k in Ks]
    hV = [pinned(v) for v in Vs]
    hS = [[tuple(pinned(t) for t in st) for st in row] for row in steps]
    dK = [torch.empty_like(Ks[0]) for _ in range(nl)]
    dV = [torch.empty_like(Vs[0]) for _ in range(nl)]
    dS = [[[tuple(torch.empty_like(t) for t in steps[0][0]) for _ in range(nl)] for _ in hS]
          for _ in range(2)]
    hout = [torch.empty(w.B, w.H_q, w.D, dtype=torch.float32).pin_memory() for _ in range(nl)]
    cs = torch.cuda.current_stream(dev)
    xs = torch.cuda.Stream(dev)
    xs2 = torch.cuda.Stream(dev)  # values on a second copy engine
    ds = torch.cuda.Stream(dev)   # outputs back to the host, off the compute stream
    ev_in = [torch.cuda.Event() for _ in range(nl)]
    ev_in2 = [torch.cuda.Event() for _ in range(nl)]
    ev_used = [torch.cuda.Event() for _ in range(nl)]
    ev_sin = [torch.cuda.Event() for _ in range(2)]
    ev_sused = [torch.cuda.Event() for _ in range(2)]
    for e in ev_used + ev_sused:
        e.record(cs)
    kinds = [kind for _, _, kind in wb.calls]

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
                if kinds[j] == "none":
                    out = caches[l].decode(q)
                else:
                    out = caches[l].append_decode(k_t, v_t, q)
                ds.wait_stream(cs)
                with torch.cuda.stream(ds):
                    hout[l].copy_(out, non_blocking=True)
                out.record_stream(ds)
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
    cs.wait_stream(ds)   # the last outputs are on the host
    b.record(cs)
    torch.cuda.synchronize(dev)
    barrier(dev)
    ms = reduce_max(a.elapsed_time(b), dev)
    units = wb.units_step
    h2d = nl * (2 * Ks[0].numel() * 2 + len(hS) * sum(t.numel() * 2 for t in steps[0][0]))
    d2h = nl * len(hS) * w.B * w.H_q * w.D * 4
    return {"value": world * units * n / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n, "ms_per_step": ms / n,
            "copies": "H2D on two copy streams (keys, values), step k+1's inputs during step k; "
                      "outputs D2H on a third stream; the first step's inputs are copied inside the "
                      "timed region with nothing to overlap"}


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
    # Non-uniform levels (KVQuant's non-uniform quantization): four levels
    # fitted by Lloyd's algorithm on a few matrices of the same cache (keys per
    # channel, values per token), timed like the modes above.
    from oracle import diag as odiag
    nuq = {}
    for which, axis in (("K", 0), ("V", 1)):
        Xs = (K if which == "K" else V).reshape(N, T, D)
        lev = odiag.fit_levels(Xs[:2].float().cpu().numpy(), axis, 32, 4)
        levc = (ctypes.c_double * 4)(*[float(v) for v in lev])
        run = lambda: L.kivi_fake_quant_levels(src[which], dt, N, T, D, axis, 32, 4, levc, xhp, None,
                                               errp, sp)
        for _ in range(args.warmup):
            if run():
                raise RuntimeError("kivi_fake_quant_levels failed")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            run()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        us = 1e3 * e0.elapsed_time(e1) / args.steps
        nuq[f"{which}_us"] = us
        nuq[f"{which}_gbs"] = elems * 6 / (us / 1e6) / 1e9
        nuq[f"{which}_rel_err"] = (float(err.sum()) / norms[which]) ** 0.5
        nuq[f"{which}_levels"] = [float(v) for v in lev]
    modes["nonuniform_levels_4"] = nuq
    launches = len(plan) * args.steps + 2 * args.steps
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kivi", "reference"], default="kivi")
    ap.add_argument("--layers", type=int, default=0,
                    help="layer caches per step (default: the workload's own count)")
    ap.add_argument("--e2e-steps", dest="e2e_steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", dest="cpu_seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", dest="no_cpu_baseline", action="store_true")
    ap.add_argument("--no-per-config", dest="no_per_config", action="store_true",
                    help="skip the other workloads' measurements")
    ap.add_argument("--workload", default=WORKLOAD, choices=WORKLOAD_NAMES)
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
