"""Benchmark: QJL key quantization + compressed-key decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa|long|prefill|single|sweep-m<M>-d<D>|paged-gqa|dequant-gqa|search|turbo-gqa|
                turbo-paged-gqa|turbo-dequant-gqa|turbo-gqa-d64]

A step is one pass of the whole hot path over one batch of the workload:
quantize every key of the batch (sign code + fp16 norm, jl_quantize_keys) and
run one decode step of attention over the compressed cache
(jl_decode_attention: query projection, scorer, combine).  The default
workload is GQA decode: batch 8, 32 query / 8 KV heads, d=128, m=256, context
32768.  Inputs are seeded synthetic tensors (workloads.py) already resident
in HBM; they exceed L2 (126 MB), so no flush is needed between steps.

The paged-gqa workload times a serving step instead: one
jl_decode_attention_paged call that appends every sequence's new key and
value to a shuffled page pool and attends over its ragged context (the cache
is filled once, untimed; the lengths stay fixed from step to step, so every
step rewrites the same slots).

The search workload times one jl_search_topk call: the top-10 index vectors
of each of 128 queries over 8,388,608 compressed vectors (scores on the
tensor cores; the roofline is the tensor peak).

The turbo-gqa workload times the TurboQuant-prod step on the gqa cache:
jl_turbo_quantize_keys over every key (rotation product and residual sketch on
the tensor cores) and one jl_turbo_decode_attention call.

The dequant-gqa workload times the explicit dequantizer: one
jl_dequantize_keys call turning the gqa cache's codes and norms back into
bf16 keys.  turbo-dequant-gqa does the same for the turbo-gqa cache's
TurboQuant-prod codes (one jl_turbo_dequantize_keys call; the reconstruction
matrix is built once, untimed).

Multi-GPU (torchrun): every rank runs its own batch of the same workload
(independent sequences, no data-path collective), timing is the max over ranks
and ``value`` counts the keys of all ranks ("scaling": "weak").

The timed region records CUDA events only at its two ends: an event between
two kernels makes the second wait for the first to drain, which would cut the
programmatic-dependent-launch overlap the library relies on.  Per-phase
durations come from each phase run alone, K calls back to back, right after
the timed steps (still under the clock sampler).

The JSON line also carries: those per-phase timings, the roofline of the
dominant kernel (algorithmic bytes / measured duration against the measured
HBM copy bandwidth), the end-to-end number through the Python binding with
pinned host buffers (H2D copies of the step's inputs and D2H of its output
inside the timed region), SM clocks sampled during the timed region, and the
float64 oracle timed on a bounded sample on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------
# helpers

FALLBACK_BF16_TFLOPS = 1590.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def load_tensor_peak():
    """Dense bf16 tensor peak (burst figure: the kernel is timed alone)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured bf16_tflops (fp16 runs at the bf16 rate)"
    return FALLBACK_BF16_TFLOPS, "fallback bf16 TFLOP/s"


def pick_workload(name: str, batch: int = 0) -> workloads.Workload:
    w = _pick(name)
    return w.with_(B=batch) if batch else w


def rank_workload(args, rank: int) -> workloads.Workload:
    """This rank's batch: sequences [rank*B, (rank+1)*B) of the global batch
    (every rank holds B sequences of its own; weak scaling)."""
    return workloads.shard(pick_workload(args.workload, args.batch), rank)


def _pick(name: str) -> workloads.Workload:
    if name == "long-cp":
        # the long workload, its context split across the ranks
        return workloads.ALL["long"]
    if name.startswith("sweep-"):
        # sweep-m<M>-d<D>
        m = int(name.split("-m")[1].split("-")[0])
        d = int(name.split("-d")[1])
        return workloads.SWEEP_BASE.with_(m=m, d=d)
    return workloads.ALL[name]


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "bit_jl_key_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e:
        return None
    if e.get("source_hash") != kernel_source_hash(e["sources"]):
        return None
    return e


class ClockSampler:
    """SM clock, power and throttle-reason samples for the timed region, read
    by a thread: from NVML every 5 ms (nvidia-smi every 100 ms where NVML
    cannot be loaded).  Reading only: nothing is set.  ``region_start`` /
    ``region_end`` bracket the region (host times taken after a device
    synchronize on both sides, so they bound the device's work).  A region
    shorter than a few sampling intervals holds few samples of its own;
    ``region_end(top_up=fn)`` then keeps the GPU under the same load, running
    fn (one untimed step) until the region and its continuation hold
    ``min_samples``.  The summary says how many samples fell inside the
    region and how many in the continuation."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    # NVML clocks-event reason bits -> the names above
    NVML_BITS = ((0x8, "hw_slowdown"), (0x80, "hw_slowdown"), (0x40, "hw_thermal_slowdown"),
                 (0x20, "sw_thermal_slowdown"), (0x4, "sw_power_cap"))

    def __init__(self, gpu_index: int, min_samples: int = 3):
        self.gpu_index = gpu_index
        self.min_samples = min_samples
        self.proc = None
        self.nvml = None
        self.samples = []          # (host time, (sm MHz, max sm MHz, power W, reasons))
        self.lock = threading.Lock()
        self.stop = threading.Event()
        self.thread = None
        self.source = None
        self.interval_ms = None
        self.t0 = self.t1 = None
        self.t_end = None
        self.power_limit = None

    def feed(self, line: str, t=None):
        """Parse one nvidia-smi CSV line (ignored when malformed)."""
        c = [x.strip() for x in line.split(",")]
        if len(c) < 9:
            return
        try:
            smp = (float(c[1]), float(c[2]), float(c[3]),
                   [n for n, v in zip(self.NAMES, c[5:9]) if v.lower().startswith("active")])
        except ValueError:
            return
        with self.lock:
            self.samples.append((time.monotonic() if t is None else t, smp))

    def _smi_reader(self):
        for line in self.proc.stdout:
            self.feed(line)

    def _nvml_poller(self, h, max_mhz):
        nv = self.nvml
        while not self.stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                try:
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except AttributeError:
                    bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                reasons = sorted({n for b, n in self.NVML_BITS if bits & b})
                with self.lock:
                    self.samples.append((time.monotonic(), (mhz, max_mhz, watts, reasons)))
            except Exception:  # noqa: BLE001 -- a failed read is a missing sample
                pass
            self.stop.wait(0.005)

    def _device_uuid(self):
        try:
            u = str(torch.cuda.get_device_properties(self.gpu_index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:  # noqa: BLE001
            return None

    def _start_nvml(self) -> bool:
        try:
            import pynvml as nv
            nv.nvmlInit()
        except Exception:  # noqa: BLE001
            return False
        self.nvml = nv
        try:
            uuid = self._device_uuid()
            h = (nv.nvmlDeviceGetHandleByUUID(uuid) if uuid
                 else nv.nvmlDeviceGetHandleByIndex(self.gpu_index))
            max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            try:
                self.power_limit = (nv.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0,
                                    nv.nvmlDeviceGetPowerManagementLimitConstraints(h)[1] / 1000.0)
            except Exception:  # noqa: BLE001
                self.power_limit = None
        except Exception:  # noqa: BLE001
            nv.nvmlShutdown()
            self.nvml = None
            return False
        self.source, self.interval_ms = "nvml", 5
        self.min_samples = max(self.min_samples, 10)
        self.thread = threading.Thread(target=self._nvml_poller, args=(h, max_mhz), daemon=True)
        self.thread.start()
        return True

    def _start_smi(self):
        uuid = self._device_uuid()
        gid = uuid or str(self.gpu_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        try:
            q = subprocess.run(["nvidia-smi", f"--id={gid}",
                                "--query-gpu=enforced.power.limit,power.max_limit",
                                "--format=csv,noheader,nounits"],
                               capture_output=True, text=True, timeout=10)
            lim = [x.strip() for x in q.stdout.strip().split(",")]
            self.power_limit = (float(lim[0]), float(lim[1]))
        except (OSError, ValueError, IndexError, subprocess.SubprocessError):
            self.power_limit = None
        self.source, self.interval_ms = "nvidia-smi", 100
        self.thread = threading.Thread(target=self._smi_reader, daemon=True)
        self.thread.start()

    def __enter__(self):
        if not self._start_nvml():
            self._start_smi()
        deadline = time.monotonic() + 5.0      # the first sample has arrived
        while self.thread is not None and time.monotonic() < deadline \
                and not self._count(0.0, None):
            time.sleep(0.01)
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass

    def _count(self, t_from, t_to):
        with self.lock:
            return sum(1 for t, _ in self.samples if t >= t_from and (t_to is None or t <= t_to))

    def region_start(self):
        self.t0 = time.monotonic()
        self.t1 = self.t_end = None

    def region_end(self, top_up=None, max_s=3.0):
        self.t1 = time.monotonic()
        self.t_end = self.t1
        if top_up is not None:
            self.extend(top_up, max_s)

    def extend(self, top_up, max_s=3.0):
        """Keep sampling, running top_up() (the same step, untimed), until the
        region and everything since hold min_samples samples."""
        if self.thread is not None:
            stop = time.monotonic() + max_s
            while self._count(self.t0, None) < self.min_samples and time.monotonic() < stop:
                top_up()
                torch.cuda.synchronize()
        self.t_end = time.monotonic()

    def summary(self):
        with self.lock:
            samples = list(self.samples)
        if self.t0 is not None:
            t1 = self.t1 if self.t1 is not None else float("inf")
            t_end = self.t_end if self.t_end is not None else t1
            inside = [x for t, x in samples if self.t0 <= t <= t1]
            after = [x for t, x in samples if t1 < t <= t_end]
        else:
            inside, after = [x for _, x in samples], []
        used = inside + after
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        reasons = sorted({n for x in used for n in x[3]})
        rec = {"sm_mhz": statistics.median(x[0] for x in used),
               "sm_max_mhz": max(x[1] for x in used), "reasons": reasons,
               "samples": len(used), "samples_in_region": len(inside),
               "samples_same_load_after": len(after), "source": self.source,
               "interval_ms": self.interval_ms,
               "power_w_max": max(x[2] for x in used),
               "power_limit_w": self.power_limit[0] if self.power_limit else None,
               "power_max_limit_w": self.power_limit[1] if self.power_limit else None}
        if inside:
            rec["sm_mhz_in_region"] = statistics.median(x[0] for x in inside)
        return rec


def reduce_max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank time over all ranks (the only collective the bench
    uses; the data path has none)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms_max: float) -> float:
    """Units of all ranks over the slowest rank's time (weak scaling)."""
    return units_per_rank * world / (ms_max * 1e-3)


# --------------------------------------------------------------------------
# algorithmic bytes

def quantize_bytes(w, n_keys):
    """Read the keys, write codes + fp16 norms (the sketch is 64 KB, L2)."""
    kb = 2 if w.key_dtype == torch.bfloat16 else 4
    return n_keys * (w.d * kb + w.m // 8 + 2)


def decode_bytes(w):
    """Per KV key: code (m/8 B) + fp16 norm (2 B) + bf16 value row (2d B)."""
    return w.B * w.Hkv * w.T * (w.m // 8 + 2 + 2 * w.d)


def reconstruction_error(jl, w, S, signs, norms, K, rows=65536):
    """Measured D_mse of the dequantizer on the first rows of the cache:
    mean over keys of ||k - khat||^2 / ||k||^2, beside the closed form
    ((pi/2) d - 1) / m for a Gaussian sketch.  Measurement only."""
    n = min(rows, signs.shape[0])
    khat = jl.jl_dequantize_keys(signs[:n], norms[:n], S).float()
    k = K.reshape(-1, w.d)[:n].float()
    rel = ((khat - k) ** 2).sum(1) / (k * k).sum(1)
    return {"mean_rel_sq_error": float(rel.mean()),
            "predicted": (math.pi / 2 * w.d - 1) / w.m, "samples": n}


def score_error(jl, w, Q, S, signs, norms, V, K, max_rows=16):
    """Normalised error of the GPU estimator against the exact inner product
    on sampled (b, query head) rows: rms over keys of (s - <q,k>) / (|q||k|),
    next to the closed form sqrt((pi/2 - 1/d) / m) of the estimator's variance
    for independent Gaussian q, k.  Measurement only (exact products by a
    plain fp32 matmul of the stored bf16 values)."""
    out, sc = jl.jl_decode_attention(Q, S, signs, norms, V,
                                     softmax_scale=w.softmax_scale, want_scores=True)
    rows = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    step = max(1, len(rows) // max_rows)
    errs = []
    for (b, h) in rows[::step][:max_rows]:
        q = Q[b, h].float()
        k = K[b, h // w.G].float()
        exact = k @ q
        denom = k.norm(dim=1) * q.norm()
        errs.append(((sc[b, h] - exact) / denom).double())
    e = torch.cat(errs)
    return {"rms_normalised": float(torch.sqrt(torch.mean(e * e))),
            "predicted": math.sqrt((math.pi / 2 - 1.0 / w.d) / w.m),
            "bits_per_key": w.m + 16, "bits_per_coordinate": (w.m + 16) / w.d,
            "samples": int(e.numel())}


# --------------------------------------------------------------------------
# our arm

def _barrier(world, dev):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)


def run_paged(args, rank, world, local_rank):
    """Serving step over a paged cache: append + decode in one call (QJL keys,
    or TurboQuant-prod keys for turbo-paged-gqa)."""
    import bit_jl_key_b200 as jl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args, rank)
    turbo = w.name.startswith("turbo")
    bits = workloads.TURBO_MSE_BITS
    peak, peak_kind = load_peaks()
    P = workloads.PAGE_TOKENS
    lens, table, num_pages = workloads.paged_layout(w, P)
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    # fill the pool (untimed): keys and values of every slot, quantized in place
    # pages of this rank's pool, seeded apart from every other rank's pool
    pool = w.with_(B=num_pages, T=P, first_seq=rank * (w.B * -(-w.T // P) + 16))
    Kp = workloads.keys(pool, dev)
    if turbo:
        Pi, Pinv = jl.jl_turbo_rotation_init(w.d, workloads.TURBO_ROTATION_SEED, device=dev)
        words = jl.turbo_code_words(bits, w.m, w.d)
        sign_pages = torch.empty((num_pages, w.Hkv, P, words), dtype=torch.int32, device=dev)
        norm_pages = torch.empty((num_pages, w.Hkv, P, 2), dtype=torch.float16, device=dev)
        jl.jl_turbo_quantize_keys(Kp.view(-1, w.d), Pi, S, bits, codes=sign_pages.view(-1, words),
                                  norms=norm_pages.view(-1, 2))
    else:
        words = w.m // 32
        sign_pages = torch.empty((num_pages, w.Hkv, P, words), dtype=torch.int32, device=dev)
        norm_pages = torch.empty((num_pages, w.Hkv, P), dtype=torch.float16, device=dev)
        jl.jl_quantize_keys(Kp.view(-1, w.d), S, sign_pages.view(-1, words), norm_pages.view(-1))
    del Kp
    value_pages = workloads.values(pool, dev)
    Q = workloads.queries(w, dev)
    Kn, Vn = workloads.new_tokens(w, dev)
    seq = lens.to(dev)
    tab = table.to(dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    wsb = (jl.jl_turbo_decode_paged_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.m, w.d, bits)
           if turbo else jl.jl_decode_paged_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.m, w.d))
    ws = torch.empty((wsb,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    attended = int((lens.long() + 1).sum()) * w.Hkv     # KV keys scored per step

    def step():
        if turbo:
            jl.jl_turbo_decode_attention_paged(Q, Pinv, S, sign_pages, norm_pages, value_pages,
                                               tab, seq, w.T, bits, Pi=Pi, K_new=Kn, V_new=Vn,
                                               softmax_scale=w.softmax_scale, out=out,
                                               workspace=ws)
        else:
            jl.jl_decode_attention_paged(Q, S, sign_pages, norm_pages, value_pages, tab, seq,
                                         w.T, K_new=Kn, V_new=Vn, softmax_scale=w.softmax_scale,
                                         out=out, workspace=ws)

    for _ in range(args.warmup):
        step()
    _barrier(world, dev)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error after warm-up")
    # events only around the whole run: an event between two calls would make
    # each call wait for the previous one to drain (no overlap of the next
    # call's first kernel with the previous call's last)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        _barrier(world, dev)
        clk.region_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        _barrier(world, dev)
        clk.region_end(top_up=step)
    ms_step = reduce_max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    d_ms = ms_step
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error in the timed region")

    # end to end: the step's new query, key and value (and the lengths) from
    # pinned host memory, the output back to it; the cache stays resident
    e2e = None
    if not args.no_e2e:
        hQ, hK, hV = (t.cpu().pin_memory() for t in (Q, Kn, Vn))
        hL = lens.clone().pin_memory()
        hOut = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hQ, hK, hV, hL))
        d2h = hOut.numel() * hOut.element_size()

        def e2e_step():
            Q.copy_(hQ, non_blocking=True)
            Kn.copy_(hK, non_blocking=True)
            Vn.copy_(hV, non_blocking=True)
            seq.copy_(hL, non_blocking=True)
            step()
            hOut.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        _barrier(world, dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        _barrier(world, dev)
        e_ms = reduce_max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
        e2e = {"value": whole_job_rate(attended, world, e_ms), "unit": "keys/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    per_key = (words * 4 + 4 if turbo else w.m // 8 + 2) + 2 * w.d
    db = attended * per_key
    gbs = db / (d_ms * 1e-3) / 1e9
    traffic = ncu_traffic("decode:" + w.name)
    phases = {"decode": {"ms": d_ms, "keys_scored_per_s": attended / (d_ms * 1e-3),
                         "head_key_pairs_per_s": attended * w.G / (d_ms * 1e-3),
                         "algorithmic_bytes": db, "GB_per_s": gbs,
                         "frac_of_hbm_peak": gbs / peak,
                         "appended_keys": w.B * w.Hkv}}
    roof = {"kernel": "jl_turbo_decode_attention_paged" if turbo else "jl_decode_attention_paged",
            "bound": "hbm", "achieved": gbs,
            "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
            "frac": gbs / peak, "algorithmic_bytes_per_launch": db,
            "traffic": traffic["dram_bytes_per_launch"] if traffic else None}
    return {
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": whole_job_rate(attended, world, ms_step), "unit": "keys/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} max_len={w.T} "
                               f"d={w.d} m={w.m} page={P} lens={lens.tolist()} + 1 appended"
                               + (f", {bits}-bit cells + 1-bit residual QJL" if turbo else ""),
                   "global_batch": w.B * world, "seq_len": w.T,
                   "parallelism": f"dp{world}",
                   "l2": "cache exceeds L2 (126 MB); no flush"},
        "phases": phases,
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }


def turbo_reconstruction_error(jl, w, codes, norms, R, bits, K, rows=65536):
    """Measured reconstruction error of the TurboQuant-prod dequantizer on the
    first rows of the cache, mean over keys of ||k - khat||^2, beside the QJL
    error of the residual, mean of ||k||^2 ||r||^2 ((pi/2) d - 1) / m (its
    expectation over Gaussian sketches).  Measurement only."""
    n = min(rows, codes.shape[0])
    khat = jl.jl_turbo_dequantize_keys(codes[:n], norms[:n], R, bits).double()
    k = K.reshape(-1, w.d)[:n].double()
    meas = ((khat - k) ** 2).sum(1)
    nk = norms[:n, 0].double()
    nr = norms[:n, 1].double()
    pred = (nk * nr) ** 2 * ((math.pi / 2) * w.d - 1) / w.m
    return {"mean_sq_error": float(meas.mean()), "predicted": float(pred.mean()),
            "mean_rel_sq_error": float((meas / (k * k).sum(1)).mean()), "samples": n}


def run_dequant(args, rank, world, local_rank):
    """Explicit dequantizer over a cache's codes: khat in bf16 (QJL codes of
    the gqa cache, or TurboQuant-prod codes of the turbo-gqa cache)."""
    import bit_jl_key_b200 as jl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args, rank)
    turbo = w.name == "turbo-dequant-gqa"
    peak, peak_kind = load_peaks()
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    K = workloads.keys(w, dev)
    if turbo:                                                   # untimed set-up
        bits = workloads.TURBO_MSE_BITS
        Pi, Pinv = jl.jl_turbo_rotation_init(w.d, workloads.TURBO_ROTATION_SEED, device=dev)
        signs, norms = jl.jl_turbo_quantize_keys(K.view(-1, w.d), Pi, S, bits)
        R = jl.jl_turbo_dequant_basis(Pinv, S)
        recon = (None if args.no_score_error
                 else turbo_reconstruction_error(jl, w, signs, norms, R, bits, K))
        code_bytes = (bits * w.d + w.m) // 8 + 4
        kdim = w.d + w.m
        api = "jl_turbo_dequantize_keys"
    else:
        signs, norms = jl.jl_quantize_keys(K.view(-1, w.d), S)
        recon = None if args.no_score_error else reconstruction_error(jl, w, S, signs, norms, K)
        code_bytes = w.m // 8 + 2
        kdim = w.m
        api = "jl_dequantize_keys"
    del K
    torch.cuda.empty_cache()
    n = signs.shape[0]
    out = torch.empty((n, w.d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if turbo:
            jl.jl_turbo_dequantize_keys(signs, norms, R, bits, out=out)
        else:
            jl.jl_dequantize_keys(signs, norms, S, out=out)

    for _ in range(args.warmup):
        step()
    _barrier(world, dev)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error after warm-up")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        _barrier(world, dev)
        clk.region_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        _barrier(world, dev)
        clk.region_end(top_up=step)
    ms = reduce_max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error in the timed region")

    e2e = None
    if not args.no_e2e:
        hS = signs.cpu().pin_memory()
        hN = norms.cpu().pin_memory()
        hOut = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            signs.copy_(hS, non_blocking=True)
            norms.copy_(hN, non_blocking=True)
            step()
            hOut.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        _barrier(world, dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e_steps = max(3, args.steps // 4)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        _barrier(world, dev)
        e_ms = reduce_max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)
        e2e = {"value": whole_job_rate(n, world, e_ms), "unit": "keys/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": hS.numel() * 4 + hN.numel() * 2,
               "d2h_bytes_per_step": hOut.numel() * 2}

    nbytes = n * (code_bytes + 2 * w.d)
    gbs = nbytes / (ms * 1e-3) / 1e9
    traffic = ncu_traffic("dequant:" + w.name)
    return {
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": whole_job_rate(n, world, ms), "unit": "keys/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": (f"{w.name}: {n} codes, m={w.m}, d={w.d}"
                                + (f", {bits}-bit cells" if turbo else "") + " -> bf16 keys"),
                   "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
                   "l2": "inputs and outputs exceed L2 (126 MB); no flush"},
        "phases": {"dequantize": {"ms": ms, "keys_per_s": n / (ms * 1e-3),
                                  "algorithmic_bytes": nbytes, "GB_per_s": gbs,
                                  "frac_of_hbm_peak": gbs / peak,
                                  "tflops": n * 2 * kdim * w.d / (ms * 1e-3) / 1e12}},
        "roofline": {"kernel": api, "bound": "hbm", "achieved": gbs,
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": gbs / peak, "algorithmic_bytes_per_launch": nbytes,
                     "traffic": traffic["dram_bytes_per_launch"] if traffic else None},
        "reconstruction_error": recon,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }


def search_launches_per_call(N, nq, sms=148):
    """Kernels one jl_search_topk call launches: per pass of 128 queries the
    query projection, the warm-start sample pass and its merge (when the
    index has at least eight tiles of 256 per CTA), the full pass and the
    final merge."""
    tiles = -(-N // 256)
    grid = min(sms, tiles)
    per_pass = 3 + (2 if tiles // (grid * 4) >= 2 else 0)
    return per_pass * -(-nq // 128)


def run_search(args, rank, world, local_rank):
    """Top-k inner-product search over a compressed index."""
    import bit_jl_key_b200 as jl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args, rank)
    k = workloads.SEARCH_K
    hbm_peak, _ = load_peaks()
    tpeak, tkind = load_tensor_peak()
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    K = workloads.keys(w, dev)                                    # index vectors, untimed
    signs, norms = jl.jl_quantize_keys(K.view(-1, w.d), S)
    del K
    torch.cuda.empty_cache()
    Q = workloads.queries(w, dev).view(-1, w.d)
    N, nq = signs.shape[0], Q.shape[0]
    ws = torch.empty((jl.jl_search_workspace_bytes(nq, w.m, w.d, k),), dtype=torch.uint8,
                     device=dev)
    oi = torch.empty((nq, k), dtype=torch.int32, device=dev)
    osc = torch.empty((nq, k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        jl.jl_search_topk(Q, S, signs, norms, k, out_index=oi, out_scores=osc, workspace=ws)

    for _ in range(args.warmup):
        step()
    _barrier(world, dev)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error after warm-up")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        _barrier(world, dev)
        clk.region_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        _barrier(world, dev)
        clk.region_end(top_up=step)
    ms = reduce_max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error in the timed region")

    e2e = None
    if not args.no_e2e:
        # the queries from pinned host memory, the top-k lists back to it
        hQ = Q.cpu().pin_memory()
        hI = torch.empty(oi.shape, dtype=oi.dtype).pin_memory()
        hS = torch.empty(osc.shape, dtype=osc.dtype).pin_memory()

        def e2e_step():
            Q.copy_(hQ, non_blocking=True)
            step()
            hI.copy_(oi, non_blocking=True)
            hS.copy_(osc, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        _barrier(world, dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        _barrier(world, dev)
        e_ms = reduce_max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
        e2e = {"value": whole_job_rate(N * nq, world, e_ms), "unit": "query-vector pairs/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": hQ.numel() * hQ.element_size(),
               "d2h_bytes_per_step": hI.numel() * 4 + hS.numel() * 4}

    flops = 2.0 * w.m * N * nq                 # the estimator's m multiply-adds per pair
    tflops = flops / (ms * 1e-3) / 1e12
    nbytes = N * (w.m // 8 + 2)
    return {
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": whole_job_rate(N * nq, world, ms), "unit": "query-vector pairs/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": f"{w.name}: {nq} queries x {N} vectors, d={w.d}, m={w.m}, "
                               f"top-{k}",
                   "global_batch": nq * world, "seq_len": N, "parallelism": f"dp{world}",
                   "l2": "index (285 MB of codes and norms) exceeds L2; no flush"},
        "phases": {"search": {"ms": ms, "pairs_per_s": N * nq / (ms * 1e-3),
                              "tflops": tflops, "frac_of_tensor_peak": tflops / tpeak,
                              "index_bytes": nbytes,
                              "index_GB_per_s": nbytes / (ms * 1e-3) / 1e9,
                              "frac_of_hbm_peak": nbytes / (ms * 1e-3) / 1e9 / hbm_peak}},
        "roofline": {"kernel": "jl_search_topk", "bound": "tensor", "achieved": tflops,
                     "peak": tpeak, "peak_kind": tkind, "unit": "TFLOP/s",
                     "frac": tflops / tpeak, "algorithmic_flops_per_launch": flops,
                     "traffic": None},
        "e2e": e2e,
        "gpu_launches": search_launches_per_call(
            N, nq, torch.cuda.get_device_properties(dev).multi_processor_count) * args.steps,
        "clocks": clk.summary(),
    }


def run_turbo(args, rank, world, local_rank):
    """TurboQuant-prod step over the turbo-gqa cache: quantize every key
    (rotation product, cells, residual QJL) and one decode step over the
    cell-plane codes."""
    import bit_jl_key_b200 as jl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args, rank)
    bits = workloads.TURBO_MSE_BITS
    peak, peak_kind = load_peaks()
    Pi, Pinv = jl.jl_turbo_rotation_init(w.d, workloads.TURBO_ROTATION_SEED, device=dev)
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    K = workloads.keys(w, dev)
    Kf = K.view(-1, w.d)
    n_keys = Kf.shape[0]
    words = jl.turbo_code_words(bits, w.m, w.d)
    codes = torch.empty((n_keys, words), dtype=torch.int32, device=dev)
    norms = torch.empty((n_keys, 2), dtype=torch.float16, device=dev)
    V = workloads.values(w, dev)
    Q = workloads.queries(w, dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((jl.jl_turbo_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.m, w.d, bits),),
                     dtype=torch.uint8, device=dev)
    c4 = codes.view(w.B, w.Hkv, w.T, words)
    n4 = norms.view(w.B, w.Hkv, w.T, 2)
    stream = torch.cuda.current_stream(dev)

    def quantize():
        jl.jl_turbo_quantize_keys(Kf, Pi, S, bits, codes=codes, norms=norms)

    def decode_call():
        jl.jl_turbo_decode_attention(Q, Pinv, S, c4, n4, V, bits, softmax_scale=w.softmax_scale,
                                     out=out, workspace=ws)

    def step():
        quantize()
        decode_call()

    def timed_loop(fn, n):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / n

    for _ in range(args.warmup):
        step()
    _barrier(world, dev)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error after warm-up")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        _barrier(world, dev)
        clk.region_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        _barrier(world, dev)
        clk.region_end()
        q_ms = timed_loop(quantize, args.steps)
        d_ms = timed_loop(decode_call, args.steps)
        _barrier(world, dev)
        clk.extend(top_up=step)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error in the timed region")
    ms_step = reduce_max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)

    # estimator quality on sampled heads (untimed): normalised error of the
    # scores against the exact inner products
    score_err = None
    if not args.no_score_error:
        _, sc = jl.jl_turbo_decode_attention(Q, Pinv, S, c4, n4, V, bits, want_scores=True,
                                             workspace=ws)
        errs = []
        for b in range(min(w.B, 2)):
            for h in range(0, w.Hq, max(1, w.Hq // 4)):
                kv = K[b, h // w.G].double()
                q = Q[b, h].double()
                exact = kv @ q
                denom = kv.norm(dim=1) * q.norm()
                errs.append(((sc[b, h].double() - exact) / denom).pow(2).mean().item())
        score_err = {"rms_normalised_error": math.sqrt(sum(errs) / len(errs)),
                     "heads_sampled": len(errs),
                     "definition": "rms over sampled heads and all keys of "
                                   "(score - <q,k>) / (||q|| ||k||)"}

    e2e = None
    if not args.no_e2e:
        hK = K.cpu().pin_memory()
        hV = V.cpu().pin_memory()
        hQ = Q.cpu().pin_memory()
        hOut = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            K.copy_(hK, non_blocking=True)
            V.copy_(hV, non_blocking=True)
            Q.copy_(hQ, non_blocking=True)
            step()
            hOut.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        _barrier(world, dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e_steps = max(3, args.steps // 4)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        _barrier(world, dev)
        e_ms = reduce_max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)
        e2e = {"value": whole_job_rate(n_keys, world, e_ms), "unit": "keys/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": (hK.numel() + hV.numel() + hQ.numel()) * 2,
               "d2h_bytes_per_step": hOut.numel() * 2}

    per_key = words * 4 + 4
    qb = n_keys * (2 * w.d + per_key)
    db = n_keys * (per_key + 2 * w.d) + w.B * w.Hq * w.d * 2 * 2
    phases = {
        "quantize": {"ms": q_ms, "keys_per_s": n_keys / (q_ms * 1e-3), "algorithmic_bytes": qb,
                     "GB_per_s": qb / (q_ms * 1e-3) / 1e9,
                     "tflops": n_keys * 2 * (w.d * w.d + w.m * w.d) / (q_ms * 1e-3) / 1e12},
        "decode": {"ms": d_ms, "keys_scored_per_s": n_keys / (d_ms * 1e-3),
                   "algorithmic_bytes": db, "GB_per_s": db / (d_ms * 1e-3) / 1e9},
    }
    for ph in phases.values():
        ph["frac_of_hbm_peak"] = ph["GB_per_s"] / peak
    dom = max(phases, key=lambda k: phases[k]["ms"])
    kname = {"quantize": "jl_turbo_quantize_keys", "decode": "jl_turbo_decode_attention"}[dom]
    traffic = ncu_traffic(("turbo_quantize" if dom == "quantize" else "turbo_decode") + ":" + w.name)
    return {
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": whole_job_rate(n_keys, world, ms_step), "unit": "keys/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} T={w.T} d={w.d} "
                               f"m={w.m}, {bits}-bit cells + 1-bit residual QJL",
                   "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
                   "l2": "inputs exceed L2 (126 MB); no flush"},
        "phases": phases,
        "phase_timing": "each phase alone: K back-to-back calls, CUDA events at the ends",
        "roofline": {"kernel": kname, "bound": "hbm", "achieved": phases[dom]["GB_per_s"],
                     "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                     "frac": phases[dom]["GB_per_s"] / peak,
                     "algorithmic_bytes_per_launch": phases[dom]["algorithmic_bytes"],
                     "traffic": traffic["dram_bytes_per_launch"] if traffic else None},
        "score_error": score_err,
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clk.summary(),
    }


def _timed_loop(stream, fn, n):
    """Mean device time per call of n back-to-back calls (events at the ends
    only: an event between calls would drain the stream)."""
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / n


def graph_step_time(stream, step, n, warm=3):
    """Device time per step of `step` captured once into a CUDA graph and
    replayed n times (the launch-bound small workloads: the host no longer
    paces the kernels).  The library's launches are capturable: they only
    enqueue on the caller's stream (programmatic dependent launches become
    graph edges) and never allocate or synchronise.  Returns None when the
    capture fails."""
    try:
        for _ in range(warm):
            step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                step()
        stream.wait_stream(side)
        for _ in range(warm):
            g.replay()
        torch.cuda.synchronize()
        ms = _timed_loop(stream, g.replay, n)
        del g
        return ms
    except RuntimeError:
        torch.cuda.synchronize()
        return None


def phase_records(w, n_keys, q_ms, d_ms, peak, decode, extra_fixed=None):
    """Per-phase rates and roofline fractions from event-timed durations."""
    qb = quantize_bytes(w, n_keys)
    phases = {"quantize": {"ms": q_ms, "keys_per_s": n_keys / (q_ms * 1e-3),
                           "tokens_per_s": w.B * w.T / (q_ms * 1e-3),
                           "algorithmic_bytes": qb,
                           "GB_per_s": qb / (q_ms * 1e-3) / 1e9}}
    phases["quantize"]["frac_of_hbm_peak"] = phases["quantize"]["GB_per_s"] / peak
    if decode:
        db = decode_bytes(w)
        phases["decode"] = {"ms": d_ms, "keys_scored_per_s": n_keys / (d_ms * 1e-3),
                            "head_key_pairs_per_s": w.B * w.Hq * w.T / (d_ms * 1e-3),
                            "algorithmic_bytes": db,
                            "GB_per_s": db / (d_ms * 1e-3) / 1e9}
        phases["decode"]["frac_of_hbm_peak"] = phases["decode"]["GB_per_s"] / peak
        if extra_fixed:
            phases["decode"]["fixed_bytes_not_counted"] = extra_fixed
    return phases


PHASE_KERNEL = {"quantize": "jl_quantize_keys (quantize_tc_kernel)",
                "decode": "jl_decode_attention (qproj + decode_scorer_kernel + combine)"}


def load_tensor_peaks():
    """(burst, sustained) dense bf16 TFLOP/s from MEASURED_PEAKS.json, else the
    fallback burst figure for both."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return (float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    "measured")
    return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def quantize_flops(w, n_keys):
    """The projection K S^T: 2 m d flops per key."""
    return 2 * w.m * w.d * n_keys


def roofline_of(phase, rec, w, peak, peak_kind, full_size=True, n_keys=None):
    """Roofline entry of one phase: its algorithmic bytes (or, for a quantizer
    whose flops per byte exceed the ridge of the measured peaks, its flops)
    over its event-timed duration, against the measured HBM copy bandwidth
    (or the measured bf16 tensor peak).  DRAM traffic per launch comes from
    the committed ncu summary when the kernel's source is unchanged and the
    workload is the full-size one the summary was scaled to."""
    traffic = ncu_traffic(phase + ":" + w.name) if full_size else None
    r = {"kernel": PHASE_KERNEL[phase], "bound": "hbm", "achieved": rec["GB_per_s"],
         "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
         "frac": rec["GB_per_s"] / peak,
         "algorithmic_bytes_per_launch": rec["algorithmic_bytes"],
         "traffic": traffic["dram_bytes_per_launch"] if traffic else None}
    if phase == "quantize" and n_keys:
        t_burst, t_sus, t_kind = load_tensor_peaks()
        flops = quantize_flops(w, n_keys)
        intensity = flops / rec["algorithmic_bytes"]
        ridge = t_burst * 1e12 / (peak * 1e9)
        tf = flops / (rec["ms"] * 1e-3) / 1e12
        r["flops_per_launch"] = flops
        r["flop_per_byte"] = intensity
        r["ridge_flop_per_byte"] = ridge
        r["tensor_tflops"] = tf
        r["frac_of_bf16_burst"] = tf / t_burst
        r["frac_of_bf16_sustained"] = tf / t_sus
        if intensity > ridge:
            r.update({"bound": "tensor", "achieved": tf, "peak": t_burst,
                      "peak_kind": f"{t_kind} bf16_tflops (burst; the phase is timed alone)",
                      "unit": "TFLOP/s", "frac": tf / t_burst})
    if traffic:
        for k in ("dram_read_bytes_per_launch", "dram_write_bytes_per_launch",
                  "l2_write_bytes_per_launch", "write_side"):
            if k in traffic:
                r[k.replace("_per_launch", "")] = traffic[k]
    return r


def measure_config(jl, w, dev, steps, warmup, peak, peak_kind, with_score_error, clk=None):
    """One more workload on one GPU: quantize every key, then one decode step
    over the compressed cache (prefill: quantize only).  Returns a record with
    the step time, per-phase rates and rooflines (and, for the sketch-size
    sweep, the estimator's error against the exact inner products)."""
    stream = torch.cuda.current_stream(dev)
    decode = w.name != "prefill"
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    K = workloads.keys(w, dev)
    Kf = K.view(-1, w.d)
    n_keys = Kf.shape[0]
    W = w.m // 32
    signs = torch.empty((n_keys, W), dtype=torch.int32, device=dev)
    norms = torch.empty((n_keys,), dtype=torch.float16, device=dev)
    if decode:
        V = workloads.values(w, dev)
        Q = workloads.queries(w, dev)
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((jl.jl_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.m, w.d),),
                         dtype=torch.uint8, device=dev)
        sg4 = signs.view(w.B, w.Hkv, w.T, W)
        nr3 = norms.view(w.B, w.Hkv, w.T)

    def quantize():
        jl.jl_quantize_keys(Kf, S, signs, norms)

    def decode_call():
        jl.jl_decode_attention(Q, S, sg4, nr3, V, softmax_scale=w.softmax_scale,
                               out=out, workspace=ws)

    def step():
        quantize()
        if decode:
            decode_call()

    # each workload starts from an idle GPU, as the headline does: the
    # previous config's sustained load can leave the power controller
    # holding the clocks down for a while
    torch.cuda.synchronize(dev)
    time.sleep(1.0)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    if clk is not None:
        clk.region_start()
    ms = _timed_loop(stream, step, steps)
    if clk is not None:
        clk.region_end()
    q_ms = _timed_loop(stream, quantize, steps)
    d_ms = _timed_loop(stream, decode_call, steps) if decode else 0.0
    if clk is not None:
        clk.extend(top_up=step)
    if jl.jl_device_error() != 0:
        raise RuntimeError(f"device error in workload {w.name}")
    phases = phase_records(w, n_keys, q_ms, d_ms, peak, decode)
    rec = {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} T={w.T} d={w.d} m={w.m}",
           "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "keys_per_s": n_keys / (ms * 1e-3), "phases": phases,
           "rooflines": {ph: roofline_of(ph, phases[ph], w, peak, peak_kind, n_keys=n_keys)
                         for ph in phases},
           "l2": "inputs exceed L2 (126 MB); no flush" if n_keys * w.d * 2 > 126e6
                 else "inputs fit in L2; latency-bound parity workload"}
    if clk is not None:
        rec["clocks"] = clk.summary()
    if n_keys * w.d * 2 <= 126e6 // 8:
        # launch-bound: the same step replayed from a CUDA graph
        g_ms = graph_step_time(stream, step, steps)
        if g_ms is not None:
            rec["graph"] = {"ms_per_step": g_ms, "keys_per_s": n_keys / (g_ms * 1e-3),
                            "note": "the step captured once into a CUDA graph and replayed; "
                                    "ms_per_step above is the eager launch loop"}
    if w.name == "prefill":
        rec["quantize_tokens_per_s"] = w.T / (q_ms * 1e-3)
        rec["quantize_tokens_per_s_note"] = ("tokens of all 32 layers x 8 KV heads per second "
                                             "(keys/s divided by layers x heads)")
    if decode and with_score_error:
        rec["score_error"] = score_error(jl, w, Q, S, sg4, nr3, V, K)
    del K, signs, norms
    if decode:
        del V, Q, out, ws
    torch.cuda.empty_cache()
    return rec


def other_configs():
    """The workloads measured beside the headline one: the single-head parity
    workload, long-context MHA decode, prefill quantization and the eight
    points of the sketch-size sweep."""
    return ([workloads.SINGLE, workloads.LONG, workloads.PREFILL] + workloads.sweep_points())


def config_key(w) -> str:
    return w.name if w.name != "sweep" else f"sweep-m{w.m}-d{w.d}"


def run_context_parallel(args, rank, world, local_rank):
    """--workload long-cp: one sequence's context split across the ranks
    (strong scaling).  Rank r holds keys context_range(T, world, r) of every
    head; a step quantizes the rank's slice of keys, decodes it to softmax
    states, all-gathers the states and merges them (the output is the same on
    every rank).  value = all keys of the context over the slowest rank's
    step time."""
    import bit_jl_key_b200 as jl
    from bit_jl_key_b200.context_parallel import context_range, decode_context_parallel

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = pick_workload(args.workload, args.batch)
    a, b = context_range(w.T, world, rank)
    wl = w.with_(T=b - a)                       # this rank's share, for the byte counts
    peak, peak_kind = load_peaks()
    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    K = workloads.keys(w, dev)[:, :, a:b].contiguous()
    V = workloads.values(w, dev)[:, :, a:b].contiguous()
    torch.cuda.empty_cache()
    Q = workloads.queries(w, dev)
    W = w.m // 32
    n_keys = wl.B * wl.Hkv * wl.T
    signs = torch.empty((wl.B, wl.Hkv, wl.T, W), dtype=torch.int32, device=dev)
    norms = torch.empty((wl.B, wl.Hkv, wl.T), dtype=torch.float16, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    ws_bytes = jl.jl_decode_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.T, wl.m, wl.d)
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def quantize():
        jl.jl_quantize_keys(K.view(-1, w.d), S, signs.view(-1, W), norms.view(-1))

    def decode_call():
        decode_context_parallel(Q, S, signs, norms, V, w.softmax_scale, out=out, workspace=ws)

    def step():
        quantize()
        decode_call()

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error after warm-up")
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        clk.region_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        barrier()
        clk.region_end()
        q_ms = _timed_loop(stream, quantize, args.steps)
        d_ms = _timed_loop(stream, decode_call, args.steps)
        barrier()
        clk.extend(top_up=step)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error in the timed region")
    ms_step = reduce_max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    q_ms = reduce_max_over_ranks(q_ms, world, dev)
    d_ms = reduce_max_over_ranks(d_ms, world, dev)
    keys_all = w.B * w.Hkv * w.T

    # ---- end to end: the rank's keys, values and the queries from pinned
    # host memory, the output back
    e2e = None
    if not args.no_e2e:
        hK, hV, hQ = (t.cpu().pin_memory() for t in (K, V, Q))
        hOut = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hK, hV, hQ))

        def e2e_step():
            K.copy_(hK, non_blocking=True)
            V.copy_(hV, non_blocking=True)
            Q.copy_(hQ, non_blocking=True)
            step()
            hOut.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        barrier()
        e_steps = max(3, args.steps // 4)
        e_ms = _timed_loop(stream, e2e_step, e_steps)
        barrier()
        e_ms = reduce_max_over_ranks(e_ms, world, dev)
        e2e = {"value": keys_all / (e_ms * 1e-3), "unit": "keys/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hOut.numel() * 2}
    phases = phase_records(wl, n_keys, q_ms, d_ms, peak, True,
                           {"states exchanged per rank": w.B * w.Hq * (w.d + 2) * 4})
    rooflines = {ph: roofline_of(ph, phases[ph], wl, peak, peak_kind, full_size=False,
                                 n_keys=n_keys) for ph in phases}
    rooflines["decode"]["kernel"] = ("jl_decode_attention_state (qproj + decode_scorer_kernel "
                                     "+ combine) + all-gather + merge_states_kernel")
    dom = max(phases, key=lambda k: phases[k]["ms"])
    return {
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": keys_all / (ms_step * 1e-3), "unit": "keys/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": f"{w.name} context split over {world} rank(s): B={w.B} "
                               f"Hq={w.Hq} Hkv={w.Hkv} T={w.T} (this rank {wl.T}) "
                               f"d={w.d} m={w.m}",
                   "global_batch": w.B, "seq_len": w.T, "parallelism": f"cp{world}",
                   "l2": "inputs exceed L2 (126 MB) at up to 8 ranks; no flush"},
        "phases": phases,
        "phase_timing": "each phase alone: K back-to-back calls, CUDA events at the ends; "
                        "max over ranks",
        "roofline": rooflines[dom],
        "rooflines": rooflines,
        "e2e": e2e,
        "gpu_launches": 5 * args.steps,
        "clocks": clk.summary(),
    }


def run_ours(args, rank, world, local_rank):
    import bit_jl_key_b200 as jl

    if args.workload == "long-cp":
        return run_context_parallel(args, rank, world, local_rank)
    if args.workload in ("turbo-gqa", "turbo-gqa-d64"):
        return run_turbo(args, rank, world, local_rank)
    if args.workload == "search":
        return run_search(args, rank, world, local_rank)
    if args.workload in ("paged-gqa", "turbo-paged-gqa"):
        return run_paged(args, rank, world, local_rank)
    if args.workload in ("dequant-gqa", "turbo-dequant-gqa"):
        return run_dequant(args, rank, world, local_rank)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = rank_workload(args, rank)
    decode = w.name != "prefill"
    peak, peak_kind = load_peaks()

    S = jl.jl_sketch_init(w.m, w.d, w.sketch_seed, device=dev)
    K = workloads.keys(w, dev)
    Kf = K.view(-1, w.d)
    n_keys = Kf.shape[0]
    W = w.m // 32
    signs = torch.empty((n_keys, W), dtype=torch.int32, device=dev)
    norms = torch.empty((n_keys,), dtype=torch.float16, device=dev)
    if decode:
        V = workloads.values(w, dev)
        Q = workloads.queries(w, dev)
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        ws_bytes = jl.jl_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.T, w.m, w.d)
        ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
        sg4 = signs.view(w.B, w.Hkv, w.T, W)
        nr3 = norms.view(w.B, w.Hkv, w.T)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 1 + (3 if decode else 0)

    def quantize():
        jl.jl_quantize_keys(Kf, S, signs, norms)

    def decode_call():
        jl.jl_decode_attention(Q, S, sg4, nr3, V, softmax_scale=w.softmax_scale,
                               out=out, workspace=ws)

    def step():
        quantize()
        if decode:
            decode_call()

    def timed_loop(fn, n):
        """Mean device time per call of n back-to-back calls (events at the
        ends only: an event between calls would drain the stream)."""
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / n

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error after warm-up")

    # timed region: whole steps, events at its ends only; then each phase
    # alone, back to back, for the per-phase durations and the roofline
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        clk.region_start()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        barrier()
        clk.region_end()
        q_ms = timed_loop(quantize, args.steps)
        d_ms = timed_loop(decode_call, args.steps) if decode else 0.0
        barrier()
        clk.extend(top_up=step)
    ms_total = t0.elapsed_time(t1)
    if jl.jl_device_error() != 0:
        raise RuntimeError("device error in the timed region")

    ms_step = reduce_max_over_ranks(ms_total / args.steps, world, dev)
    keys_all = n_keys * world
    value = whole_job_rate(n_keys, world, ms_step)

    # ---- estimator quality on sampled heads (untimed)
    score_err = recon_err = None
    if decode and not args.no_score_error:
        score_err = score_error(jl, w, Q, S, sg4, nr3, V, K)
        recon_err = reconstruction_error(jl, w, S, signs, norms, K)

    # ---- end to end through the binding with pinned host buffers
    e2e = None
    if not args.no_e2e:
        hK = K.cpu().pin_memory()
        del K
        torch.cuda.empty_cache()
        Kd = torch.empty(hK.shape, dtype=hK.dtype, device=dev)
        h2d = hK.numel() * hK.element_size()
        if decode:
            hV = V.cpu().pin_memory()
            hQ = Q.cpu().pin_memory()
            hOut = torch.empty(out.shape, dtype=out.dtype).pin_memory()
            Vd, Qd = V, Q
            h2d += hV.numel() * hV.element_size() + hQ.numel() * hQ.element_size()
            d2h = hOut.numel() * hOut.element_size()
        else:
            hSig = torch.empty(signs.shape, dtype=signs.dtype).pin_memory()
            hNrm = torch.empty(norms.shape, dtype=norms.dtype).pin_memory()
            d2h = hSig.numel() * 4 + hNrm.numel() * 2

        def e2e_step():
            Kd.copy_(hK, non_blocking=True)
            if decode:
                Vd.copy_(hV, non_blocking=True)
                Qd.copy_(hQ, non_blocking=True)
            jl.jl_quantize_keys(Kd.view(-1, w.d), S, signs, norms)
            if decode:
                jl.jl_decode_attention(Qd, S, sg4, nr3, Vd,
                                       softmax_scale=w.softmax_scale, out=out,
                                       workspace=ws)
                hOut.copy_(out, non_blocking=True)
            else:
                hSig.copy_(signs, non_blocking=True)
                hNrm.copy_(norms, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e_steps = max(3, args.steps // 4)
        e0.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e1.record(stream)
        barrier()
        e_ms = reduce_max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)
        e2e = {"value": whole_job_rate(n_keys, world, e_ms), "unit": "keys/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    # ---- roofline of the dominant kernel, and of both phases
    fixed = None
    if decode:
        # per-call bytes outside the per-key accounting: listed, not in GB/s
        fixed = {"queries": Q.numel() * Q.element_size(),
                 "sketch": S.numel() * S.element_size(),
                 "out": out.numel() * out.element_size(),
                 "workspace (projections + partial states)": int(ws_bytes)}
    phases = phase_records(w, n_keys, q_ms, d_ms, peak, decode, fixed)
    rooflines = {ph: roofline_of(ph, phases[ph], w, peak, peak_kind, full_size=not args.batch,
                                 n_keys=n_keys) for ph in phases}
    dom = max(phases, key=lambda k: phases[k]["ms"])
    roof = rooflines[dom]

    clocks = clk.summary()
    line = {
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": value, "unit": "keys/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} T={w.T} "
                               f"d={w.d} m={w.m}",
                   "global_batch": w.B * world, "seq_len": w.T,
                   "parallelism": f"dp{world}",
                   "l2": "inputs exceed L2 (126 MB); no flush"},
        "phases": phases,
        "phase_timing": "each phase alone: K back-to-back calls, CUDA events at the ends",
        "roofline": roof,
        "rooflines": rooflines,
        "score_error": score_err,
        "reconstruction_error": recon_err,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    return line


def measure_other_configs(jl, dev, args, peak, peak_kind):
    steps = max(3, min(args.steps, 10))
    warmup = max(3, min(args.warmup, 5))
    torch.cuda.empty_cache()
    recs = {}
    with ClockSampler(dev.index or 0) as clk:
        for w in other_configs():
            rec = measure_config(jl, w, dev, steps, warmup, peak, peak_kind,
                                 with_score_error=(w.name == "sweep" and not args.no_score_error),
                                 clk=clk)
            cb = getattr(args, "config_baselines", {}).get(config_key(w))
            if cb is not None:
                rec["cpu_baseline"] = cb
            recs[config_key(w)] = rec
    recs["note"] = ("each workload alone on one GPU, after the headline; steps and warm-up "
                    "as listed per workload; rates and rooflines as the headline's; clocks "
                    "per workload from its own timed region")
    return recs


# --------------------------------------------------------------------------
# oracle timing (cpu_baseline and the reference arm)

def oracle_sample(w: workloads.Workload):
    """A bounded sample of the workload for the float64 oracle: the first
    (b, kv-head) unit of keys/values and its G query heads (prefill: the first
    16384 keys).  Returns (callable running one oracle step, keys per step,
    description)."""
    import numpy as np
    import oracle

    S64 = oracle.sketch(w.m, w.d, w.sketch_seed)
    if w.name == "search":
        n, nq = 262144, 4
        X = workloads.keys(w.with_(T=n)).view(-1, w.d).double().numpy()
        sig, _, n16, _ = oracle.quantize(X, S64)            # set-up, untimed
        n64 = oracle.fp16_bits_to_f64(n16)
        Qs = workloads.queries(w).view(-1, w.d)[:nq].double().numpy()

        def run():
            oracle.search_topk(Qs, S64, sig, n64, workloads.SEARCH_K)
        return run, n * nq, (f"{nq} queries x the first {n} index vectors of the workload's "
                             f"recipe (scores + top-{workloads.SEARCH_K})")
    if w.name == "dequant-gqa":
        n = 16384
        Kf = workloads.keys(w.with_(B=1, Hkv=1, T=n)).view(-1, w.d).double().numpy()
        sig, _, n16, _ = oracle.quantize(Kf, S64)          # set-up, untimed
        n64 = oracle.fp16_bits_to_f64(n16)

        def run():
            oracle.dequantize(sig, n64, S64)
        return run, n, f"first {n} codes of the workload's recipe (dequantize only)"
    if w.name == "turbo-dequant-gqa":
        from oracle import turbo as tq
        n = 131072
        bits = workloads.TURBO_MSE_BITS
        Kf = workloads.keys(w.with_(B=1, Hkv=1, T=n)).view(-1, w.d).double().numpy()
        c = tq.lloyd_max(w.d, bits)                           # set-up, untimed
        Pit = tq.rotation_stored(w.d, workloads.TURBO_ROTATION_SEED)
        q = tq.quantize(Kf, Pit, c, S64)
        nk = oracle.fp16_bits_to_f64(q["norm16"])
        nr = oracle.fp16_bits_to_f64(q["rnorm16"])

        def run():
            tq.dequantize(q["cell"], q["signs"], nk, nr, Pit, S64, c)
        return run, n, f"first {n} codes of the workload's recipe (dequantize only)"
    if w.name in ("turbo-gqa", "turbo-paged-gqa", "turbo-gqa-d64"):
        from oracle import turbo as tq
        T = w.T
        sub = w.with_(B=1, Hkv=1, Hq=w.G, T=T)
        K = workloads.keys(sub).double().numpy().reshape(-1, w.d)
        V = workloads.values(sub).double().numpy()
        Q = workloads.queries(sub).double().numpy()
        bits = workloads.TURBO_MSE_BITS
        c = tq.lloyd_max(w.d, bits)                           # set-up, untimed
        Pit = tq.rotation_stored(w.d, workloads.TURBO_ROTATION_SEED)

        def run():
            q = tq.quantize(K, Pit, c, S64)
            tq.decode(Q, Pit, S64, c, q["cell"].reshape(1, 1, T, w.d),
                      q["signs"].reshape(1, 1, T, -1),
                      oracle.fp16_bits_to_f64(q["norm16"]).reshape(1, 1, T),
                      oracle.fp16_bits_to_f64(q["rnorm16"]).reshape(1, 1, T), V,
                      w.softmax_scale)
        return run, T, (f"one (b, kv-head) unit: {T} keys, {w.G} query heads, "
                        f"TurboQuant-prod quantize + decode in float64")
    if w.name == "prefill":
        n = 16384
        Kf = workloads.keys(w.with_(B=1, Hkv=1, T=n)).view(-1, w.d).double().numpy()

        def run():
            oracle.quantize(Kf, S64)
        return run, n, f"first {n} keys of the workload's recipe (quantize only)"
    T = w.T if w.name != "long" else 32768
    sub = w.with_(B=1, Hkv=1, Hq=w.G, T=T)
    K = workloads.keys(sub).double().numpy()
    V = workloads.values(sub).double().numpy()
    Q = workloads.queries(sub).double().numpy()

    def run():
        sig, nrm, n16, _ = oracle.quantize(K.reshape(-1, w.d), S64)
        oracle.decode(Q, S64, sig.reshape(1, 1, T, w.m // 32),
                      oracle.fp16_bits_to_f64(n16).reshape(1, 1, T), V,
                      w.softmax_scale)
    return run, T, (f"one (b, kv-head) unit: {T} keys, {w.G} query heads, "
                    f"quantize + decode in float64")


def unit_of(w) -> str:
    return "query-vector pairs/s" if w.name == "search" else "keys/s"


def time_oracle(w, steps=1, warmup=0, min_seconds=0.0):
    """The oracle on the host cores over its bounded sample of the workload:
    `steps` runs of the sample, repeated until at least min_seconds of CPU
    work have been timed."""
    import oracle
    run, keys, desc = oracle_sample(w)
    for _ in range(warmup):
        run()
    t = time.perf_counter()
    n = 0
    while True:
        for _ in range(steps):
            run()
        n += steps
        if time.perf_counter() - t >= min_seconds:
            break
    dt = (time.perf_counter() - t) / n
    return {"value": keys / dt, "unit": unit_of(w), "cores": oracle.max_threads(),
            "kind": "oracle", "sample": desc + (f", repeated {n} times" if n > 1 else ""),
            "s_per_step": dt, "seconds_timed": dt * n}


def run_reference(args, rank, world):
    w = rank_workload(args, rank)
    if rank != 0:
        return None
    cb = time_oracle(w, steps=args.steps, warmup=args.warmup)
    return {
        "impl": "reference",
        "metric": "decode keys scored/s and achieved HBM GB/s (% peak); quantize tokens/s",
        "value": cb["value"], "unit": unit_of(w), "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": cb["s_per_step"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} T={w.T} "
                               f"d={w.d} m={w.m}",
                   "global_batch": w.B * world, "seq_len": w.T,
                   "parallelism": f"dp{world}"},
        "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
        "e2e": {"value": cb["value"], "unit": unit_of(w), "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gqa")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (small profiling cases)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-score-error", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the selected workload (default gqa runs also time "
                         "the single, long, prefill and sweep workloads)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local_rank))
    try:
        # the oracle runs before any GPU work on rank 0 (bounded sample)
        cb = None
        args.config_baselines = {}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            # about 10 s of oracle work for the line's own baseline, 2 s for
            # each other config's (the default run stays within minutes)
            cb = time_oracle(pick_workload(args.workload, args.batch), steps=1,
                             min_seconds=10.0)
            if args.workload == "gqa" and not args.no_configs:
                for w in other_configs():
                    c = time_oracle(w, steps=1, min_seconds=2.0)
                    args.config_baselines[config_key(w)] = {
                        k: c[k] for k in ("value", "unit", "cores", "kind", "sample")}
        line = run_ours(args, rank, world, local_rank)
        if world == 1 and args.workload == "gqa" and not args.no_configs:
            # the other workloads, each on its own, after the headline's
            # tensors are released (weak-scaling runs skip them)
            import bit_jl_key_b200 as jl
            peak, peak_kind = load_peaks()
            line["configs"] = measure_other_configs(
                jl, torch.device("cuda", local_rank), args, peak, peak_kind)
        if cb is not None:
            line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
