"""Throughput of on-device decoding of entropy-coded weights (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one process per GPU)

A step decodes the whole LLaMA-2-7B-shaped stack -- 32 layers x {q, k, v, o 4096x4096; gate, up
11008x4096; down 4096x11008}, 6.48 G weights drawn from the seeded generators (N(0, 0.02) with 1%
of entries x 8), Float8-E4M3 with per-row AbsMax scales, per-tensor 12-bit rANS tables, 64 KiB
chunks, 128 streams, run 8 -- from its rANS streams in HBM into bf16 in HBM with ONE eq_decode
call over all 224 tensors (the pages decode a transformer block's weights together; the whole
model is the same call with more descriptors).  The weights are quantised and coded by the GPU
compressor, which is bit-identical to the oracle's encoder, so the timed containers are the ones
the full-stack parity test checks.  Every rank decodes its own copy (weak scaling; the decode has
no exchange step).  Timing: CUDA events on the launching stream around each step, the L2 flushed
between steps by writing a 256 MiB buffer (the step's 18 GB of traffic dwarfs the L2 anyway), max
over ranks.  `e2e` repeats the step through the C ABI with pinned host buffers: per tensor the
host -> device copy of its coded arrays and its decode (eq_decode_from_host), then the step's
status word read back.

The other workloads are reported under "also", each with its own roofline, issue roofline and
oracle baseline where one applies: the 1024x1024 E4M3 weight, the Int8 8192x8192 weight (7-, 8-
and 12-bit tables), the fused decode-GEMV on the 13B MLP (batch 1/4/16) and the MLP block, the
DFloat11 decode, EntroLLM-style integer codes, super weights, the GPU compressor and the block
pipeline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decoded params/s (rANS decode to bf16)"
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, ~8 TB/s

# sources of each captured kernel (its ncu record is used only while they hash the same)
CSRC_COMMON = ["eq_dequant.cuh", "eq_internal.cuh"]
RECORD_SOURCES = {
    "decode_e4m3_12bit": ["eq_rans_decode.cu", "eq_rans_core.cuh"] + CSRC_COMMON,
    "decode_int8_7bit": ["eq_rans_decode.cu", "eq_rans_core.cuh"] + CSRC_COMMON,
    "gemv_e4m3_12bit_b1": ["eq_rans_gemv.cu", "eq_rans_core.cuh"] + CSRC_COMMON,
    "gemv_e4m3_12bit_b4": ["eq_rans_gemv.cu", "eq_rans_core.cuh"] + CSRC_COMMON,
    "gemv_e4m3_12bit_b16": ["eq_rans_gemv.cu", "eq_rans_core.cuh"] + CSRC_COMMON,
    "huff_df11": ["eq_huff_decode.cu"] + CSRC_COMMON,
    "huff_uint8": ["eq_huff_decode.cu"] + CSRC_COMMON,
}


def kernel_sources_sha(key: str) -> str:
    """sha256 of the kernel's sources with comments removed and whitespace collapsed, so that an
    edit of a comment keeps a capture valid and any change of code does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in RECORD_SOURCES[key]:
        src = open(os.path.join(ROOT, "decoding_interleaved_rans_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()


def measured_record(key: str):
    """The kernel's committed ncu figures (profiles/traffic.json), or None when its sources
    changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(key)
    if not rec or rec.get("sources_sha256") != kernel_sources_sha(key):
        return None
    return rec


def measured_traffic(key: str, units: int):
    """DRAM bytes per launch from the committed ncu capture, scaled to `units` weights."""
    rec = measured_record(key)
    return None if rec is None else rec["dram_bytes_per_launch"] * units / rec["weights_per_launch"]


def issue_roofline(key: str, units: int, seconds: float, sm_mhz):
    """The instruction-issue roofline beside the HBM one: lane-instructions per weight from the
    committed ncu capture (warp instructions x 32), issued per second, against SMs x 4 schedulers
    x 32 lanes x the SM clock sampled during the timed region."""
    import torch
    rec = measured_record(key)
    if rec is None or "warp_instructions_per_launch" not in rec or not sm_mhz:
        return None
    per_weight = 32.0 * rec["warp_instructions_per_launch"] / rec["weights_per_launch"]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peak = sms * 4 * 32 * sm_mhz * 1e6
    achieved = per_weight * units / seconds
    return {"bound": "issue", "lane_instr_per_weight": per_weight, "achieved": achieved,
            "peak": peak, "unit": "lane-instr/s", "frac": achieved / peak, "sms": sms,
            "sm_mhz": sm_mhz, "source": f"warp instructions of the committed ncu capture '{key}'"}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "src": "fallback"}


def roofline(alg_bytes: float, seconds: float, peaks: dict, key: str | None, units: int,
             kernel: str) -> dict:
    """HBM roofline object: algorithmic bytes per launch over the event time, against the measured
    copy bandwidth (frac) and the nominal ~8 TB/s (frac_nominal)."""
    achieved = alg_bytes / seconds / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_src": peaks["src"],
            "frac_nominal": achieved / NOMINAL_HBM_GBS, "nominal_peak": NOMINAL_HBM_GBS,
            "traffic": measured_traffic(key, units) if key else None,
            "alg_bytes_per_launch": alg_bytes, "kernel": kernel}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms in the background.

    The sampler starts before the warm-up and a one-second untimed soak, so the clock has settled
    and samples exist even when the timed steps take only milliseconds; summary() reports the
    samples taken from 0.25 s before the timed region starts to its end (mark() brackets it)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.samples: list[tuple[float, str]] = []
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def wait_first_sample(self, timeout: float = 5.0):
        end = time.time() + timeout
        while self.proc and not self.samples and time.time() < end:
            time.sleep(0.05)

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        lo = (self.t0 or 0) - 0.25
        hi = (self.t1 or time.time()) + 0.05
        sm, mx, reasons, pw = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.samples:
            if not lo <= ts <= hi:
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                pw.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(pw) if pw else None,
                "window_s": round(hi - lo, 3)}


def dist_setup():
    import torch

    from decoding_interleaved_rans_b200 import dist
    world, rank, local = dist.env_rank()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    from decoding_interleaved_rans_b200 import dist
    dist.barrier()


def max_over_ranks(world, v: float) -> float:
    from decoding_interleaved_rans_b200 import dist
    return dist.max_over_ranks(v, device="cuda")


def time_steps(fn, steps, warmup, flush, stream):
    """CUDA-event time of each of `steps` calls of fn on `stream`, the L2 flushed before each."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    return times


# ------------------------------------------------------------------------------------------------
# workloads
# ------------------------------------------------------------------------------------------------

def prepare_rans(eq, wl_name: str, prob_bits: int | None = None):
    """Quantise + encode a one-tensor workload with the library's host compressor (no oracle)."""
    wl = synth.WORKLOADS[wl_name]
    spec = wl.tensors[0]
    w = spec.generate()
    fmt = eq.EQ_SYM_E4M3 if wl.symfmt == "e4m3" else eq.EQ_SYM_INT8
    sym, sc = eq.codec.quantize(w, fmt, wl.int8_div)
    del w
    h = eq.codec.rans_encode(sym, sc, fmt, wl.chunk_symbols, wl.streams, wl.run,
                             prob_bits=prob_bits or wl.prob_bits)
    return wl, h


def build_llama_stack(eq, dev):
    """The LLaMA-2-7B-shaped stack: each tensor drawn on the host from the seeded generators (a
    thread draws tensor i + 1 while the GPU codes tensor i), then quantised and rANS-coded by the
    GPU compressor.  Returns (DeviceRans list, frequency tables, seconds spent)."""
    import queue

    import torch
    wl = synth.WORKLOADS["llama2_7b"]
    q: queue.Queue = queue.Queue(maxsize=2)

    def producer():
        for spec in wl.tensors:
            q.put(torch.from_numpy(spec.generate()).pin_memory())
        q.put(None)

    t0 = time.time()
    th = threading.Thread(target=producer, daemon=True)
    th.start()
    tensors, freqs = [], []
    while True:
        w = q.get()
        if w is None:
            break
        wd = w.to(dev, non_blocking=True)
        sym, sc = eq.quantize_device(wd, eq.EQ_SYM_E4M3)
        f = eq.normalize_freqs(eq.histogram_device(sym).cpu().numpy(), 12)
        tensors.append(eq.rans_encode_device(sym, sc, eq.EQ_SYM_E4M3, wl.chunk_symbols,
                                             wl.streams, wl.run, freqs=f))
        freqs.append(f)
        del wd, sym
    th.join()
    torch.cuda.synchronize()
    return wl, tensors, freqs, time.time() - t0


def decode_launches(tensors) -> int:
    """Kernel launches one eq_decode call over `tensors` makes: one per kernel variant, each
    split into launches of at most 256 descriptors."""
    groups: dict = {}
    for t in tensors:
        if t.num_chunks:
            key = (t.symfmt, t.run, t.prob_bits)
            groups[key] = groups.get(key, 0) + 1
    return sum((n + 255) // 256 for n in groups.values())


# ------------------------------------------------------------------------------------------------
# oracle baselines (the plain C decoder, timed as it stands on the host cores)
# ------------------------------------------------------------------------------------------------

def _oracle_rans_from_device(t, freqs):
    import oracle
    u = lambda x, dt: x.cpu().numpy().view(dt)  # noqa: E731
    return oracle.RansTensor(t.rows, t.cols, t.symfmt, t.prob_bits, t.chunk_symbols, t.streams,
                             t.run, np.asarray(freqs, np.uint32), u(t.states, np.uint32),
                             u(t.word_off, np.uint64), u(t.words, np.uint16),
                             u(t.scales, np.uint16))


def _oracle_rans_from_host(h):
    import oracle
    return oracle.RansTensor(h.rows, h.cols, h.symfmt, h.prob_bits, h.chunk_symbols, h.streams,
                             h.run, h.freqs, h.states, h.word_off, h.words, h.scales)


def _chunk_syms(o, c: int) -> int:
    chunk = o.chunk_symbols or o.cols
    return min(chunk, o.numel - c * chunk)


def _decode_pairs(pairs, threads: int) -> float:
    """Decode (container, chunk) pairs with the oracle, one chunk per call, on `threads` threads
    (the C decoder releases the GIL); returns the seconds taken."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    def one(p):
        rc, _ = oracle.rans_decode_bf16(p[0], chunks=[p[1]], threads=1)
        assert rc == 0

    t0 = time.perf_counter()
    if threads <= 1:
        for p in pairs:
            one(p)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, pairs))
    return time.perf_counter() - t0


def oracle_rans_rates(containers, budget_s: float, seed: int = 0) -> dict:
    """The oracle's rANS decode + dequantisation on chunks drawn from every container: once on
    one thread, once chunk-parallel over every host core; each sized to about budget_s."""
    cores = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(seed)
    o0 = containers[0]
    per_sym = _decode_pairs([(o0, 0)], 1) / _chunk_syms(o0, 0)  # probe
    out = {"cores": cores}
    for label, thr in (("single_thread", 1), ("all_cores", cores)):
        want = budget_s * thr / max(per_sym, 1e-12)  # symbols that fit the budget
        per_tensor = max(1, int(want / len(containers) / max(1, _chunk_syms(o0, 0))))
        pairs = []
        for o in containers:
            k = min(o.num_chunks, per_tensor)
            pairs += [(o, int(c)) for c in sorted(rng.choice(o.num_chunks, k, replace=False))]
        secs = _decode_pairs(pairs, thr)
        syms = sum(_chunk_syms(o, c) for o, c in pairs)
        out[label] = {"value": syms / secs, "params": syms, "chunks": len(pairs),
                      "seconds": secs, "threads": thr}
    return out


def cpu_baseline_obj(rates: dict, config_params: int, sample: str) -> dict:
    """cpu_baseline: the all-cores rate as the value, the single-thread rate beside it, and both
    extrapolated to the whole workload."""
    a, s = rates["all_cores"], rates["single_thread"]
    return {"value": a["value"], "unit": "params/s", "cores": rates["cores"], "kind": "oracle",
            "sample": f"{sample}: {a['chunks']} chunks ({a['params']} params) chunk-parallel on "
                      f"{rates['cores']} threads; {s['chunks']} chunks ({s['params']} params) on "
                      f"one thread",
            "single_thread": s["value"],
            "projected_s_all_cores": config_params / a["value"],
            "projected_s_single_thread": config_params / s["value"]}


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def run_ours(args):
    import torch

    import decoding_interleaved_rans_b200 as eq
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    wl, tensors, freqs, build_s = build_llama_stack(eq, dev)
    outs = [torch.empty(t.rows, t.cols, dtype=torch.bfloat16, device=dev) for t in tensors]
    status = eq.new_status(dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    numel = sum(t.numel for t in tensors)
    coded = sum(t.compressed_bytes for t in tensors)
    alg_bytes = coded + 2 * numel
    launches = decode_launches(tensors)

    def flush():
        flush_buf.fill_(1)

    def step():
        eq.decode(tensors, outs, status, stream)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        clk.wait_first_sample()
        soak_end = time.time() + 1.0  # untimed: let the clocks settle under load
        while time.time() < soak_end:
            step()
            torch.cuda.synchronize()
        barrier(world)
        clk.mark(True)
        times = time_steps(step, args.steps, args.warmup, flush, stream)
        torch.cuda.synchronize()
        clk.mark(False)
    barrier(world)
    assert int(status.item()) == 0, "decode reported corrupt data"
    mean_s = max_over_ranks(world, statistics.mean(times))
    clocks = clk.summary()

    # end to end through the C ABI with host buffers (pinned): every step copies each tensor's
    # coded arrays host -> device and decodes it (eq_decode_from_host), then reads the step's
    # status word back; the decoded bf16 weights stay in HBM for the layers that use them
    pinned = [eq.PinnedRans.from_device(t) for t in tensors]
    h2d = sum(p.h2d_bytes() for p in pinned)
    st_host = torch.empty(1, dtype=torch.int32).pin_memory()
    copy_stream = torch.cuda.Stream(dev)

    def e2e_step():
        for t, p, o in zip(tensors, pinned, outs):
            eq.decode_from_host(t, p, o, status, stream, pieces=1, copy_stream=copy_stream)
        st_host.copy_(status, non_blocking=True)

    e2e_s = max_over_ranks(world, statistics.mean(
        time_steps(e2e_step, max(3, args.steps // 4), 3, flush, stream)))
    assert int(st_host.item()) == 0
    del pinned

    cpu = None
    if rank == 0 and not args.no_cpu:
        # the oracle on chunks drawn from every one of the 224 containers the GPU decodes
        conts = [_oracle_rans_from_device(t, f) for t, f in zip(tensors, freqs)]
        rates = oracle_rans_rates(conts, budget_s=8.0)
        cpu = cpu_baseline_obj(rates, numel, "chunks drawn from each of the 224 tensors")
        del conts
    del outs, tensors
    torch.cuda.empty_cache()

    also = []
    if not args.no_extra:
        also = extra_measurements(eq, dev, stream, flush, peaks, args, clocks.get("sm_mhz"),
                                  cpu_on=(rank == 0 and not args.no_cpu))
    barrier(world)
    if rank != 0:
        return
    kernel = "rans_decode_kernel<run 8, E4M3, 12-bit table>"
    line = {
        "metric": METRIC, "value": numel * world / mean_s, "unit": "params/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8->bf16", "data": "synthetic",
        "config": {"workload": "LLaMA-2-7B-shaped stack: 32 layers x {q,k,v,o 4096x4096; "
                               "gate,up 11008x4096; down 4096x11008}, N(0,0.02) with 1% x8 "
                               "outliers, Float8-E4M3, per-row AbsMax, per-tensor 12-bit tables, "
                               "64 KiB chunks, 128 streams, run 8; all 224 tensors in one "
                               "eq_decode call -> bf16",
                   "tensors": len(wl.tensors), "params_per_gpu": numel,
                   "compressed_bytes": coded, "bits_per_param": 8 * coded / numel,
                   "coder": "GPU compressor (bit-identical to the oracle's encoder)",
                   "build_s": build_s,
                   "l2": "inputs far larger than L2 (5.3 GB coded, 13 GB out); also flushed "
                         "between steps (256 MiB write)",
                   "parallelism": f"replicas x{world}"},
        "gbs": alg_bytes / mean_s / 1e9,
        "roofline": roofline(alg_bytes, mean_s, peaks, "decode_e4m3_12bit", numel, kernel),
        "issue_roofline": issue_roofline("decode_e4m3_12bit", numel, mean_s, clocks.get("sm_mhz")),
        "e2e": {"value": numel * world / e2e_s, "unit": "params/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": 4, "ms_per_step": e2e_s * 1e3,
                "result_read_back": "status word; the decoded bf16 weights stay in HBM",
                "path": "eq_decode_from_host per tensor (pinned host arrays copied, then "
                        "decoded)"},
        "gpu_launches": args.steps * launches,
        "launches_per_step": launches,
        "clocks": clocks,
        "also": also,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def extra_measurements(eq, dev, stream, flush, peaks, args, sm_mhz, cpu_on: bool):
    """The other workloads, each with its own roofline (and issue roofline and oracle baseline
    where one applies)."""
    import oracle
    import torch
    out = []
    steps = max(5, args.steps // 2)

    def cpu_rans(hosts, params, sample, budget=3.0):
        if not cpu_on:
            return None
        rates = oracle_rans_rates([_oracle_rans_from_host(h) for h in hosts], budget_s=budget)
        return cpu_baseline_obj(rates, params, sample)

    # ---- the single 1024 x 1024 E4M3 weight (16 KiB chunks, 32 streams): a latency case, 64
    # chunks of one warp each
    wl, h = prepare_rans(eq, "e4m3_1k")
    t = eq.DeviceRans.upload(h, dev)
    o = torch.empty(h.rows, h.cols, dtype=torch.bfloat16, device=dev)
    st = eq.new_status(dev)
    sec = statistics.mean(time_steps(lambda: eq.decode([t], [o], st, stream), steps, 3, flush,
                                     stream))
    assert int(st.item()) == 0
    alg = t.compressed_bytes + 2 * t.numel
    out.append({"what": "E4M3 1024x1024 N(0,0.02), 12-bit table, 16 KiB chunks, 32 streams",
                "params": t.numel, "ms": sec * 1e3, "params_per_s": t.numel / sec,
                "bits_per_param": 8 * t.compressed_bytes / t.numel,
                "roofline": roofline(alg, sec, peaks, None, t.numel,
                                     "rans_decode_kernel<run 8, E4M3, 12-bit table>"),
                "note": "64 chunks = 64 warps: bound by launch latency, not by HBM",
                "cpu_baseline": cpu_rans([h], t.numel, "every chunk", 1.0)})
    del t, o, h

    # ---- Int8 8192 x 8192 (H = 2.0 bits), 7-bit table (pair-table decode), with 8- and 12-bit
    # tables beside it; e2e from pinned host memory and the bf16-offload comparison
    for pb in (7, 8, 12):
        wl, h = prepare_rans(eq, "int8_8k", prob_bits=pb)
        t = eq.DeviceRans.upload(h, dev)
        o = torch.empty(h.rows, h.cols, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        sec = statistics.mean(time_steps(lambda: eq.decode([t], [o], st, stream), steps, 3,
                                         flush, stream))
        assert int(st.item()) == 0
        alg = t.compressed_bytes + 2 * t.numel
        kern = f"rans_decode_kernel<run 8, Int8, {pb}-bit table>"
        e = {"what": f"Int8 8192x8192 Laplace(0,0.01) clip 6b (H=2.0 bits), 64 KiB chunks, "
                     f"128 streams, {pb}-bit table", "params": t.numel, "ms": sec * 1e3,
             "params_per_s": t.numel / sec, "bits_per_param": 8 * t.compressed_bytes / t.numel,
             "roofline": roofline(alg, sec, peaks, "decode_int8_7bit" if pb == 7 else None,
                                  t.numel, kern)}
        if pb == 7:
            e["issue_roofline"] = issue_roofline("decode_int8_7bit", t.numel, sec, sm_mhz)
            src = eq.PinnedRans.from_host(h)
            st_host = torch.empty(1, dtype=torch.int32).pin_memory()
            out_host = torch.empty(h.rows, h.cols, dtype=torch.bfloat16).pin_memory()
            cs = torch.cuda.Stream(dev)

            def e2e_step():
                eq.decode_from_host(t, src, o, st, stream, pieces=1, copy_stream=cs)
                st_host.copy_(st, non_blocking=True)
            e2e_s = statistics.mean(time_steps(e2e_step, steps, 3, flush, stream))
            off_s = statistics.mean(time_steps(lambda: o.copy_(out_host, non_blocking=True),
                                               steps, 3, flush, stream))
            e["e2e"] = {"value": t.numel / e2e_s, "unit": "params/s",
                        "h2d_bytes_per_step": src.h2d_bytes(), "d2h_bytes_per_step": 4,
                        "ms_per_step": e2e_s * 1e3}
            e["offload_comparison"] = {
                "bf16_h2d_ms": off_s * 1e3, "bf16_h2d_bytes": 2 * t.numel,
                "coded_h2d_plus_decode_ms": e2e_s * 1e3, "speedup": off_s / e2e_s,
                "pages_claim": "DFloat11: 2.3-46.2x over CPU offload (end to end, their models "
                               "and hardware)"}
            e["cpu_baseline"] = cpu_rans([h], t.numel, "chunks drawn from the tensor")
            del src, out_host
        out.append(e)
        del t, o, h

    # ---- fused decode + GEMV over the three 13B MLP weights (gate, up 13824x5120; down
    # 5120x13824), E4M3, 12-bit tables, one row per chunk; algorithmic bytes = the coded weights
    # read (+ x and y)
    wl = synth.WORKLOADS["mlp_13b"]
    hosts, mats = [], []
    for spec in wl.tensors:
        sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_E4M3)
        h = eq.codec.rans_encode(sym, sc, eq.EQ_SYM_E4M3, wl.chunk_for(spec), wl.streams, wl.run)
        hosts.append(h)
        mats.append(eq.DeviceRans.upload(h, dev))
        del sym, sc
    params = sum(m.numel for m in mats)
    coded = sum(m.compressed_bytes for m in mats)
    gemv_cpu = None
    if cpu_on:
        # the oracle's decode of sampled rows, then its fp64 GEMV over them (batch 1)
        rng = np.random.default_rng(4)
        secs, n_s = 0.0, 0
        for h in hosts:
            o_ = _oracle_rans_from_host(h)
            rows = sorted(rng.choice(h.rows, 96, replace=False).tolist())
            xb = synth.activations(1, h.cols, 4)
            t0 = time.perf_counter()
            rc, wbits = oracle.rans_decode_bf16(o_, chunks=rows, threads=1)
            wr = wbits.reshape(h.rows, h.cols)[rows]
            oracle.gemv_f64(wr, xb)
            secs += time.perf_counter() - t0
            assert rc == 0
            n_s += len(rows) * h.cols
        gemv_cpu = {"value": n_s / secs, "unit": "params/s", "cores": 1, "kind": "oracle",
                    "sample": f"96 rows of each of gate/up/down ({n_s} params): decode + "
                              f"dequant, then the fp64 GEMV, batch 1, one thread",
                    "projected_s_single_thread": params / (n_s / secs)}
    del hosts
    for batch in wl.batches:
        xs = [torch.randn(batch, m.cols, device=dev).to(torch.bfloat16) for m in mats]
        ys = [torch.empty(batch, m.rows, dtype=torch.float32, device=dev) for m in mats]
        st = eq.new_status(dev)

        def layer():
            for m, x, y in zip(mats, xs, ys):
                eq.decode_gemv(m, x, y, st, stream)
        sec = statistics.mean(time_steps(layer, steps, 3, flush, stream))
        assert int(st.item()) == 0
        alg = coded + sum(x.numel() * 2 for x in xs) + sum(y.numel() * 4 for y in ys)
        key = f"gemv_e4m3_12bit_b{batch}"
        kern = "rans_gemv_tc_kernel" if batch >= 8 else "rans_gemv_kernel"
        e = {"what": f"fused decode+GEMV, 13B MLP gate/up/down, batch {batch}",
             "params": params, "ms": sec * 1e3, "params_per_s": params / sec,
             "bits_per_param": 8 * coded / params, "launches_per_step": len(mats),
             "roofline": roofline(alg, sec, peaks, key, params, kern),
             "issue_roofline": issue_roofline(key, params, sec, sm_mhz)}
        if batch == 1 and gemv_cpu:
            e["cpu_baseline"] = gemv_cpu
        out.append(e)
        # the whole MLP block: gate and up products, SiLU gate to bf16, down product
        byname = {spec.name: m for spec, m in zip(wl.tensors, mats)}
        g, u, d = byname["gate"], byname["up"], byname["down"]
        xb = xs[[spec.name for spec in wl.tensors].index("gate")]
        yb = torch.empty(batch, d.rows, dtype=torch.float32, device=dev)
        scratch = torch.empty(eq.mlp_scratch_bytes(g.rows, batch), dtype=torch.uint8, device=dev)
        sec = statistics.mean(time_steps(lambda: eq.mlp_decode(g, u, d, xb, yb, scratch, st,
                                                               stream), steps, 3, flush, stream))
        assert int(st.item()) == 0
        out.append({"what": f"MLP block from coded weights (13B: gate, up, SiLU gate, down), "
                            f"batch {batch}",
                    "params": params, "ms": sec * 1e3, "params_per_s": params / sec,
                    "roofline": roofline(coded + xb.numel() * 2 + yb.numel() * 4, sec, peaks,
                                         None, params, "eq_mlp_decode kernels")})
    del mats

    # ---- DFloat11: algorithmic bytes = EncodedExponent + PackedSignMantissa + Gaps + block_out
    # read, 2 B/weight written
    w = synth.WORKLOADS["df11_8k"].tensors[0].generate().ravel()
    hh = eq.codec.huff_encode(w)
    dh = eq.DeviceHuff.upload(hh, dev)
    ob = torch.empty(dh.n, dtype=torch.bfloat16, device=dev)
    st = eq.new_status(dev)
    sec = statistics.mean(time_steps(lambda: eq.huff_bf16_decode(dh, ob, st, stream), steps, 3,
                                     flush, stream))
    assert int(st.item()) == 0
    alg = dh.compressed_bytes + 2 * dh.n
    e = {"what": "DFloat11 bf16 decode, 8192x28672 N(0,0.015)", "params": dh.n, "ms": sec * 1e3,
         "params_per_s": dh.n / sec, "bits_per_param": 8 * dh.compressed_bytes / dh.n,
         "roofline": roofline(alg, sec, peaks, "huff_df11", dh.n, "huff_decode_kernel"),
         "issue_roofline": issue_roofline("huff_df11", dh.n, sec, sm_mhz)}
    if cpu_on:
        # the oracle's sequential canonical decode over the first 2^24 weights
        n_s = 1 << 24
        # the sample's own bit count: the oracle checks that its codes end exactly there
        bits_s = int(hh.lengths[(w[:n_s] >> 7) & 0xFF].astype(np.int64).sum())
        ho = oracle.HuffTensor(n_s, 8, hh.threads_per_block, bits_s, hh.lengths,
                               hh.enc_exp, hh.sign_mant[:n_s], hh.gaps, hh.block_out)
        t0 = time.perf_counter()
        rc, dec = oracle.huff_decode_bf16(ho)
        dt = time.perf_counter() - t0
        assert rc == 0 and np.array_equal(dec, w[:n_s])
        e["cpu_baseline"] = {"value": n_s / dt, "unit": "params/s", "cores": 1, "kind": "oracle",
                             "sample": f"the first {n_s} weights, sequential canonical decode "
                                       "(the oracle's decoder is single-threaded)",
                             "projected_s_single_thread": dh.n / (n_s / dt)}
    out.append(e)
    del dh, ob, hh, w

    # ---- EntroLLM-style integer weights: a phi3-mini-shaped MLP weight (8192 x 3072,
    # N(0, 0.02)), uint8 and uint4 codes Huffman-coded, decoded by the two-stage kernel
    w = synth.normal(8192, 3072, 0.02, 6)
    for bits in (8, 4):
        hi_ = eq.codec.entrollm_encode(w, bits)
        di = eq.DeviceHuffInt.upload(hi_, dev)
        oi = torch.empty(di.n, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        sec = statistics.mean(time_steps(lambda: eq.huff_int_decode(di, oi, st, stream), steps,
                                         3, flush, stream))
        assert int(st.item()) == 0
        alg = di.compressed_bytes + 2 * di.n
        key = "huff_uint8" if bits == 8 else None
        out.append({"what": f"EntroLLM-style uint{bits} codes, Huffman-coded, 8192x3072 N(0,0.02)",
                    "params": di.n, "ms": sec * 1e3, "params_per_s": di.n / sec,
                    "bits_per_param": 8 * di.compressed_bytes / di.n,
                    "roofline": roofline(alg, sec, peaks, key, di.n,
                                         "huff_decode_kernel<integer codes>"),
                    "issue_roofline": issue_roofline(key, di.n, sec, sm_mhz) if key else None,
                    "pages_context": "EntroLLM: 5.58 bits/param from uint8 on phi3-mini (real "
                                     "weights, Jetson)"})
        del di, oi, hi_
    del w

    # ---- super weights: the Int8 workload with 6 planted outliers (50-200x the typical weight),
    # kept exactly in the patch list and out of their rows' scales; the decode writes them back
    wl = synth.WORKLOADS["int8_8k"]
    w = wl.tensors[0].generate()
    synth.plant_super_weights(w, 6, 2)
    pidx, pval = eq.codec.super_weights(w)
    sym, sc = eq.codec.quantize_excluding(w, eq.EQ_SYM_INT8, wl.int8_div, pidx)
    hs = eq.codec.rans_encode(sym, sc, eq.EQ_SYM_INT8, wl.chunk_symbols, wl.streams, wl.run,
                              prob_bits=wl.prob_bits)
    hs.patch_idx, hs.patch_val = pidx, pval
    rows_sw = sorted({int(j) // w.shape[1] for j in pidx})
    psym, psc = eq.codec.quantize(w[rows_sw], eq.EQ_SYM_INT8, wl.int8_div)
    collapsed = float((psym == 0).mean())
    del w, sym, sc, psym, psc
    ts_ = eq.DeviceRans.upload(hs, dev)
    osw = torch.empty(hs.rows, hs.cols, dtype=torch.bfloat16, device=dev)
    st = eq.new_status(dev)
    sec = statistics.mean(time_steps(lambda: eq.decode([ts_], [osw], st, stream), steps, 3,
                                     flush, stream))
    assert int(st.item()) == 0
    alg = ts_.compressed_bytes + 2 * ts_.numel
    out.append({"what": "Int8 8192x8192 with 6 super weights (patch list written back in the "
                        f"decode epilogue), {wl.prob_bits}-bit table", "params": ts_.numel,
                "ms": sec * 1e3, "params_per_s": ts_.numel / sec, "super_weights": int(pidx.size),
                "zero_symbols_in_their_rows_without_exclusion": collapsed,
                "roofline": roofline(alg, sec, peaks, None, ts_.numel,
                                     f"rans_decode_kernel<run 8, Int8, {wl.prob_bits}-bit table> "
                                     "+ patch epilogue")})
    del ts_, osw, hs

    # ---- GPU compressor: fp32 weights in HBM -> quantise, histogram, frequency table (host),
    # rANS plan + encode; wall clock around the whole call (it reads the word total back once)
    wdev = torch.from_numpy(wl.tensors[0].generate()).to(dev)
    times_c = []
    for it in range(4):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        sym, sc = eq.quantize_device(wdev, eq.EQ_SYM_INT8, wl.int8_div)
        tc = eq.rans_encode_device(sym, sc, eq.EQ_SYM_INT8, wl.chunk_symbols, wl.streams, wl.run,
                                   prob_bits=wl.prob_bits)
        torch.cuda.synchronize()
        if it:
            times_c.append(time.perf_counter() - t0)
    sec = statistics.mean(times_c)
    n_c = wdev.numel()
    out.append({"what": "GPU compression (quantise + histogram + rANS plan + encode), Int8 8192x8192",
                "params": n_c, "ms": sec * 1e3, "params_per_s": n_c / sec,
                "projected_70B_s": 70e9 / (n_c / sec),
                "pages_claim": "70B compressed in < 10 min (summaries) / < 30 min (abstract)",
                "kernel": "quantize_kernel + histogram_kernel + rans_encode_kernel x2"})
    del wdev, sym, sc, tc
    torch.cuda.empty_cache()

    # ---- block-by-block decode overlapped with the block's forward GEMMs (4 LLaMA-2-7B-shaped
    # layers, coded on the GPU): compute alone on resident bf16 weights, decode then compute,
    # overlapped
    from decoding_interleaved_rans_b200.pipeline import BlockPipeline
    wl7 = synth.scaled(synth.WORKLOADS["llama2_7b"], layers=4)
    blocks, resident = [], []
    for layer in range(4):
        hs, rs = [], []
        for spec in [t for t in wl7.tensors if t.name.startswith(f"layers.{layer}.")]:
            wt = torch.from_numpy(spec.generate()).to(dev)
            sym, sc = eq.quantize_device(wt, eq.EQ_SYM_E4M3)
            hs.append(eq.rans_encode_device(sym, sc, eq.EQ_SYM_E4M3, wl7.chunk_symbols,
                                            wl7.streams, wl7.run))
            rs.append(wt.to(torch.bfloat16))
            del wt, sym, sc
        blocks.append(hs)
        resident.append(rs)
    pipe = BlockPipeline(blocks)
    lparams = sum(t.numel for b in blocks for t in b)
    for tokens in (1, 512):
        xt = torch.randn(tokens, 11008, device=dev).to(torch.bfloat16)

        def fwd(i, ws):
            for w_ in ws:
                torch.matmul(xt[:, :w_.shape[1]], w_.t())
        ts_c = time_steps(lambda: [fwd(i, resident[i]) for i in range(4)], steps, 3, flush, stream)
        ts_s = time_steps(lambda: pipe.run(fwd, overlap=False), steps, 3, flush, stream)
        ts_o = time_steps(lambda: pipe.run(fwd, overlap=True), steps, 3, flush, stream)
        assert int(pipe.status.item()) == 0
        c, sq, ov = (statistics.mean(v) for v in (ts_c, ts_s, ts_o))
        out.append({"what": f"4 LLaMA-2-7B layers, {tokens} token(s): forward GEMMs on resident "
                            f"bf16 vs decode-then-compute vs overlapped",
                    "params": lparams, "compute_ms": c * 1e3, "sequential_ms": sq * 1e3,
                    "overlapped_ms": ov * 1e3, "slowdown_sequential": sq / c,
                    "slowdown_overlapped": ov / c,
                    "pages_claim": "1.5-2x slower than bf16 (EntQuant), 2-3x (DFloat11 forum)",
                    "kernel": "rans_decode_kernel + cuBLAS bf16 GEMM"})
    del pipe, blocks, resident

    # ---- fused decode + GEMV over the ~2-bit Int8 8192x8192 weight, one row per chunk and 32
    # streams (the fused kernel's layout), with the 7-bit pair table and with the 12-bit table
    wl8 = synth.WORKLOADS["int8_8k"]
    spec = wl8.tensors[0]
    sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_INT8, wl8.int8_div)
    for pb in (7, 12):
        m = eq.DeviceRans.upload(
            eq.codec.rans_encode(sym, sc, eq.EQ_SYM_INT8, spec.cols, 32, 8, prob_bits=pb), dev)
        for batch in (1, 4, 16):
            x = torch.randn(batch, m.cols, device=dev).to(torch.bfloat16)
            y = torch.empty(batch, m.rows, dtype=torch.float32, device=dev)
            st = eq.new_status(dev)
            sec = statistics.mean(time_steps(lambda: eq.decode_gemv(m, x, y, st, stream), steps,
                                             3, flush, stream))
            assert int(st.item()) == 0
            alg = m.compressed_bytes + x.numel() * 2 + y.numel() * 4
            kern = "rans_gemv_tc_kernel" if batch >= 8 else "rans_gemv_kernel"
            out.append({"what": f"fused decode+GEMV, Int8 8192x8192 (~2 bits/param), one row per "
                                f"chunk, {pb}-bit table, batch {batch}",
                        "params": m.numel, "ms": sec * 1e3, "params_per_s": m.numel / sec,
                        "bits_per_param": 8 * m.compressed_bytes / m.numel,
                        "roofline": roofline(alg, sec, peaks, None, m.numel, kern)})
        del m
    return out


# ------------------------------------------------------------------------------------------------
# the reference arm: the oracle itself, on the host cores
# ------------------------------------------------------------------------------------------------

def run_reference(args):
    """The oracle timed on the host cores on the headline workload; rank 0 only.  Each step
    decodes the same bounded sample: the first 16 rows of each of the 224 tensors of the
    LLaMA-2-7B-shaped stack, drawn from the same seeds and coded by the oracle (each sample with
    its own 12-bit table), chunk-parallel over every core."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    wl = synth.WORKLOADS["llama2_7b"]
    conts = []
    for spec in wl.tensors:
        sym, sc = oracle.quantize(spec.generate(row_lo=0, row_hi=16), oracle.E4M3)
        conts.append(oracle.rans_encode(sym, sc, oracle.E4M3, wl.chunk_symbols, wl.streams,
                                        wl.run))
    cores = len(os.sched_getaffinity(0))
    syms = sum(o.numel for o in conts)

    pairs = [(o, c) for o in conts for c in range(o.num_chunks)]

    def step():
        _decode_pairs(pairs, cores)
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    dt = statistics.mean(times)
    v = syms / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "params/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u8->bf16", "data": "synthetic",
            "config": {"workload": "LLaMA-2-7B-shaped stack: 32 layers x {q,k,v,o 4096x4096; "
                                   "gate,up 11008x4096; down 4096x11008}, N(0,0.02) with 1% x8 "
                                   "outliers, Float8-E4M3, per-tensor 12-bit tables, 64 KiB "
                                   "chunks, 128 streams, run 8 -> bf16",
                       "sample": "first 16 rows of each of the 224 tensors per step "
                                 f"({syms} params)", "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": "params/s", "cores": cores, "kind": "oracle",
                             "sample": f"first 16 rows of each of the 224 tensors ({syms} "
                                       "params) per step"},
            "e2e": {"value": v, "unit": "params/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# one kernel alone, for ncu
# ------------------------------------------------------------------------------------------------

def profile_kernel(kind: str, launches: int = 5):
    """A few launches of one kernel on its workload, nothing else: the command ncu captures."""
    import torch

    import decoding_interleaved_rans_b200 as eq
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    if kind == "decode":
        _, h = prepare_rans(eq, "int8_8k")
        t = eq.DeviceRans.upload(h, dev)
        out = torch.empty(h.rows, h.cols, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.decode([t], [out], st)  # noqa: E731
    elif kind == "huff":
        w = synth.WORKLOADS["df11_8k"].tensors[0].generate(row_lo=0, row_hi=2048).ravel()
        dh = eq.DeviceHuff.upload(eq.codec.huff_encode(w), dev)
        ob = torch.empty(dh.n, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.huff_bf16_decode(dh, ob, st)  # noqa: E731
    elif kind == "huffint":
        di = eq.DeviceHuffInt.upload(eq.codec.entrollm_encode(synth.normal(8192, 3072, 0.02, 6), 8),
                                     dev)
        ob = torch.empty(di.n, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.huff_int_decode(di, ob, st)  # noqa: E731
    elif kind in ("gemv", "gemv4", "gemv16"):
        # the 13B MLP down projection, batch 1 / 4 (CUDA cores) or 16 (tensor-core tile)
        batch = {"gemv": 1, "gemv4": 4, "gemv16": 16}[kind]
        wl = synth.WORKLOADS["mlp_13b"]
        spec = wl.tensors[2]
        sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_E4M3)
        t = eq.DeviceRans.upload(eq.codec.rans_encode(sym, sc, eq.EQ_SYM_E4M3, wl.chunk_for(spec),
                                                      wl.streams, wl.run), dev)
        x = torch.randn(batch, t.cols, device=dev).to(torch.bfloat16)
        y = torch.empty(batch, t.rows, dtype=torch.float32, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.decode_gemv(t, x, y, st)  # noqa: E731
    elif kind == "decode12":
        # one LLaMA-2-7B-shaped gate projection (11008 x 4096, N(0, 0.02) with 1% x 8 outliers),
        # E4M3, 12-bit table: the kernel of the headline stack
        spec = next(s for s in synth.WORKLOADS["llama2_7b"].tensors if s.rows == 11008)
        sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_E4M3)
        t = eq.DeviceRans.upload(eq.codec.rans_encode(sym, sc, eq.EQ_SYM_E4M3, 65536, 128, 8), dev)
        out = torch.empty(t.rows, t.cols, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.decode([t], [out], st)  # noqa: E731
    elif kind == "layer":
        # one LLaMA-2-7B-shaped layer (q, k, v, o, gate, up, down; the headline stack's first
        # layer, drawn from the seeded generators and coded on the GPU), decoded in one call: the
        # headline's kernel in the headline's launch shape
        import torch as _t
        wl = synth.WORKLOADS["llama2_7b"]
        ts = []
        for spec in wl.tensors[:7]:
            w = _t.from_numpy(spec.generate()).to(dev)
            sym, sc = eq.quantize_device(w, eq.EQ_SYM_E4M3)
            ts.append(eq.rans_encode_device(sym, sc, eq.EQ_SYM_E4M3, wl.chunk_symbols, wl.streams,
                                            wl.run))
            del w, sym
        outs = [_t.empty(t.rows, t.cols, dtype=_t.bfloat16, device=dev) for t in ts]
        st = eq.new_status(dev)
        fn = lambda: eq.decode(ts, outs, st)  # noqa: E731
    elif kind == "gateup":
        # the 13B MLP block at batch 1: gate and up in the fused kernel (then the down product)
        wl = synth.WORKLOADS["mlp_13b"]
        mats = []
        for spec in wl.tensors:
            sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_E4M3)
            mats.append(eq.DeviceRans.upload(eq.codec.rans_encode(
                sym, sc, eq.EQ_SYM_E4M3, wl.chunk_for(spec), wl.streams, wl.run), dev))
        g, u, d = mats
        x = torch.randn(1, g.cols, device=dev).to(torch.bfloat16)
        y = torch.empty(1, d.rows, dtype=torch.float32, device=dev)
        scratch = torch.empty(eq.mlp_scratch_bytes(g.rows, 1), dtype=torch.uint8, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.mlp_decode(g, u, d, x, y, scratch, st)  # noqa: E731
    elif kind == "gemv7":
        # the ~2-bit Int8 weight, one row per chunk, 7-bit table, batch 1
        wl = synth.WORKLOADS["int8_8k"]
        sym, sc = eq.codec.quantize(wl.tensors[0].generate(), eq.EQ_SYM_INT8, wl.int8_div)
        t = eq.DeviceRans.upload(eq.codec.rans_encode(sym, sc, eq.EQ_SYM_INT8, 8192, 32, 8,
                                                      prob_bits=7), dev)
        x = torch.randn(1, t.cols, device=dev).to(torch.bfloat16)
        y = torch.empty(1, t.rows, dtype=torch.float32, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.decode_gemv(t, x, y, st)  # noqa: E731
    else:
        raise SystemExit(f"unknown kernel {kind}")
    for _ in range(launches):
        fn()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    print(f"profiled {kind}: {launches} launches ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile-kernel", default=None,
                    choices=["decode", "huff", "huffint", "gemv", "gemv4", "gemv16", "decode12",
                             "gemv7", "layer", "gateup"],
                    help="launch one kernel a few times and exit (for ncu)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="headline only, no other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle baselines")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_kernel:
        profile_kernel(args.profile_kernel)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        from decoding_interleaved_rans_b200 import dist
        dist.shutdown()


if __name__ == "__main__":
    main()
