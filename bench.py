"""Throughput of on-device decoding of entropy-coded weights (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one process per GPU)

A step decodes the whole Int8 8192x8192 Laplace weight (H = 2.0 bits, 64 KiB chunks, 128
interleaved streams, run 8, 7-bit frequency table: one pair-table lookup and one renormalisation
per two steps) from its rANS stream in HBM into bf16 in HBM: one eq_decode launch.
Every rank decodes its own copy (weak scaling; the decode has no exchange step).  Timing: CUDA
events on the launching stream around each step, the L2 flushed between steps by writing a
256 MiB buffer, max over ranks.  `e2e` repeats the step through the C ABI with host buffers:
pinned host -> device copy of the coded arrays, decode, device -> host read of the step's status
word (the decoded weight stays in HBM for its layer; `e2e_weights_to_host` also copies it back).
Secondary lines under "also": the same weight with 8- and 12-bit tables, the fused decode-GEMV on the
13B MLP (batch 1/4/16), the MLP block, the DFloat11 decode, the GPU compressor and the block
pipeline, each with its own roofline or comparison.
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

WORKLOAD = "int8_8k"
METRIC = "decoded params/s (rANS decode to bf16)"


KERNEL_SOURCES = {
    "rans_decode_kernel": ["eq_rans_decode.cu", "eq_rans_core.cuh", "eq_dequant.cuh",
                           "eq_internal.cuh"],
    "huff_decode_kernel": ["eq_huff_decode.cu", "eq_dequant.cuh", "eq_internal.cuh"],
    "rans_gemv_kernel": ["eq_rans_gemv.cu", "eq_rans_core.cuh", "eq_dequant.cuh",
                         "eq_internal.cuh"],
}


def kernel_sources_sha(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "decoding_interleaved_rans_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def measured_record(kernel: str):
    """The kernel's committed ncu figures (profiles/traffic.json), or None when its sources
    changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec or rec.get("sources_sha256") != kernel_sources_sha(kernel):
        return None
    return rec


def measured_traffic(kernel: str, units: int):
    """DRAM bytes per launch from the committed ncu capture, scaled to `units` weights."""
    rec = measured_record(kernel)
    return None if rec is None else rec["dram_bytes_per_launch"] * units / rec["weights_per_launch"]


def issue_roofline(kernel: str, units: int, seconds: float, sm_mhz):
    """The instruction-issue roofline beside the HBM one: lane-instructions per weight from the
    committed ncu capture (warp instructions x 32), issued per second, against SMs x 4 schedulers
    x 32 lanes x the SM clock sampled during the timed region."""
    import torch
    rec = measured_record(kernel)
    if rec is None or "warp_instructions_per_launch" not in rec or not sm_mhz:
        return None
    per_weight = 32.0 * rec["warp_instructions_per_launch"] / rec["weights_per_launch"]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peak = sms * 4 * 32 * sm_mhz * 1e6
    achieved = per_weight * units / seconds
    return {"bound": "issue", "lane_instr_per_weight": per_weight, "achieved": achieved,
            "peak": peak, "unit": "lane-instr/s", "frac": achieved / peak, "sms": sms,
            "sm_mhz": sm_mhz, "source": "warp instructions of the committed ncu capture"}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "src": "fallback"}


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


def prepare_rans(eq, wl_name: str, prob_bits: int | None = None):
    """Quantise + encode the workload with the library's own host compressor (no oracle)."""
    wl = synth.WORKLOADS[wl_name]
    spec = wl.tensors[0]
    w = spec.generate()
    fmt = eq.EQ_SYM_E4M3 if wl.symfmt == "e4m3" else eq.EQ_SYM_INT8
    sym, sc = eq.codec.quantize(w, fmt, wl.int8_div)
    del w
    h = eq.codec.rans_encode(sym, sc, fmt, wl.chunk_symbols, wl.streams, wl.run,
                             prob_bits=prob_bits or wl.prob_bits)
    return wl, h


def time_steps(fn, steps, warmup, flush, stream):
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


def run_ours(args):
    import torch

    import decoding_interleaved_rans_b200 as eq
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks = measured_peaks()
    wl, h = prepare_rans(eq, WORKLOAD)
    t = eq.DeviceRans.upload(h, dev)
    out = torch.empty(h.rows, h.cols, dtype=torch.bfloat16, device=dev)
    status = eq.new_status(dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.fill_(1)

    def step():
        eq.decode([t], [out], status, stream)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        clk.wait_first_sample()
        soak_end = time.time() + 1.0  # untimed: let the clocks settle under load
        while time.time() < soak_end:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        barrier(world)
        clk.mark(True)
        times = time_steps(step, args.steps, args.warmup, flush, stream)
        torch.cuda.synchronize()
        clk.mark(False)
    barrier(world)
    assert int(status.item()) == 0, "decode reported corrupt data"
    mean_s = statistics.mean(times)
    mean_s = max_over_ranks(world, mean_s)
    numel = h.rows * h.cols
    alg_bytes = t.compressed_bytes + 2 * numel

    # end to end through the public API with host buffers (pinned), copies inside the timed
    # region: every step decodes the weight straight from host memory (eq_decode_from_host: the
    # coded arrays cross the bus, then decode; splitting them into pieces that decode while the
    # next is copied measured slower, the decode being an eighth of the transfer) and reads back
    # the step's status word (its metric: zero = every chunk decoded cleanly); the bf16 weight
    # stays in HBM for the layer that uses it.  e2e_weights_to_host also copies the whole decoded
    # weight back.
    src = eq.PinnedRans.from_host(h)
    out_host = torch.empty(h.rows, h.cols, dtype=torch.bfloat16).pin_memory()
    st_host = torch.empty(1, dtype=torch.int32).pin_memory()
    h2d = src.h2d_bytes()
    copy_stream = torch.cuda.Stream(dev)

    def e2e_step(full):
        eq.decode_from_host(t, src, out, status, stream, pieces=1, copy_stream=copy_stream)
        st_host.copy_(status, non_blocking=True)
        if full:
            out_host.copy_(out, non_blocking=True)

    e2e_s = max_over_ranks(world, statistics.mean(
        time_steps(lambda: e2e_step(False), max(5, args.steps // 2), 3, flush, stream)))
    assert int(st_host.item()) == 0
    e2e_full_s = max_over_ranks(world, statistics.mean(
        time_steps(lambda: e2e_step(True), max(3, args.steps // 4), 2, flush, stream)))
    assert int(status.item()) == 0
    # CPU offload for comparison (DFloat11 page: its speedups are quoted against offloading the bf16
    # weights to the host): the bf16 weight itself copied host -> device every step
    offload_s = max_over_ranks(world, statistics.mean(
        time_steps(lambda: out.copy_(out_host, non_blocking=True), max(3, args.steps // 4), 2,
                   flush, stream)))

    also = []
    if not args.no_extra:
        # the same weight with 8-bit (one renormalisation per two steps, one lookup per step) and
        # 12-bit tables (a renormalisation point after every step)
        for pb, how in ((8, "renormalisation every second step"),
                        (12, "renormalisation every step")):
            _, hx = prepare_rans(eq, WORKLOAD, prob_bits=pb)
            tx = eq.DeviceRans.upload(hx, dev)
            tsx = time_steps(lambda: eq.decode([tx], [out], status, stream),
                             max(5, args.steps // 2), 3, flush, stream)
            assert int(status.item()) == 0
            sx = statistics.mean(tsx)
            ax = (tx.compressed_bytes + 2 * numel) / sx / 1e9
            also.append({"what": f"same Int8 weight, {pb}-bit table ({how})",
                         "params": numel, "ms": sx * 1e3, "params_per_s": numel / sx, "gbs": ax,
                         "frac_of_peak": ax / peaks["hbm_gbs"],
                         "bits_per_param": 8 * tx.compressed_bytes / numel,
                         "kernel": f"rans_decode_kernel<run 8, Int8, {pb}-bit table>"})
            del tx, hx
        also += extra_measurements(eq, dev, stream, flush, peaks, args)
    barrier(world)
    if rank != 0:
        return
    achieved = alg_bytes / mean_s / 1e9
    line = {
        "metric": METRIC, "value": numel * world / mean_s, "unit": "params/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8->bf16", "data": "synthetic",
        "config": {"workload": "Int8 8192x8192 Laplace(0,0.01) clip 6b, H=2.0 bits, 64 KiB "
                               f"chunks, {wl.streams} streams, run 8, {wl.prob_bits}-bit table -> bf16",
                   "params_per_gpu": numel, "compressed_bytes": t.compressed_bytes,
                   "bits_per_param": 8 * t.compressed_bytes / numel,
                   "l2": "flushed between steps (256 MiB write)", "parallelism": f"replicas x{world}"},
        "gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": measured_traffic("rans_decode_kernel", numel),
                     "peak_src": peaks["src"],
                     "kernel": f"rans_decode_kernel<run 8, Int8, {wl.prob_bits}-bit table>",
                     "alg_bytes_per_launch": alg_bytes},
        "e2e": {"value": numel * world / e2e_s, "unit": "params/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": 4, "ms_per_step": e2e_s * 1e3,
                "result_read_back": "status word; the decoded bf16 weight stays in HBM",
                "path": "eq_decode_from_host (pinned host arrays copied, then decoded)"},
        "e2e_weights_to_host": {"value": numel * world / e2e_full_s, "unit": "params/s",
                                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4 + 2 * numel,
                                "ms_per_step": e2e_full_s * 1e3},
        "offload_comparison": {"bf16_h2d_ms": offload_s * 1e3, "bf16_h2d_bytes": 2 * numel,
                               "coded_h2d_plus_decode_ms": e2e_s * 1e3, "coded_h2d_bytes": h2d,
                               "speedup": offload_s / e2e_s,
                               "pages_claim": "DFloat11: 2.3-46.2x over CPU offload (end to end, "
                                              "their models and hardware)"},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "also": also,
    }
    line["issue_roofline"] = issue_roofline("rans_decode_kernel", numel, mean_s,
                                            line["clocks"].get("sm_mhz"))
    # the same for the lines whose kernel and kind of weight the other captures cover
    for e in also:
        if e["what"].startswith("DFloat11 bf16 decode"):
            e["issue_roofline"] = issue_roofline("huff_decode_kernel", e["params"], e["ms"] / 1e3,
                                                 line["clocks"].get("sm_mhz"))
        elif e["what"] == "fused decode+GEMV, 13B MLP gate/up/down, batch 1":
            e["issue_roofline"] = issue_roofline("rans_gemv_kernel", e["params"], e["ms"] / 1e3,
                                                 line["clocks"].get("sm_mhz"))
    if not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(h, numel)
    print(json.dumps(line), flush=True)


def extra_measurements(eq, dev, stream, flush, peaks, args):
    """Fused decode-GEMV (13B MLP, batch 1/4/16) and DFloat11 decode (8192x28672 bf16)."""
    import torch
    out = []
    steps = max(5, args.steps // 2)
    # DFloat11: algorithmic bytes = EncodedExponent + PackedSignMantissa + Gaps + block_out
    # read, 2 B/weight written
    w = synth.WORKLOADS["df11_8k"].tensors[0].generate().ravel()
    hh = eq.codec.huff_encode(w)
    del w
    dh = eq.DeviceHuff.upload(hh, dev)
    ob = torch.empty(dh.n, dtype=torch.bfloat16, device=dev)
    st = eq.new_status(dev)
    ts = time_steps(lambda: eq.huff_bf16_decode(dh, ob, st, stream), steps, 3, flush, stream)
    assert int(st.item()) == 0
    sec = statistics.mean(ts)
    alg = dh.compressed_bytes + 2 * dh.n
    out.append({"what": "DFloat11 bf16 decode, 8192x28672 N(0,0.015)", "params": dh.n,
                "ms": sec * 1e3, "params_per_s": dh.n / sec, "gbs": alg / sec / 1e9,
                "frac_of_peak": alg / sec / 1e9 / peaks["hbm_gbs"],
                "bits_per_param": 8 * dh.compressed_bytes / dh.n,
                "kernel": "huff_decode_kernel"})
    del dh, ob
    # EntroLLM-style integer weights: a phi3-mini-shaped MLP weight (8192 x 3072, N(0, 0.02)),
    # uint8 and uint4 codes Huffman-coded, decoded by the two-stage kernel
    w = synth.normal(8192, 3072, 0.02, 6)
    for bits in (8, 4):
        hi_ = eq.codec.entrollm_encode(w, bits)
        di = eq.DeviceHuffInt.upload(hi_, dev)
        oi = torch.empty(di.n, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        ti = time_steps(lambda: eq.huff_int_decode(di, oi, st, stream), steps, 3, flush, stream)
        assert int(st.item()) == 0
        sec = statistics.mean(ti)
        alg = di.compressed_bytes + 2 * di.n
        out.append({"what": f"EntroLLM-style uint{bits} codes, Huffman-coded, 8192x3072 N(0,0.02)",
                    "params": di.n, "ms": sec * 1e3, "params_per_s": di.n / sec,
                    "gbs": alg / sec / 1e9, "frac_of_peak": alg / sec / 1e9 / peaks["hbm_gbs"],
                    "bits_per_param": 8 * di.compressed_bytes / di.n,
                    "pages_context": "EntroLLM: 5.58 bits/param from uint8 on phi3-mini (real "
                                     "weights, Jetson)",
                    "kernel": "huff_decode_kernel<integer codes>"})
        del di, oi, hi_
    del w
    # super weights: the Int8 workload with 6 planted outliers (50-200x the typical weight), kept
    # exactly in the patch list and out of their rows' scales; the decode writes them back
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
    tsw = time_steps(lambda: eq.decode([ts_], [osw], st, stream), steps, 3, flush, stream)
    assert int(st.item()) == 0
    sec = statistics.mean(tsw)
    alg = ts_.compressed_bytes + 2 * ts_.numel
    out.append({"what": "Int8 8192x8192 with 6 super weights (patch list written back in the "
                        f"decode epilogue), {wl.prob_bits}-bit table", "params": ts_.numel,
                "ms": sec * 1e3,
                "params_per_s": ts_.numel / sec, "gbs": alg / sec / 1e9,
                "frac_of_peak": alg / sec / 1e9 / peaks["hbm_gbs"], "super_weights": int(pidx.size),
                "zero_symbols_in_their_rows_without_exclusion": collapsed,
                "kernel": f"rans_decode_kernel<run 8, Int8, {wl.prob_bits}-bit table> + patch "
                          "epilogue"})
    del ts_, osw, hs
    # GPU compressor: fp32 weights in HBM -> quantise, histogram, frequency table (host), rANS
    # plan + encode; wall clock around the whole call (it reads the word total back once)
    wl = synth.WORKLOADS["int8_8k"]
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
    # the whole LLaMA-2-7B-shaped stack (32 layers x 7 tensors, 6.48 G weights, N(0, 0.02) with 1%
    # outliers x 8, E4M3, 12-bit tables): weights drawn on the GPU, quantised and coded by the
    # GPU compressor, then every tensor decoded to bf16 in one eq_decode call
    wl7 = synth.WORKLOADS["llama2_7b"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    full, outs7 = [], []
    for spec in wl7.tensors:
        wt = torch.randn(spec.rows, spec.cols, device=dev, generator=gen) * 0.02
        wt = torch.where(torch.rand(spec.rows, spec.cols, device=dev, generator=gen) < 0.01,
                         wt * 8.0, wt)
        sym, sc = eq.quantize_device(wt, eq.EQ_SYM_E4M3)
        full.append(eq.rans_encode_device(sym, sc, eq.EQ_SYM_E4M3, wl7.chunk_symbols, wl7.streams,
                                          wl7.run))
        outs7.append(torch.empty(spec.rows, spec.cols, dtype=torch.bfloat16, device=dev))
        del wt, sym, sc
    st = eq.new_status(dev)
    n7 = sum(t.numel for t in full)
    coded7 = sum(t.compressed_bytes for t in full)
    ts7 = time_steps(lambda: eq.decode(full, outs7, st, stream), 3, 2, flush, stream)
    assert int(st.item()) == 0
    sec = statistics.mean(ts7)
    alg = coded7 + 2 * n7
    out.append({"what": "LLaMA-2-7B-shaped stack, 224 tensors, E4M3 12-bit tables, one eq_decode "
                        "call", "params": n7, "ms": sec * 1e3, "params_per_s": n7 / sec,
                "gbs": alg / sec / 1e9, "frac_of_peak": alg / sec / 1e9 / peaks["hbm_gbs"],
                "bits_per_param": 8 * coded7 / n7, "data": "drawn on the GPU (torch generator)",
                "kernel": "rans_decode_kernel<run 8, E4M3, 12-bit table>"})
    del full, outs7
    torch.cuda.empty_cache()
    # block-by-block decode overlapped with the block's forward GEMMs (4 LLaMA-2-7B-shaped layers,
    # coded on the GPU): compute alone on resident bf16 weights, decode then compute, overlapped
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
            for w in ws:
                torch.matmul(xt[:, :w.shape[1]], w.t())
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
    # fused decode + GEMV over the three 13B MLP weights (gate, up 13824x5120; down 5120x13824);
    # algorithmic bytes = the coded weights read (+ x and y)
    wl = synth.WORKLOADS["mlp_13b"]
    mats = []
    for spec in wl.tensors:
        sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_E4M3)
        h = eq.codec.rans_encode(sym, sc, eq.EQ_SYM_E4M3, wl.chunk_for(spec), wl.streams, wl.run)
        mats.append(eq.DeviceRans.upload(h, dev))
        del sym, sc, h
    params = sum(m.numel for m in mats)
    coded = sum(m.compressed_bytes for m in mats)
    for batch in wl.batches:
        xs = [torch.randn(batch, m.cols, device=dev).to(torch.bfloat16) for m in mats]
        ys = [torch.empty(batch, m.rows, dtype=torch.float32, device=dev) for m in mats]
        st = eq.new_status(dev)

        def layer():
            for m, x, y in zip(mats, xs, ys):
                eq.decode_gemv(m, x, y, st, stream)
        ts = time_steps(layer, steps, 3, flush, stream)
        assert int(st.item()) == 0
        sec = statistics.mean(ts)
        alg = coded + sum(x.numel() * 2 for x in xs) + sum(y.numel() * 4 for y in ys)
        out.append({"what": f"fused decode+GEMV, 13B MLP gate/up/down, batch {batch}",
                    "params": params, "ms": sec * 1e3, "params_per_s": params / sec,
                    "gbs": alg / sec / 1e9, "frac_of_peak": alg / sec / 1e9 / peaks["hbm_gbs"],
                    "bits_per_param": 8 * coded / params, "kernel": "rans_gemv_kernel",
                    "launches_per_step": len(mats)})
        # the whole MLP block: gate and up products, SiLU gate to bf16, down product
        byname = {spec.name: m for spec, m in zip(wl.tensors, mats)}
        g, u, d = byname["gate"], byname["up"], byname["down"]
        xb = xs[[spec.name for spec in wl.tensors].index("gate")]
        yb = torch.empty(batch, d.rows, dtype=torch.float32, device=dev)
        scratch = torch.empty(eq.mlp_scratch_bytes(g.rows, batch), dtype=torch.uint8, device=dev)
        ts = time_steps(lambda: eq.mlp_decode(g, u, d, xb, yb, scratch, st, stream), steps, 3,
                        flush, stream)
        assert int(st.item()) == 0
        sec = statistics.mean(ts)
        out.append({"what": f"MLP block from coded weights (13B: gate, up, SiLU gate, down), "
                            f"batch {batch}",
                    "params": params, "ms": sec * 1e3, "params_per_s": params / sec,
                    "kernel": "rans_gemv_kernel x3 + silu_mul_kernel", "launches_per_step": 4})
    del mats
    # fused decode + GEMV over the ~2-bit Int8 8192x8192 weight, one row per chunk and 32 streams
    # (the fused kernel's layout), with the 7-bit pair table and with the 12-bit table
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
            ts = time_steps(lambda: eq.decode_gemv(m, x, y, st, stream), steps, 3, flush, stream)
            assert int(st.item()) == 0
            sec = statistics.mean(ts)
            alg = m.compressed_bytes + x.numel() * 2 + y.numel() * 4
            out.append({"what": f"fused decode+GEMV, Int8 8192x8192 (~2 bits/param), one row per "
                                f"chunk, {pb}-bit table, batch {batch}",
                        "params": m.numel, "ms": sec * 1e3, "params_per_s": m.numel / sec,
                        "gbs": alg / sec / 1e9, "frac_of_peak": alg / sec / 1e9 / peaks["hbm_gbs"],
                        "bits_per_param": 8 * m.compressed_bytes / m.numel,
                        "kernel": "rans_gemv_tc_kernel" if batch >= 8 else "rans_gemv_kernel"})
        del m
    return out


def cpu_baseline(h, numel, seconds_budget: float = 20.0):
    """The oracle's decoder (plain C, chunk-parallel over the host cores) on the same container."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    o = oracle.RansTensor(h.rows, h.cols, h.symfmt, h.prob_bits, h.chunk_symbols, h.streams,
                          h.run, h.freqs, h.states, h.word_off, h.words, h.scales)
    n_chunks = o.num_chunks
    # time a small probe, then size the sample to stay within the budget
    probe = list(range(min(n_chunks, cores)))
    t0 = time.perf_counter()
    oracle.rans_decode_bf16(o, chunks=probe, threads=cores)
    per_chunk = (time.perf_counter() - t0) / max(1, len(probe)) * cores
    take = max(1, min(n_chunks, int(seconds_budget / max(per_chunk / cores, 1e-9))))
    chunks = list(range(take))
    t0 = time.perf_counter()
    rc, _ = oracle.rans_decode_bf16(o, chunks=chunks, threads=cores)
    dt = time.perf_counter() - t0
    assert rc == 0
    syms = sum(min(h.chunk_symbols, numel - c * h.chunk_symbols) for c in chunks)
    return {"value": syms / dt, "unit": "params/s", "cores": cores, "kind": "oracle",
            "sample": f"{take} of {n_chunks} chunks ({syms} params), decode + dequant to bf16, "
                      f"{cores} threads", "seconds": dt}


def run_reference(args):
    """The oracle timed on the host cores, same workload/metric; rank 0 only."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    wl = synth.WORKLOADS[WORKLOAD]
    sym, sc = oracle.quantize(wl.tensors[0].generate(), oracle.INT8, wl.int8_div)
    o = oracle.rans_encode(sym, sc, oracle.INT8, wl.chunk_symbols, wl.streams, wl.run,
                           prob_bits=wl.prob_bits)
    h = o
    cores = len(os.sched_getaffinity(0))
    take = min(o.num_chunks, max(cores * 4, 64))
    chunks = list(range(take))
    for _ in range(args.warmup):
        oracle.rans_decode_bf16(o, chunks=chunks[:cores], threads=cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        rc, _ = oracle.rans_decode_bf16(o, chunks=chunks, threads=cores)
        times.append(time.perf_counter() - t0)
        assert rc == 0
    dt = statistics.mean(times)
    syms = take * h.chunk_symbols
    v = syms / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "params/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u8->bf16", "data": "synthetic",
            "config": {"workload": "Int8 8192x8192 Laplace(0,0.01) clip 6b, H=2.0 bits, 64 KiB "
                                   f"chunks, 128 streams, run 8, {wl.prob_bits}-bit table -> bf16",
                       "sample_chunks": take, "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": "params/s", "cores": cores, "kind": "oracle",
                             "sample": f"{take} of {o.num_chunks} chunks per step"},
            "e2e": {"value": v, "unit": "params/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def profile_kernel(kind: str, launches: int = 5):
    """A few launches of one kernel on its workload, nothing else: the command ncu captures."""
    import torch

    import decoding_interleaved_rans_b200 as eq
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    if kind == "decode":
        _, h = prepare_rans(eq, WORKLOAD)
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
    elif kind in ("gemv", "gemv16"):
        # the 13B MLP down projection, batch 1 (CUDA cores) or 16 (tensor-core tile)
        batch = 16 if kind == "gemv16" else 1
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
        # E4M3, 12-bit table: the decode of the model-stack line
        spec = next(s for s in synth.WORKLOADS["llama2_7b"].tensors if s.rows == 11008)
        sym, sc = eq.codec.quantize(spec.generate(), eq.EQ_SYM_E4M3)
        t = eq.DeviceRans.upload(eq.codec.rans_encode(sym, sc, eq.EQ_SYM_E4M3, 65536, 128, 8), dev)
        out = torch.empty(t.rows, t.cols, dtype=torch.bfloat16, device=dev)
        st = eq.new_status(dev)
        fn = lambda: eq.decode([t], [out], st)  # noqa: E731
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
                    choices=["decode", "huff", "gemv", "gemv16", "decode12", "gemv7"],
                    help="launch one kernel a few times and exit (for ncu)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the GEMV / DFloat11 lines")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline")
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
