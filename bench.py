"""Benchmark of the Huffman weight-decoding hot path on B200.

One step = one pass of the whole hot path over the 4096x4096 4-bit Laplace
tensor (32 word-interleaved lanes per 8192-symbol chunk):
    decode -> packed uint4 codes, decode -> dequantize -> bf16, and the fused
    decode -> dequantize -> GEMV (batch 1),
each through the C ABI of libentro.  Inputs are resident in HBM.  The working
set is made larger than L2: 40 replicas of the encoded tensor (160 MB of coded
payload alone, against a 126 MB L2) and of its outputs rotate, each kernel on
the next replica, so every kernel reads coded words that no recent kernel
touched and writes outputs whose lines must first be evicted -- the steady
state of decoding a model much larger than L2 (no flush kernel, so the decode
code stays warm as it would in serving).  Times come from CUDA events on the
launching stream: the K timed steps run back to back between one pair of
events, and each kernel's own duration is the mean over K launches of it back
to back (events between the calls would add gaps of their own, ~2.5 us each).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

With N > 1 (torchrun) every rank decodes its own replica of the workload (the
chunks are independent problems; no data-path collective), and the line
reports the whole-job rate from the slowest rank ("weak" scaling).
--impl reference times the CPU oracle doing the same step on a bounded sample.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "decoded Gsym/s and % HBM roofline (Huffman decode+dequant); fused GEMV tok/s"
WORKLOAD = "laplace_4096x4096_u4"
REPLICAS = 40
NOMINAL_HBM_GBS = 7700.0  # B200 HBM3e, HGX figure (context beside the measured copy peak)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ distributed plumbing

def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dist, dist.get_rank(), ws, int(os.environ.get("LOCAL_RANK", "0"))
    return None, 0, 1, 0


def _max_over_ranks(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(dist, device):
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms while running."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.bus = ""
        if device.type == "cuda":
            pr = torch.cuda.get_device_properties(device)
            self.bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10 and (not self.bus or parts[0].lower().endswith(self.bus[-10:])):
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=5)
        rows = self.rows
        if not rows:
            return {"samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        util = [num(r[4]) for r in rows]
        loaded = [num(r[1]) for r in rows if num(r[4]) and num(r[4]) > 0 and num(r[1]) is not None] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": sorted(reasons), "samples": len(rows),
                "util_max": max(u for u in util if u is not None) if any(u is not None for u in util) else None}


# ------------------------------------------------------------------ CPU oracle leg

def _oracle_step(blob: bytes, chunks, threads: int, x_bits: np.ndarray):
    """The oracle on host cores: decode the sample's chunks to codes, to bf16 weights,
    and through the fp64 GEMV, chunk ranges split over threads (the EntroLLM
    multi-threaded chunk decoder).  Returns symbols processed."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    p = oracle.params(blob)
    C, K = p["chunk_symbols"], p["cols"]
    c0, c1 = chunks
    bounds = np.linspace(c0, c1, threads + 1).astype(int)

    def work(i):
        a, b = int(bounds[i]), int(bounds[i + 1])
        if a >= b:
            return 0
        q = oracle.decode_chunks(blob, a, b)                     # pass 1: codes
        q2 = oracle.decode_chunks(blob, a, b)                    # pass 2: codes -> bf16
        wb = oracle.dequant_bf16(q2, p["scale"], p["zero"])
        q3 = oracle.decode_chunks(blob, a, b)                    # pass 3: -> GEMV over the rows
        wg = oracle.dequant_bf16(q3, p["scale"], p["zero"]).reshape(-1, K)
        oracle.gemv(wg, x_bits)
        return q.size + wb.size + wg.size

    with ThreadPoolExecutor(threads) as ex:
        return sum(ex.map(work, range(threads)))


def cpu_baseline(seconds: float = 12.0):
    import oracle
    W = workloads.get(WORKLOAD)
    spec = W.tensors[0]
    w = workloads.weights(W, spec).numpy()
    t_enc = time.perf_counter()
    blob = oracle.encode(w, W.bits, W.quant_mode, W.max_len, W.fmt, W.chunk_symbols(spec.cols))
    t_enc = time.perf_counter() - t_enc
    p = oracle.params(blob)
    x_bits = workloads.bf16_bits(workloads.activations(0, 1, spec.cols))
    threads = max(1, min(os.cpu_count() or 1, 64))
    n_chunks = p["n_chunks"]
    total, t0, reps = 0, time.perf_counter(), 0
    while True:
        total += _oracle_step(blob, (0, n_chunks), threads, x_bits)
        reps += 1
        if time.perf_counter() - t0 >= seconds or reps >= 8:
            break
    dt = time.perf_counter() - t0
    # one thread on a 1/32 sample of the chunks (the sequential decoder's rate)
    sample1 = (0, max(1, n_chunks // 32))
    total1, t1, reps1 = 0, time.perf_counter(), 0
    while True:
        total1 += _oracle_step(blob, sample1, 1, x_bits)
        reps1 += 1
        if time.perf_counter() - t1 >= seconds / 4 or reps1 >= 4:
            break
    dt1 = time.perf_counter() - t1
    return {"value": total / dt / 1e9, "unit": "Gsym/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} pass(es) of the whole {spec.rows}x{spec.cols} tensor "
                      f"({n_chunks} chunks; codes, bf16 and GEMV passes), chunk ranges over {threads} threads, "
                      f"{dt:.1f} s",
            "single_thread": {"value": total1 / dt1 / 1e9, "unit": "Gsym/s", "cores": 1,
                              "sample": f"{reps1} pass(es) of chunks {sample1[0]}..{sample1[1]} "
                                        f"(codes, bf16 and GEMV passes), {dt1:.1f} s"},
            "oracle_encode_s": round(t_enc, 3)}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    W = workloads.get(WORKLOAD)
    spec = W.tensors[0]
    w = workloads.weights(W, spec).numpy()
    blob = oracle.encode(w, W.bits, W.quant_mode, W.max_len, W.fmt, W.chunk_symbols(spec.cols))
    p = oracle.params(blob)
    x_bits = workloads.bf16_bits(workloads.activations(0, 1, spec.cols))
    threads = max(1, min(os.cpu_count() or 1, 64))
    sample = (0, min(p["n_chunks"], 256))                         # 1/8 of the tensor per step
    for _ in range(args.warmup):
        _oracle_step(blob, sample, threads, x_bits)
    t0 = time.perf_counter()
    syms = 0
    for _ in range(args.steps):
        syms += _oracle_step(blob, sample, threads, x_bits)
    dt = time.perf_counter() - t0
    value = syms / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "Gsym/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u4->bf16/fp64",
            "data": "synthetic", "config": _config(W, spec, p["chunk_symbols"]),
            "cpu_baseline": {"value": value, "unit": "Gsym/s", "cores": threads, "kind": "oracle",
                             "sample": f"chunks {sample[0]}..{sample[1]} of {p['n_chunks']} per step "
                                       f"(codes, bf16 and GEMV passes) over {threads} threads"},
            "e2e": {"value": value, "unit": "Gsym/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _config(W, spec, chunk):
    return {"workload": W.name, "shape": [spec.rows, spec.cols], "bits": W.bits, "quant": "asymmetric",
            "max_code_len": W.max_len, "chunk_symbols": chunk, "lanes": 32, "gemv_batch": 1,
            "l2": f"inputs larger than L2: {REPLICAS} rotating replicas (image + outputs), "
                  "each kernel on a different replica; no flush"}


# ------------------------------------------------------------------ native arm

def run_native(args, dist, rank, world, local_rank):
    import huffman_decode_canonical_b200 as entro
    entro.set_overlap(not args.no_overlap)

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    W = workloads.get(WORKLOAD)
    spec = W.tensors[0]
    chunk = W.chunk_symbols(spec.cols)
    w = workloads.weights(W, spec).numpy()
    blob = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=W.fmt,
                             chunk_symbols=chunk)
    info = blob.info()
    reps = [entro.upload(blob, device=device) for _ in range(REPLICAS)]
    dt = reps[0]
    n = info["n"]
    codes = [r.empty_codes() for r in reps]
    bf = [r.empty_bf16() for r in reps]
    x = workloads.activations(0, 1, spec.cols).to(device)
    y = [torch.empty((1, spec.rows), dtype=torch.float32, device=device) for _ in reps]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    counter = [0]

    def next_rep():
        r = counter[0] % REPLICAS
        counter[0] += 1
        return r

    kernels = [("codes", lambda r: reps[r].decode_codes(out=codes[r], status=status)),
               ("bf16", lambda r: reps[r].decode_dequant_bf16(out=bf[r], status=status)),
               ("gemv", lambda r: reps[r].decode_gemv(x, y=y[r], status=status))]

    def step():
        for _, fn in kernels:
            fn(next_rep())

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device)
    clocks.start()
    # untimed burn-in so that clock samples cover a loaded GPU even for short runs
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        step()
        torch.cuda.synchronize(device)
    # The K steps run back to back between one pair of events (events between
    # the calls would add their own gaps); the GPU is kept busy while the host
    # enqueues them, so the events measure device time only.
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(dist, device)
    torch.cuda.synchronize(device)
    wall0 = time.perf_counter()
    torch.cuda._sleep(int(args.steps * 300e-6 * 2.0e9))
    ev0.record(stream)
    for s in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    wall = time.perf_counter() - wall0
    _barrier(dist, device)
    step_ms = ev0.elapsed_time(ev1) / args.steps
    # Each kernel's own duration: K launches of it back to back (rotating
    # replicas), between one pair of events.
    mean_ms = {}
    for name, fn in kernels:
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(device)
        torch.cuda._sleep(int(args.steps * 100e-6 * 2.0e9))
        k0.record(stream)
        for s in range(args.steps):
            fn(next_rep())
        k1.record(stream)
        torch.cuda.synchronize(device)
        mean_ms[name] = k0.elapsed_time(k1) / args.steps
    clk = clocks.stop()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    step_ms_max = _max_over_ranks(dist, step_ms, device)
    bf16_ms_max = _max_over_ranks(dist, mean_ms["bf16"], device)

    # algorithmic bytes per launch: coded bits (no lane padding) + chunk index + output
    coded = info["coded_bits"] / 8.0
    index = info["index_bytes"]
    alg = {"codes": coded + index + dt.codes_nbytes(), "bf16": coded + index + 2.0 * n,
           "gemv": coded + index + 2.0 * spec.cols + 4.0 * spec.rows}
    peak, peak_kind = _peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    kern = {}
    for k in mean_ms:
        us = 1e3 * mean_ms[k]
        gbs = alg[k] / (mean_ms[k] * 1e-3) / 1e9
        kern[k] = {"us": round(us, 3), "gsym_s": round(n / (mean_ms[k] * 1e-3) / 1e9, 2),
                   "alg_bytes": int(alg[k]), "achieved_gbs": round(gbs, 1), "hbm_frac": round(gbs / peak, 4),
                   "issue_bound": _issue_ceiling(k, n, mean_ms[k], clk.get("sm_mhz"), sms)}
    kern["gemv"]["tok_s"] = round(1.0 / (mean_ms["gemv"] * 1e-3), 1)
    achieved = alg["bf16"] / (bf16_ms_max * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "lanes_kernel<4, bf16> (decode + dequant to bf16)",
                "achieved": round(achieved, 1), "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs",
                "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": _traffic("bf16"),
                "peak_nominal": NOMINAL_HBM_GBS, "frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                "issue_bound": kern["bf16"]["issue_bound"]}

    e2e = _e2e(entro, blob, dt, device, stream, args, n, codes[0], bf[0], x, y[0], status)
    e2e["value"] = _max_over_ranks(dist, -e2e["value"], device) * -1 if dist is not None else e2e["value"]
    if rank != 0:
        return 0
    cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline()
    value = world * 3 * n / (step_ms_max * 1e-3) / 1e9
    line = {"metric": METRIC, "value": round(value, 3), "unit": "Gsym/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u4 codes -> bf16 / fp32 accumulate",
            "data": "synthetic", "config": _config(W, spec, chunk), "launch_overlap": not args.no_overlap,
            "value_definition": "symbols decoded per second over the step (3 passes of n = 16.8M symbols); "
                                "K steps back to back between one pair of CUDA events",
            "kernels_timing": "each kernel alone: K launches back to back (rotating replicas) between one "
                              "pair of CUDA events, per-launch mean",
            "kernels": kern,
            "bits_per_weight": {"coded": round(info["coded_bits"] / n, 4),
                                "payload": round(8.0 * info["payload_bytes"] / n, 4),
                                "all_in": round(8.0 * (info["payload_bytes"] + info["index_bytes"] + 16384) / n, 4)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 3 * args.steps,
            "clocks": clk, "wall_s_timed": round(wall, 4)}
    print(json.dumps(line), flush=True)
    return 0


def _kernel_source_hash() -> str:
    """Hash of the kernel sources with comments and whitespace removed (a comment edit
    does not change the kernels whose traffic profiles/traffic.json records)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in ("huffman_decode_canonical_b200/csrc/decode.cu", "huffman_decode_canonical_b200/csrc/blob_format.h"):
        with open(os.path.join(ROOT, rel)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def _profile_record(key: str, kernel: str):
    """A per-launch figure of `kernel` (`key`: "kernels" = DRAM bytes, "warp_inst" = warp
    instructions) from the committed ncu summary, or None when the summary was taken on
    other kernel sources (profiles/traffic.json records their hash)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("source_sha256_16") != _kernel_source_hash():
            return None
        return t[key].get(kernel)
    except Exception:
        return None


def _traffic(kernel: str):
    return _profile_record("kernels", kernel)


def _issue_ceiling(kernel: str, n: int, ms: float, sm_mhz, sms: int):
    """The instruction-issue bound of a decode kernel: every SM scheduler issues one warp
    instruction per clock, so with I warp instructions per launch (ncu
    smsp__inst_executed.sum) the launch takes at least I / (4 * SMs * clock).  Reported
    as symbols/s at that bound and the fraction of it achieved; None without a record
    for these kernel sources."""
    inst = _profile_record("warp_inst", kernel)
    if not inst or not sm_mhz:
        return None
    lane_inst_per_sym = 32.0 * inst / n
    ceiling = 4 * 32 * sms * sm_mhz * 1e6 / lane_inst_per_sym
    achieved = n / (ms * 1e-3)
    return {"lane_inst_per_sym": round(lane_inst_per_sym, 2), "ceiling_gsym_s": round(ceiling / 1e9, 1),
            "achieved_gsym_s": round(achieved / 1e9, 1), "frac": round(achieved / ceiling, 4),
            "clock_mhz": sm_mhz, "sms": sms}


def _e2e(entro, blob, dt, device, stream, args, n, codes, bf, x, y, status):
    """The same step through the public API with host buffers: upload the blob's device
    image from host memory, decode the three ways, read every result back."""
    import ctypes
    host_codes = torch.empty(codes.numel(), dtype=torch.uint8, pin_memory=True)
    host_bf = torch.empty(bf.shape, dtype=torch.bfloat16, pin_memory=True)
    host_y = torch.empty(y.shape, dtype=torch.float32, pin_memory=True)
    nbytes = blob.device_bytes()
    mem = torch.empty(nbytes, dtype=torch.uint8, device=device)
    lib = entro.lib()

    copy_stream = torch.cuda.Stream(device)
    drained = torch.cuda.Event()  # the previous step's reads of codes / bf / y are done
    drained.record(copy_stream)

    def one():
        # results go back on a second stream as soon as each decode is done, so the
        # transfers overlap the later decodes (and the next step's upload)
        h = ctypes.c_void_p()
        r = lib.entro_upload(blob._h, ctypes.c_void_p(mem.data_ptr()), nbytes, ctypes.c_void_p(stream.cuda_stream),
                             ctypes.byref(h))
        assert r == 0
        st = ctypes.c_void_p(status.data_ptr())
        s = ctypes.c_void_p(stream.cuda_stream)
        stream.wait_event(drained)
        done = [torch.cuda.Event() for _ in range(3)]
        assert lib.entro_decode_codes(h, ctypes.c_void_p(codes.data_ptr()), st, s) == 0
        done[0].record(stream)
        assert lib.entro_decode_dequant_bf16(h, ctypes.c_void_p(bf.data_ptr()), st, s) == 0
        done[1].record(stream)
        assert lib.entro_decode_gemv(h, ctypes.c_void_p(x.data_ptr()), 1, ctypes.c_void_p(y.data_ptr()), st, s) == 0
        done[2].record(stream)
        with torch.cuda.stream(copy_stream):
            for ev, dst, src in zip(done, (host_codes, host_bf, host_y), (codes, bf, y)):
                copy_stream.wait_event(ev)
                dst.copy_(src, non_blocking=True)
            drained.record(copy_stream)
        lib.entro_tensor_free(h)

    reps = max(3, min(args.steps, 20))
    for _ in range(2):
        one()
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    for _ in range(reps):
        one()
    torch.cuda.synchronize(device)
    dt_s = (time.perf_counter() - t0) / reps
    d2h = host_codes.numel() + 2 * host_bf.numel() + 4 * host_y.numel()
    return {"value": round(3 * n / dt_s / 1e9, 3), "unit": "Gsym/s", "h2d_bytes_per_step": int(nbytes),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(1e3 * dt_s, 4),
            "note": "entro_upload from the blob's pageable host bytes (decode tables built on the host), "
                    "three decodes, results copied to pinned host memory on a second stream as each decode "
                    "finishes; wall clock per step"}


def run_single_stream(args, dist, rank, world, local_rank):
    """The 1024x1024 8-bit tensor in the one-bitstream-per-chunk format (4096-symbol
    chunks): one step = decode to uint8 codes + decode to bf16, 40 rotating replicas."""
    import huffman_decode_canonical_b200 as entro
    entro.set_overlap(not args.no_overlap)
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    W = workloads.get(args.workload)
    spec = W.tensors[0]
    w = workloads.weights(W, spec).numpy()
    blob = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=W.fmt,
                             chunk_symbols=W.chunk_symbols(spec.cols), lanes=W.lanes)
    info = blob.info()
    reps = [entro.upload(blob, device=device) for _ in range(REPLICAS)]
    codes = [r.empty_codes() for r in reps]
    bf = [r.empty_bf16() for r in reps]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    counter = [0]

    def step():
        for fn in (lambda r: reps[r].decode_codes(out=codes[r], status=status),
                   lambda r: reps[r].decode_dequant_bf16(out=bf[r], status=status)):
            fn(counter[0] % REPLICAS)
            counter[0] += 1

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device)
    clocks.start()
    t_end = time.perf_counter() + 1.0  # burn-in so that clock samples cover a loaded GPU
    while time.perf_counter() < t_end:
        step()
        torch.cuda.synchronize(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(dist, device)
    torch.cuda.synchronize(device)
    torch.cuda._sleep(int(args.steps * 200e-6 * 2.0e9))
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    _barrier(dist, device)
    clk = clocks.stop()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    step_ms = _max_over_ranks(dist, ev0.elapsed_time(ev1) / args.steps, device)
    if rank != 0:
        return 0
    n = info["n"]
    line = {"metric": METRIC, "value": round(world * 2 * n / (step_ms * 1e-3) / 1e9, 3), "unit": "Gsym/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8 codes -> bf16",
            "data": "synthetic", "launch_overlap": not args.no_overlap,
            "config": {"workload": W.name, "rows": spec.rows, "cols": spec.cols, "format": "single stream",
                       "chunk_symbols": W.chunk_symbols(spec.cols), "replicas": REPLICAS},
            "value_definition": "symbols decoded per second over the step (decode to codes + decode to bf16)",
            "bits_per_weight": {"coded": round(info["coded_bits"] / n, 4)},
            "gpu_launches": 2 * args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def run_model(args, dist, rank, world, local_rank):
    """One step = one grouped launch over every tensor of a model-shaped workload:
    the fused GEMV of a whole decode step (tok/s) or a whole-model decode to bf16."""
    import huffman_decode_canonical_b200 as entro
    entro.set_overlap(not args.no_overlap)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from model_helpers import encode_workload

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    W = workloads.get(args.workload)
    dts, infos, t_enc = encode_workload(entro, W, device=device, limit=args.tensors or None)
    n = sum(i["n"] for i in infos)
    coded = sum(i["coded_bits"] for i in infos) / 8.0
    payload = sum(i["payload_bytes"] for i in infos)
    index = sum(i["index_bytes"] for i in infos)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    gemv = args.workload != "smollm_1p7b_u8"
    if gemv:
        xs = [workloads.activations(W.seed, args.batch, d.cols).to(device) for d in dts]
        ys = [torch.empty((args.batch, d.rows), dtype=torch.float32, device=device) for d in dts]
        g = entro.Group(dts, entro.GROUP_GEMV, xs=xs, ys=ys, batch=args.batch)
        out_bytes = sum(2 * x.numel() for x in xs) + sum(4 * y.numel() for y in ys)
    else:
        outs = [torch.empty((d.rows, d.cols), dtype=torch.bfloat16, device=device) for d in dts]
        g = entro.Group(dts, entro.GROUP_BF16, outs=outs)
        out_bytes = 2 * n
    for _ in range(args.warmup):
        g.launch(status=status)
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device)
    clocks.start()
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        g.launch(status=status)
        torch.cuda.synchronize(device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    _barrier(dist, device)
    torch.cuda.synchronize(device)
    torch.cuda._sleep(int(args.steps * 100e-6 * 2.0e9))
    for s_ in range(args.steps):
        ev[s_].record(stream)
        g.launch(status=status)
    ev[args.steps].record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    ms = sum(ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)) / args.steps
    ms = _max_over_ranks(dist, ms, device)
    if rank != 0:
        return 0
    peak, peak_kind = _peaks()
    alg = coded + index + out_bytes
    achieved = alg / (ms * 1e-3) / 1e9
    partial = " (first %d tensors)" % len(dts) if args.tensors else ""
    line = {"metric": METRIC, "value": round(world / (ms * 1e-3), 2) if gemv else round(world * n / (ms * 1e-3) / 1e9, 2),
            "unit": (f"tok/s (batch {args.batch})" if gemv else "Gsym/s") + partial, "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": f"u{W.bits} codes -> bf16" + (" x bf16 -> fp32" if gemv else ""),
            "data": "synthetic", "launch_overlap": not args.no_overlap,
            "config": {"workload": W.name, "tensors": len(dts), "symbols": n, "bits": W.bits,
                                            "batch": args.batch if gemv else None,
                                            "l2": "working set larger than L2 (whole model)"},
            "gsym_s": round(n / (ms * 1e-3) / 1e9, 1),
            "bits_per_weight": {"coded": round(8 * coded / n, 4), "payload": round(8 * payload / n, 4)},
            "roofline": {"bound": "hbm", "kernel": "lanes_kernel grouped launch", "achieved": round(achieved, 1),
                         "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": None},
            "host_encode_s": round(t_enc, 2), "gpu_launches": args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch without overlap (programmatic dependent launch, on by default)")
    ap.add_argument("--workload", default=WORKLOAD, choices=[WORKLOAD, "t4_1024x1024_u8", "smollm_1p7b_u8",
                                                             "mistral_7b_u4", "phi3_mini_u8"],
                    help="other workloads (not the default line): the 1024x1024 single-stream tensor, or "
                         "model-scale workloads timed as one grouped launch per step")
    ap.add_argument("--batch", type=int, default=1, help="GEMV batch for the model-scale GEMV workloads")
    ap.add_argument("--tensors", type=int, default=0, help="model-scale workloads: only the first N tensors")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    dist, rank, world, local_rank = _dist()
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        if args.workload == "t4_1024x1024_u8":
            return run_single_stream(args, dist, rank, world, local_rank)
        if args.workload != WORKLOAD:
            return run_model(args, dist, rank, world, local_rank)
        return run_native(args, dist, rank, world, local_rank)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
