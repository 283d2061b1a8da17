"""Benchmark of the Huffman weight-decoding hot path on B200.

The line's headline is the fused-GEMV rate on a Mistral-7B-shaped model: one
simulated token-generation step = the fused decode ->
dequantize -> GEMV of all 224 projection tensors (32 layers of q, k, v, o,
gate, up, down; Laplace weights, tensor-level asymmetric 4-bit codes, one
Huffman code per tensor, 6.98 G weights, ~1.42 GB of coded bytes) against bf16
activations at batch 1, as ONE grouped launch through the C ABI of libentro.
value = tokens/s = 1 / step time.  The coded model (1.4 GB) is far larger than
L2, so every step streams its weights from HBM; no flush is needed.  Times come
from CUDA events on the launching stream: K steps back to back between one pair
of events (events between launches would add gaps of their own).

Extra keys, each one grouped launch or a set of launches timed the same way:
  * mistral batch 4 and 16 (the same model, the GEMV's batched path);
  * smollm_bf16: the SmolLM-1.7B-shaped whole-model decode to bf16 (8-bit codes);
  * laplace_4096x4096_u4: the 4096x4096 4-bit tensor decoded to codes, to bf16
    and through the GEMV, 40 rotating replicas so that inputs exceed L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

With N > 1 (torchrun) every rank runs the step on its own GPU (tensors are
independent problems; no data-path collective) and the line reports the
whole-job rate from the slowest rank ("weak" scaling).  --impl reference times
the CPU oracle doing the same step on a bounded sample and extrapolates.

--profile runs only W warm-up and K timed launches of the chosen workload (no
burn-in, end-to-end leg, extras or CPU leg), so that a profiler attached to it
sees few launches; its line carries the launch time but no clocks.
"""
from __future__ import annotations

import argparse
import dataclasses
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
WORKLOAD = "mistral_7b_u4"
TENSOR_WORKLOAD = "laplace_4096x4096_u4"
REPLICAS = 40
NOMINAL_HBM_GBS = 7700.0  # B200 HBM3e, HGX figure (context beside the measured copy peak)
KERNEL_SOURCES = ("huffman_decode_canonical_b200/csrc/decode.cu", "huffman_decode_canonical_b200/csrc/rows.cuh",
                  "huffman_decode_canonical_b200/csrc/wide_decoder.cuh",
                  "huffman_decode_canonical_b200/csrc/blob_format.h")


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



# ------------------------------------------------------------------ model-shaped workloads

def encode_model(entro, W: workloads.Workload, device, limit=None, keep=0):
    """Draw, encode (libentro's host encoder, all host cores) and upload every tensor of
    W, one at a time.  Returns (device tensors, blob infos, seconds encoding, the
    serialized blobs of the first `keep` tensors)."""
    dts, infos, kept = [], [], []
    t_enc = 0.0
    specs = W.tensors if limit is None else W.tensors[:limit]
    for i, spec in enumerate(specs):
        w = workloads.weights(W, spec, device=device).cpu().numpy()
        t0 = time.perf_counter()
        blob = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=W.fmt,
                                 chunk_symbols=W.chunk_symbols(spec.cols), lanes=W.lanes)
        t_enc += time.perf_counter() - t0
        del w
        dts.append(entro.upload(blob, device=device))
        infos.append(blob.info())
        if i < keep:
            kept.append(blob.to_bytes())
        del blob
    return dts, infos, t_enc, kept


def _override(W, args):
    if not (getattr(args, "fmt", "") or getattr(args, "lanes", 0) or getattr(args, "chunk", 0)):
        return W
    fmt = {"lanes": workloads.FORMAT_LANES, "rows": workloads.FORMAT_ROWS, "rows_co": workloads.FORMAT_ROWS_CO,
           "": W.fmt}[args.fmt]
    lanes = args.lanes or W.lanes
    tiles = (workloads.FORMAT_ROWS, workloads.FORMAT_ROWS_CO)
    if fmt == workloads.FORMAT_LANES:
        rule = W.chunk_rule
    elif args.chunk:
        rule = "fixed:%d" % args.chunk
    else:  # row tiles: the workload's own tile size when it has one, else 256 columns
        rule = W.chunk_rule if W.fmt in tiles and lanes == W.lanes else "fixed:%d" % (256 * lanes)
    return dataclasses.replace(W, fmt=fmt, lanes=lanes, chunk_rule=rule)


class GemvStep:
    """The grouped fused GEMV over a model's tensors at one batch size.  Tensors with the
    same number of columns read the same activations (as the projections of one layer
    input do); every output row lands in one fp32 buffer, so a step's result comes back
    with one copy."""

    def __init__(self, entro, dts, seed, batch, device):
        self.batch = batch
        cols = sorted(set(d.cols for d in dts))
        self.x = {K: workloads.activations(seed, batch, K).to(device) for K in cols}
        self.rows = sum(d.rows for d in dts)
        self.y = torch.empty((batch * self.rows,), dtype=torch.float32, device=device)
        ys, off = [], 0
        for d in dts:
            ys.append(self.y[off: off + batch * d.rows].view(batch, d.rows))
            off += batch * d.rows
        self.ys = ys
        self.group = entro.Group(dts, entro.GROUP_GEMV, xs=[self.x[d.cols] for d in dts], ys=ys, batch=batch)
        self.x_bytes = sum(2 * x.numel() for x in self.x.values())        # distinct activation vectors
        self.io_bytes = sum(2 * batch * d.cols for d in dts) + 4 * batch * self.rows

    def launch(self, status):
        self.group.launch(status=status)


def _time_launches(fn, steps, stream, sleep_s=0.0):
    """Mean ms of `steps` calls of fn() back to back between one pair of events; the GPU
    is kept busy by a device sleep while the host enqueues them."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if sleep_s > 0:
        torch.cuda._sleep(int(sleep_s * 2.0e9))
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _step_bytes(infos, step):
    """Algorithmic bytes of one GEMV step: coded bits of every
    tensor (lane padding excluded) / 8 + chunk index + one copy of each tensor's decode
    tables + activations + outputs.  The bf16 weights are never written."""
    table = 32768 + 512
    return (sum(i["coded_bits"] for i in infos) / 8.0 + sum(i["index_bytes"] for i in infos)
            + table * len(infos) + step.io_bytes)


# ------------------------------------------------------------------ CPU oracle legs

def _oracle_sample(W, rows: int):
    """The first `rows` rows of layer 0's seven tensors, encoded by the oracle itself in the
    workload's format (the sample's own quantization parameters)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    specs = W.tensors[:7]

    def enc(spec):
        w = workloads.weights(W, spec, device="cpu").numpy()[:rows]
        blob = oracle.encode(w, W.bits, W.quant_mode, W.max_len, W.fmt, W.chunk_symbols(spec.cols), lanes=W.lanes)
        return blob, spec.cols
    with ThreadPoolExecutor(len(specs)) as ex:
        return list(ex.map(enc, specs))


def _oracle_pass(sample, threads: int, seed: int):
    """One pass of the oracle over the sample: decode every chunk bit by bit, dequantize to
    bf16, fp64 GEMV of the chunk's weights with the matching activations; chunks spread
    over threads (the EntroLLM multi-threaded chunk decoder).  Returns symbols processed."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    jobs = []
    for blob, cols in sample:
        p = oracle.params(blob)
        x = workloads.bf16_bits(workloads.activations(seed, 1, cols))
        for c in range(p["n_chunks"]):
            jobs.append((blob, p, x, c))

    def work(job):
        blob, p, x, c = job
        q = oracle.decode_chunks(blob, c, c + 1)
        wb = oracle.dequant_bf16(q, p["scale"], p["zero"])
        if p["format"] in (oracle.FMT_ROWS, oracle.FMT_ROWS_CO):
            r0, k0, nr, wd = oracle.tile(p, c)
            oracle.gemv(wb.reshape(nr, wd), np.ascontiguousarray(x[:, k0:k0 + wd]))
        else:
            oracle.gemv(wb.reshape(-1, p["cols"]), x)
        return q.size
    with ThreadPoolExecutor(threads) as ex:
        return sum(ex.map(work, jobs))


def _oracle_threads():
    return max(1, min(os.cpu_count() or 1, 64))


def cpu_baseline(W, seconds: float = 10.0, rows: int = 256):
    """The oracle doing the step's work on a bounded sample, extrapolated to the whole step."""
    t0 = time.perf_counter()
    sample = _oracle_sample(W, rows)
    t_enc = time.perf_counter() - t0
    threads = _oracle_threads()
    syms, passes, t0 = 0, 0, time.perf_counter()
    while True:
        syms += _oracle_pass(sample, threads, W.seed)
        passes += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    rate = syms / dt
    return {"value": round(rate / W.n, 6), "unit": "tok/s (batch 1)", "cores": threads, "kind": "oracle",
            "sample": f"{passes} pass(es) over the first {rows} rows of layer 0's 7 tensors "
                      f"({syms // passes} weights: bit-by-bit decode, bf16 dequant, fp64 GEMV per chunk), "
                      f"chunks over {threads} threads, {dt:.1f} s; tok/s = weights/s / {W.n} weights per step",
            "gsym_s": round(rate / 1e9, 4), "oracle_encode_s": round(t_enc, 2)}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    W = workloads.get(WORKLOAD)
    sample = _oracle_sample(W, 256)
    threads = _oracle_threads()
    for _ in range(args.warmup):
        _oracle_pass(sample, threads, W.seed)
    t0 = time.perf_counter()
    syms = 0
    for _ in range(args.steps):
        syms += _oracle_pass(sample, threads, W.seed)
    dt = time.perf_counter() - t0
    value = syms / dt / W.n
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s (batch 1)", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u4->bf16/fp64",
            "data": "synthetic", "config": _step_config(W, 1),
            "cpu_baseline": {"value": value, "unit": "tok/s (batch 1)", "cores": threads, "kind": "oracle",
                             "sample": f"per step: the first 256 rows of layer 0's 7 tensors "
                                       f"({syms // max(args.steps, 1)} weights), chunks over {threads} threads; "
                                       f"tok/s extrapolated to the step's {W.n} weights"},
            "e2e": {"value": value, "unit": "tok/s (batch 1)", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _step_config(W, batch):
    return {"workload": W.name, "tensors": len(W.tensors), "symbols": W.n, "bits": W.bits, "batch": batch,
            "format": {workloads.FORMAT_LANES: "lanes", workloads.FORMAT_ROWS: "row tiles",
                       workloads.FORMAT_ROWS_CO: "row tiles, consumption order"}.get(W.fmt, "single"),
            "lanes": W.lanes, "chunk_symbols": W.chunk_symbols(4096),
            "l2": "inputs larger than L2: the step streams 1.4 GB of coded weights (L2 126 MB); no flush"}


def _kernel_source_hash() -> str:
    """Hash of the kernel sources with comments and whitespace removed (a comment edit
    does not change the kernels whose traffic profiles/traffic.json records)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
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



# ------------------------------------------------------------------ native arm: the GEMV step

def _e2e_step(step, status, steps):
    """The step through the public API with host buffers: the activations are copied from
    pinned host memory, the grouped launch runs, and every output row is read back to
    pinned host memory before the next step starts (a token's result is needed before the
    next token's input exists).  Wall clock per step."""
    host_x = {K: x.cpu().pin_memory() for K, x in step.x.items()}
    host_y = torch.empty(step.y.shape, dtype=torch.float32, pin_memory=True)
    cur = torch.cuda.current_stream()

    def one():
        for K, hx in host_x.items():
            step.x[K].copy_(hx, non_blocking=True)
        step.launch(status)
        host_y.copy_(step.y, non_blocking=True)
        cur.synchronize()

    for _ in range(2):
        one()
    reps = max(3, min(steps, 50))
    t0 = time.perf_counter()
    for _ in range(reps):
        one()
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(1.0 / dt, 2), "unit": f"tok/s (batch {step.batch})",
            "h2d_bytes_per_step": int(sum(h.numel() * 2 for h in host_x.values())),
            "d2h_bytes_per_step": int(host_y.numel() * 4), "ms_per_step": round(1e3 * dt, 4),
            "note": "per step: activations copied from pinned host memory, one grouped launch "
                    "(entro_group_launch), all outputs copied back to pinned host memory, stream synchronised; "
                    "wall clock"}


def _smollm_bf16(entro, device, stream, steps, peak):
    """SmolLM-1.7B-shaped whole-model decode to bf16 (169 tensors, 8-bit codes), one grouped launch."""
    W = workloads.get("smollm_1p7b_u8")
    dts, infos, t_enc, _ = encode_model(entro, W, device)
    outs = [torch.empty((d.rows, d.cols), dtype=torch.bfloat16, device=device) for d in dts]
    g = entro.Group(dts, entro.GROUP_BF16, outs=outs)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    for _ in range(3):
        g.launch(status=status)
    ms = _time_launches(lambda: g.launch(status=status), max(5, min(steps, 20)), stream, 2e-4)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    n = sum(i["n"] for i in infos)
    alg = sum(i["coded_bits"] for i in infos) / 8.0 + sum(i["index_bytes"] for i in infos) + 2.0 * n
    gbs = alg / (ms * 1e-3) / 1e9
    out = {"ms": round(ms, 4), "gsym_s": round(n / (ms * 1e-3) / 1e9, 1), "alg_bytes": int(alg),
           "achieved_gbs": round(gbs, 1), "hbm_frac": round(gbs / peak, 4), "tensors": len(dts), "symbols": n,
           "bits_per_weight": round(sum(i["coded_bits"] for i in infos) / n, 4), "host_encode_s": round(t_enc, 2)}
    del outs, g, dts
    torch.cuda.empty_cache()
    return out


def _tensor_kernels(entro, device, stream, steps, peak, clk_mhz, sms, min_steps=20):
    """The 4096x4096 4-bit tensor (32 interleaved lanes per 8192-symbol chunk): decode to
    codes, to bf16 and the batch-1 GEMV, each K launches back to back over 40 rotating
    replicas (160 MB of coded words, inputs larger than L2)."""
    W = workloads.get(TENSOR_WORKLOAD)
    spec = W.tensors[0]
    w = workloads.weights(W, spec).numpy()
    blob = entro.Blob.encode(w, bits=W.bits, quant_mode=W.quant_mode, max_len=W.max_len, fmt=W.fmt,
                             chunk_symbols=W.chunk_symbols(spec.cols))
    info = blob.info()
    reps = [entro.upload(blob, device=device) for _ in range(REPLICAS)]
    n = info["n"]
    codes = [r.empty_codes() for r in reps]
    bf = [r.empty_bf16() for r in reps]
    x = workloads.activations(0, 1, spec.cols).to(device)
    y = [torch.empty((1, spec.rows), dtype=torch.float32, device=device) for _ in reps]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    counter = [0]

    def nxt():
        counter[0] += 1
        return counter[0] % REPLICAS

    kernels = [("codes", lambda: (lambda r: reps[r].decode_codes(out=codes[r], status=status))(nxt())),
               ("bf16", lambda: (lambda r: reps[r].decode_dequant_bf16(out=bf[r], status=status))(nxt())),
               ("gemv", lambda: (lambda r: reps[r].decode_gemv(x, y=y[r], status=status))(nxt()))]
    for _ in range(3):
        for _, fn in kernels:
            fn()
    coded = info["coded_bits"] / 8.0
    index = info["index_bytes"]
    alg = {"codes": coded + index + reps[0].codes_nbytes(), "bf16": coded + index + 2.0 * n,
           "gemv": coded + index + 2.0 * spec.cols + 4.0 * spec.rows}
    out = {}
    for name, fn in kernels:
        ms = _time_launches(fn, max(steps, min_steps), stream, 1e-4 if min_steps else 0.0)
        gbs = alg[name] / (ms * 1e-3) / 1e9
        out[name] = {"us": round(1e3 * ms, 3), "gsym_s": round(n / (ms * 1e-3) / 1e9, 2), "alg_bytes": int(alg[name]),
                     "achieved_gbs": round(gbs, 1), "hbm_frac": round(gbs / peak, 4),
                     "issue_bound": _issue_ceiling("tensor_" + name, n, ms, clk_mhz, sms)}
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    out["bits_per_weight"] = {"coded": round(info["coded_bits"] / n, 4),
                              "payload": round(8.0 * info["payload_bytes"] / n, 4)}
    out["note"] = ("one 4096x4096 tensor, 32 interleaved lanes per 8192-symbol chunk; each kernel K launches back "
                   "to back between one pair of CUDA events over 40 rotating replicas; the gemv figure is one "
                   "matrix, not a token")
    del reps, codes, bf, y
    torch.cuda.empty_cache()
    return out


def run_step(args, dist, rank, world, local_rank):
    import huffman_decode_canonical_b200 as entro
    entro.set_overlap(not args.no_overlap)
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    W = _override(workloads.get(WORKLOAD), args)
    t_setup = time.perf_counter()
    dts, infos, t_enc, _ = encode_model(entro, W, device)
    t_setup = time.perf_counter() - t_setup
    status = torch.zeros(1, dtype=torch.int32, device=device)
    step = GemvStep(entro, dts, W.seed, 1, device)
    for _ in range(max(3, args.warmup)):
        step.launch(status)
    torch.cuda.synchronize(device)
    if args.profile:
        return _profile_line(W, infos, lambda: step.launch(status), args, stream, status, dist, rank)
    clocks = ClockSampler(device)
    clocks.start()
    t_end = time.perf_counter() + 1.0  # burn-in, so that clock samples cover a loaded GPU
    while time.perf_counter() < t_end:
        step.launch(status)
        torch.cuda.synchronize(device)
    _barrier(dist, device)
    wall0 = time.perf_counter()
    ms = _time_launches(lambda: step.launch(status), args.steps, stream, 2e-4)
    wall = time.perf_counter() - wall0
    _barrier(dist, device)
    clk = clocks.stop()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    ms_max = _max_over_ranks(dist, ms, device)
    peak, peak_kind = _peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    n = sum(i["n"] for i in infos)
    alg = _step_bytes(infos, step)
    achieved = alg / (ms_max * 1e-3) / 1e9
    rec = _profile_record("kernels", "mistral_step")
    roofline = {"bound": "hbm", "kernel": "rows_kernel<4, gemv> (one grouped launch = the whole step)",
                "achieved": round(achieved, 1), "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs",
                "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": rec,
                "alg_bytes": int(alg), "peak_nominal": NOMINAL_HBM_GBS,
                "frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                "issue_bound": _issue_ceiling("mistral_step", n, ms_max, clk.get("sm_mhz"), sms)}
    e2e = _e2e_step(step, status, args.steps)
    e2e["value"] = -_max_over_ranks(dist, -e2e["value"], device) if dist is not None else e2e["value"]
    extras = {}
    if not args.no_extras:
        for b in (4, 16):
            sb = GemvStep(entro, dts, W.seed, b, device)
            for _ in range(3):
                sb.launch(status)
            mb = _time_launches(lambda: sb.launch(status), max(5, args.steps), stream, 2e-4)
            assert int(status.item()) == 0, f"device status {int(status.item())}"
            extras[f"mistral_batch{b}"] = {"ms": round(mb, 4), "tok_s": round(b / (mb * 1e-3), 1),
                                          "steps_s": round(1.0 / (mb * 1e-3), 1)}
            del sb
        del step, dts
        torch.cuda.empty_cache()
        extras["smollm_bf16"] = _smollm_bf16(entro, device, stream, args.steps, peak)
        extras[TENSOR_WORKLOAD] = _tensor_kernels(entro, device, stream, args.steps, peak, clk.get("sm_mhz"), sms)
    if rank != 0:
        return 0
    cpu = None if args.no_cpu_baseline or world > 1 else cpu_baseline(W)
    value = world / (ms_max * 1e-3)
    line = {"metric": METRIC, "value": round(value, 2), "unit": "tok/s (batch 1)", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u4 codes -> bf16 x bf16 -> fp32 accumulate",
            "data": "synthetic", "config": _step_config(W, 1), "launch_overlap": not args.no_overlap,
            "value_definition": "tokens/s = n_gpus / step time; a step = the fused decode -> dequantize -> GEMV "
                                "of all 224 tensors at batch 1 (one grouped launch); K steps back to back between "
                                "one pair of CUDA events",
            "gsym_s": round(n / (ms_max * 1e-3) / 1e9, 1),
            "bits_per_weight": {"coded": round(sum(i["coded_bits"] for i in infos) / n, 4),
                                "payload": round(8.0 * sum(i["payload_bytes"] for i in infos) / n, 4)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
            "clocks": clk, "host_encode_s": round(t_enc, 2), "setup_s": round(t_setup, 2),
            "wall_s_timed": round(wall, 4), "extras": extras}
    print(json.dumps(line), flush=True)
    return 0


def _profile_line(W, infos, launch, args, stream, status, dist, rank):
    """--profile: K launches after the warm-up, one short line, nothing else launched."""
    device = status.device
    ms = _time_launches(launch, args.steps, stream)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    ms = _max_over_ranks(dist, ms, device)
    if rank == 0:
        print(json.dumps({"profile": W.name, "tensors": len(infos), "symbols": sum(i["n"] for i in infos),
                          "warmup": args.warmup, "steps": args.steps, "ms_per_launch": round(ms, 5),
                          "note": "profiling run: no burn-in or clock samples; not a bench value"}), flush=True)
    return 0


# ------------------------------------------------------------------ other workloads (not the default line)

def run_model(args, dist, rank, world, local_rank):
    """One step = one grouped launch over every tensor of a model-shaped workload: the
    fused GEMV of a whole decode step (tok/s) or a whole-model decode to bf16."""
    import huffman_decode_canonical_b200 as entro
    entro.set_overlap(not args.no_overlap)
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    W = _override(workloads.get(args.workload), args)
    dts, infos, t_enc, _ = encode_model(entro, W, device, limit=args.tensors or None)
    n = sum(i["n"] for i in infos)
    coded = sum(i["coded_bits"] for i in infos) / 8.0
    payload = sum(i["payload_bytes"] for i in infos)
    index = sum(i["index_bytes"] for i in infos)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    gemv = args.workload != "smollm_1p7b_u8"
    if gemv:
        step = GemvStep(entro, dts, W.seed, args.batch, device)
        launch = lambda: step.launch(status)  # noqa: E731
        out_bytes = step.io_bytes
    else:
        outs = [torch.empty((d.rows, d.cols), dtype=torch.bfloat16, device=device) for d in dts]
        g = entro.Group(dts, entro.GROUP_BF16, outs=outs)
        launch = lambda: g.launch(status=status)  # noqa: E731
        out_bytes = 2 * n
    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize(device)
    if args.profile:
        return _profile_line(W, infos, launch, args, stream, status, dist, rank)
    clocks = ClockSampler(device)
    clocks.start()
    t_end = time.perf_counter() + 1.0
    while time.perf_counter() < t_end:
        launch()
        torch.cuda.synchronize(device)
    _barrier(dist, device)
    ms = _time_launches(launch, args.steps, stream, 2e-4)
    clk = clocks.stop()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    ms = _max_over_ranks(dist, ms, device)
    if rank != 0:
        return 0
    peak, peak_kind = _peaks()
    alg = coded + index + out_bytes
    achieved = alg / (ms * 1e-3) / 1e9
    partial = " (first %d tensors)" % len(dts) if args.tensors else ""
    line = {"metric": METRIC,
            "value": round(world * args.batch / (ms * 1e-3), 2) if gemv else round(world * n / (ms * 1e-3) / 1e9, 2),
            "unit": (f"tok/s (batch {args.batch})" if gemv else "Gsym/s") + partial, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": f"u{W.bits} codes -> bf16" + (" x bf16 -> fp32" if gemv else ""),
            "data": "synthetic", "launch_overlap": not args.no_overlap,
            "config": {"workload": W.name, "tensors": len(dts), "symbols": n, "bits": W.bits,
                       "batch": args.batch if gemv else None, "format": W.fmt, "lanes": W.lanes,
                       "l2": "working set larger than L2 (whole model)"},
            "gsym_s": round(n / (ms * 1e-3) / 1e9, 1),
            "bits_per_weight": {"coded": round(8 * coded / n, 4), "payload": round(8 * payload / n, 4)},
            "roofline": {"bound": "hbm", "kernel": "grouped launch", "achieved": round(achieved, 1),
                         "peak": peak, "peak_kind": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": None},
            "host_encode_s": round(t_enc, 2), "gpu_launches": args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def run_tensor(args, dist, rank, world, local_rank):
    """The 4096x4096 4-bit tensor's three kernels alone (the round-robin lanes format)."""
    import huffman_decode_canonical_b200 as entro
    entro.set_overlap(not args.no_overlap)
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peak, _ = _peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    clocks = ClockSampler(device)
    clocks.start()
    out = _tensor_kernels(entro, device, stream, args.steps, peak, None, sms, 0 if args.profile else 20)
    clk = clocks.stop()
    if rank == 0:
        print(json.dumps({"workload": TENSOR_WORKLOAD, "kernels": out, "clocks": clk}), flush=True)
    return 0




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



def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="default line without its extra workloads")
    ap.add_argument("--profile", action="store_true",
                    help="warm-up and timed launches only (no burn-in, e2e, extras or CPU leg): for ncu")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch without overlap (programmatic dependent launch, on by default)")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, TENSOR_WORKLOAD, "t4_1024x1024_u8", "smollm_1p7b_u8", "phi3_mini_u8"],
                    help="other workloads (not the default line): the 4096x4096 tensor's kernels, the "
                         "1024x1024 single-stream tensor, or model-scale workloads timed as one grouped launch per "
                         "step")
    ap.add_argument("--batch", type=int, default=1, help="GEMV batch for the model-scale GEMV workloads")
    ap.add_argument("--tensors", type=int, default=0, help="model-scale workloads: only the first N tensors")
    ap.add_argument("--fmt", choices=["lanes", "rows", "rows_co"], default="",
                    help="model-scale workloads: chunk format (rows_co: row tiles in consumption order)")
    ap.add_argument("--lanes", type=int, default=0, help="model-scale workloads: lanes (rows per tile) per chunk")
    ap.add_argument("--chunk", type=int, default=0, help="model-scale workloads, row tiles: symbols per chunk")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    dist, rank, world, local_rank = _dist()
    try:
        if args.impl == "reference":
            return run_reference(args, rank, world)
        if args.workload == "t4_1024x1024_u8":
            return run_single_stream(args, dist, rank, world, local_rank)
        if args.workload == TENSOR_WORKLOAD:
            return run_tensor(args, dist, rank, world, local_rank)
        if args.workload == WORKLOAD and not args.tensors and args.batch == 1:
            return run_step(args, dist, rank, world, local_rank)
        return run_model(args, dist, rank, world, local_rank)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
