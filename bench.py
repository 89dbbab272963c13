#!/usr/bin/env python
"""SplitZip lossless BF16 KV codec on B200 -- benchmark.

One step = the whole hot path over one batch: exponent histogram + top-16
codebook of every tensor, container write of every tensor, then decode of
every container back to BF16.  The workload is the Llama-3-8B-shaped KV
cache at 32K tokens (32 layers x {K,V} x 8 heads x 32768 tokens x 128 dim,
4 GiB, one codebook per (layer, K/V) tensor), synthetic and seeded (kvgen).

Rank 0 prints one JSON line.  `value` is round-trip throughput: uncompressed
bytes that went through encode and decode, over all ranks, per second of the
max-over-ranks device time.  Encode and decode are also reported alone.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl splitzip|reference]

--impl reference times the CPU oracle (test infrastructure, plain C, one
thread) on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kvgen  # noqa: E402

METRIC = "encode / decode GB/s (uncompressed) and % of HBM roofline; compression ratio"
WORKLOAD = 2          # the headline workload (and the sweep's and transfer's)
L2_BYTES = 126 * 10**6
WORKLOAD_NAMES = {0: "tiny-k-1m", 1: "llama3-8b-kv-4k", 2: "llama3-8b-kv-32k",
                  3: "llama3-70b-kv-8k-heavy-tail", 4: "paged-kv-256-requests"}
HEADER = 48
FALLBACK_HBM_GBS = 6650.0
# B200 HBM3e data-sheet bandwidth (8 TB/s; 7.7 TB/s on HGX boards).  Fractions
# of it are reported beside the fractions of the measured copy bandwidth.
SPEC_HBM_GBS = 8000.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="splitzip", choices=["splitzip", "reference"])
    p.add_argument("--workload", type=int, default=WORKLOAD, choices=sorted(WORKLOAD_NAMES),
                   help="0 tiny K tensor, 1 Llama-3-8B 4K, 2 Llama-3-8B 32K (default, the headline), "
                        "3 Llama-3-70B 8K heavy tails, 4 paged batch of 256 requests")
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-one-pass", action="store_true", help="skip the read-once and codebook-reuse encodes")
    p.add_argument("--no-workloads", action="store_true", help="skip the compact lines of the other workloads")
    p.add_argument("--tensors", type=int, default=0,
                   help="time only the first T (layer, K/V) tensors (a smaller case for profiling)")
    p.add_argument("--sweep", action="store_true",
                   help="latency sweep instead: single streams of 64 KiB .. 4 GiB (prefixes of the "
                        "workload's buffer), one JSON line per size")
    p.add_argument("--sweep-max", type=int, default=1 << 32, help="largest sweep size in bytes")
    p.add_argument("--sweep-reps", type=int, default=20)
    p.add_argument("--transfer", action="store_true",
                   help="transfer instead: the workload's cache moved GPU -> pinned host -> GPU in chunks, "
                        "raw vs compressed (encode / decode overlapped with the copies); one JSON line")
    p.add_argument("--transfer-chunk", type=int, default=4, help="tensors per chunk")
    p.add_argument("--transfer-reps", type=int, default=3)
    return p.parse_args()


def workload_config(tensors=0, workload=WORKLOAD):
    """The contiguous workloads (0-3): S tensors of n elements."""
    if workload == 0:
        n = kvgen.HEADS * 1024 * kvgen.HEAD_DIM
        return {"workload": WORKLOAD_NAMES[0],
                "shape": "[%d heads][1024 tokens][%d dim] bf16, 0.1%% of values scaled by 2^+-(20..40)"
                         % (kvgen.HEADS, kvgen.HEAD_DIM),
                "tensors": 1, "elems_per_tensor": n, "bytes": 2 * n, "codebooks": "one",
                "seed": "0x%X" % (kvgen.SEED_BASE + 0),
                "l2": "input fits the 126 MB L2: a 512 MiB write flushes it before every step; "
                      "ms_per_step is the sum of the phases"}
    layers, tokens = kvgen.CONTIGUOUS[workload]
    n = kvgen.HEADS * tokens * kvgen.HEAD_DIM
    t = 2 * layers if tensors <= 0 else min(tensors, 2 * layers)
    name = WORKLOAD_NAMES[workload]
    return {
        "workload": name if t == 2 * layers else "%s, first %d tensors" % (name, t),
        "shape": "[%d layers][K,V][%d heads][%d tokens][%d dim] bf16" % (layers, kvgen.HEADS, tokens, kvgen.HEAD_DIM),
        "tensors": t,
        "elems_per_tensor": n,
        "bytes": 2 * t * n,
        "codebooks": "one per (layer, K/V) tensor",
        "seed": "0x%X" % (kvgen.SEED_BASE + workload),
        "l2": "inputs (%d MiB) exceed the 126 MB L2; no flush between steps" % (2 * t * n >> 20),
    }


def host_cache(cfg, workload, out):
    """Fill ``out`` ([S, n] uint16 view) with the workload's tensors."""
    S = cfg["tensors"]
    if workload == 0:
        out[0] = kvgen.tiny_k_tensor()
    elif S % 2 == 0:
        kvgen.contiguous_cache(workload, layers=S // 2, out=out)
    else:
        for k in range(S):
            out[k] = kvgen.contiguous_tensor(workload, k // 2, k % 2)


class Inputs:
    """One rank's batch on the device: the plan, the page (or tensor)
    pointers in and out, the uncompressed bytes, and the host units."""

    def __init__(self, args, dev, sz):
        import torch
        self.workload = w = args.workload
        self.contiguous = w != 4
        if self.contiguous:
            cfg = workload_config(args.tensors, w)
            S, n = cfg["tensors"], cfg["elems_per_tensor"]
            # generated on the host straight into pinned memory, then resident in HBM
            self.h_in = torch.empty((S, n), dtype=torch.int16, pin_memory=True)
            host_cache(cfg, w, self.h_in.numpy().view(np.uint16))
            self.d_in = self.h_in.to(dev, non_blocking=False)
            self.d_out = torch.empty_like(self.d_in)
            self.plan = sz.BatchPlan([n] * S, n, device=dev)
            self.in_ptrs = torch.tensor([self.d_in.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64,
                                        device=dev)
            self.out_ptrs = torch.tensor([self.d_out.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64,
                                         device=dev)
            self.n_units = S
        else:
            b = kvgen.paged_batch()
            P = kvgen.PAGE_ELEMS
            lens = [int(v) * kvgen.HEADS * kvgen.HEAD_DIM for v in b.lengths]
            self.plan = sz.BatchPlan(lens, P, device=dev)
            self.pool_in = torch.zeros((b.pool_pages, P), dtype=torch.int16, device=dev)
            for r in range(b.n_requests):
                idx = torch.from_numpy(b.page_table[r]).to(dev)
                self.pool_in[idx] = torch.from_numpy(b.pages[r].view(np.int16)).to(dev)
            src = np.concatenate(b.page_table)
            dst = np.random.default_rng(kvgen.SEED_BASE + 44).permutation(b.pool_pages)[: src.size]
            self.pool_out = torch.zeros_like(self.pool_in)
            self.src_idx = torch.from_numpy(src).to(dev)
            self.dst_idx = torch.from_numpy(dst).to(dev)
            self.in_ptrs = torch.from_numpy(src * (2 * P) + self.pool_in.data_ptr()).to(dev)
            self.out_ptrs = torch.from_numpy(dst * (2 * P) + self.pool_out.data_ptr()).to(dev)
            self.batch = b
            self.n_units = b.n_requests
            cfg = {"workload": WORKLOAD_NAMES[4],
                   "shape": "%d requests of %d..%d tokens (log-uniform, rounded up to 16), pages [%d heads][16 "
                            "tokens][%d dim] bf16 scattered in a %d-page pool; decoded into a second pool under "
                            "another page table" % (b.n_requests, int(b.lengths.min()), int(b.lengths.max()),
                                                     kvgen.HEADS, kvgen.HEAD_DIM, b.pool_pages),
                   "requests": b.n_requests, "pages": int(src.size), "bytes": 2 * sum(lens),
                   "codebooks": "one per request", "seed": "0x%X" % (kvgen.SEED_BASE + 4),
                   "l2": "inputs (%d MiB) exceed the 126 MB L2; no flush between steps" % ((2 * sum(lens)) >> 20)}
        self.cfg = cfg
        self.U = int(cfg["bytes"])
        self.flush_l2 = self.U < 2 * L2_BYTES

    def unit(self, k):
        """Unit k (tensor or request stream) as host uint16."""
        if self.contiguous:
            return self.h_in[k].numpy().view(np.uint16)
        return self.batch.request_stream(k)

    def round_trip_ok(self):
        import torch
        if self.contiguous:
            return bool(torch.equal(self.d_out, self.d_in))
        return bool(torch.equal(self.pool_out[self.dst_idx], self.pool_in[self.src_idx]))


PROFILE_FILES = {
    "encode_kernel": "encode_kernel_llama3-8b-kv-32k-8tensors.md",
    "decode": "decode_kernel_llama3-8b-kv-32k-8tensors.md",
    "histogram+select": "hist_kernel_llama3-8b-kv-32k-8tensors.md",
}


# the sources each profiled kernel is built from
PROFILE_SOURCES = {
    "encode_kernel": ("sz_encode.cu", "sz_internal.cuh"),
    "decode": ("sz_decode.cu", "sz_internal.cuh"),
    "histogram+select": ("sz_hist.cu", "sz_internal.cuh"),
}


def kernel_source_hash(files=None, tree=None):
    """sha256 (16 hex digits) of the named kernel sources, or of all of
    them; ``tree`` maps a file name to its bytes instead of reading it."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "lossless_bf16_kv_splitzip_b200", "csrc")
    names = sorted(files) if files else sorted(os.path.basename(p) for p in glob.glob(os.path.join(csrc, "*")))
    h = hashlib.sha256()
    for name in names:
        h.update(name.encode())
        if tree is not None:
            h.update(tree[name])
        else:
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(phase, tensors, total_tensors):
    """DRAM bytes per launch from the committed ncu summary of that kernel
    (dram__bytes_read.sum + dram__bytes_write.sum, scaled from the 8-tensor
    capture to the launch's tensor count); None when that kernel's sources
    changed since the counters were taken."""
    name = PROFILE_FILES.get(phase)
    if name is None:
        return None
    try:
        fields = {}
        with open(os.path.join(ROOT, "profiles", name)) as f:
            for line in f:
                if ":" in line and not line.startswith(("|", "#", " ")):
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("kernel_source_sha256", "").split(" ")[0] != kernel_source_hash(PROFILE_SOURCES[phase]):
            return None
        return int(int(fields["traffic_per_full_launch_bytes"]) * tensors / total_tensors)
    except Exception:
        return None


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [t.strip() for t in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- reference arm
def run_reference(args):
    """The CPU oracle on bounded samples: each step encodes and decodes one
    unit of the workload (a (layer, K/V) tensor, or a request), in order,
    single-threaded."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    w = args.workload
    if w == 4:
        b = kvgen.paged_batch()
        n_units = b.n_requests
        cfg = {"workload": WORKLOAD_NAMES[4], "requests": n_units,
               "bytes": int(2 * b.lengths.sum() * kvgen.HEADS * kvgen.HEAD_DIM)}
        unit_of = b.request_stream
        what = "one request's pages"
    else:
        cfg = workload_config(0, w)
        n_units = cfg["tensors"]

        def unit_of(i):
            return kvgen.tiny_k_tensor() if w == 0 else kvgen.contiguous_tensor(w, i // 2, i % 2)
        what = "one %d MiB tensor" % (cfg["elems_per_tensor"] * 2 >> 20)
    cache = {}

    def unit(i):
        if i not in cache:
            cache[i] = unit_of(i)
        return cache[i]

    times, nbytes = [], []
    for s in range(args.warmup + args.steps):
        x = unit(s % n_units)
        t0 = time.perf_counter()
        blob = oracle.encode(x)
        y = oracle.decode(blob, x.size)
        dt = time.perf_counter() - t0
        assert np.array_equal(y[:16], x[:16])
        if s >= args.warmup:
            times.append(dt)
            nbytes.append(2 * x.size)
        if len(cache) > 4:
            cache.pop(next(iter(cache)))
    per_step = float(np.mean(times))
    value = float(np.sum(nbytes)) / float(np.sum(times)) / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_step * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: oracle encode + decode of %s, units taken in order" % what},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(inputs, seconds):
    """The oracle as it stands (one thread) on the first units of the
    workload until about `seconds` of CPU work have run."""
    import oracle
    oracle.build()
    done, t_total, nbytes = 0, 0.0, 0
    while done < inputs.n_units and t_total < seconds:
        x = inputs.unit(done)
        t0 = time.perf_counter()
        blob = oracle.encode(x)
        oracle.decode(blob, x.size)
        t_total += time.perf_counter() - t0
        nbytes += 2 * x.size
        done += 1
    kind = "requests" if inputs.workload == 4 else "(layer, K/V) tensors" if inputs.workload else "tensor"
    return {"value": round(nbytes / t_total / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "oracle encode + decode of the first %d of %d %s (%.1f s)"
                      % (done, inputs.n_units, kind, t_total)}


# ------------------------------------------------------------ latency sweep
def run_sweep(args):
    """Encode (histogram + codebook + container: sz_compress, and the
    two-call sz_histogram_codebook + sz_encode) and decode latency of one
    stream through the single-stream C ABI, for power-of-two sizes from
    64 KiB to 4 GiB.  A stream of b bytes is the first b bytes of the
    workload's buffer ([layer][K,V][head][token][dim]), coded as one stream
    with one codebook.  Each size's calls are captured once in CUDA graphs;
    a rep replays them between two events after a write of 512 MiB that
    flushes L2.  Every size is checked by its round trip (the parity tests
    compare such prefixes with the oracle byte for byte)."""
    import torch

    import lossless_bf16_kv_splitzip_b200 as sz

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    layers, tokens = kvgen.CONTIGUOUS[WORKLOAD]
    nt = kvgen.HEADS * tokens * kvgen.HEAD_DIM
    sizes_b = [1 << k for k in range(16, 33) if (1 << k) <= args.sweep_max]
    n_max = max(sizes_b) // 2
    tensors = -(-n_max // nt)
    h_in = torch.empty((tensors, nt), dtype=torch.int16, pin_memory=True)
    host = h_in.numpy().view(np.uint16)
    if tensors % 2 == 0:
        kvgen.contiguous_cache(WORKLOAD, layers=tensors // 2, out=host)
    else:
        for k in range(tensors):
            host[k] = kvgen.contiguous_tensor(WORKLOAD, k // 2, k % 2)
    d_flat = h_in.to(dev).view(-1)
    cap, wsb = sz.sz_plan(n_max)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    dec = torch.empty(n_max, dtype=torch.int16, device=dev)
    cb = torch.empty(16, dtype=torch.uint8, device=dev)
    size = torch.zeros(1, dtype=torch.int64, device=dev)
    est = torch.zeros(1, dtype=torch.int32, device=dev)
    dst = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    peak, peak_kind = measured_peak()
    stream = torch.cuda.Stream(dev)
    # The frame every number below sits in: the same events around an empty
    # graph, and around a graph of one tiny kernel (a 4-element add), after
    # the same flush.
    tiny = torch.zeros(4, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        g_one = torch.cuda.CUDAGraph()
        tiny.add_(1)
        with torch.cuda.graph(g_one, stream=stream):
            tiny.add_(1)
        t0, t1 = [], []
        for _ in range(3 + args.sweep_reps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            flush.fill_(1)
            ev[0].record(stream); ev[1].record(stream)
            flush.fill_(2)
            ev[2].record(stream); g_one.replay(); ev[3].record(stream)
            stream.synchronize()
            t0.append(ev[0].elapsed_time(ev[1]) / 1e3)
            t1.append(ev[2].elapsed_time(ev[3]) / 1e3)
        del g_one
    print(json.dumps({"sweep_frame": "events after the flush, nothing between / one tiny kernel graph",
                      "empty_us": round(float(np.median(t0[3:])) * 1e6, 2),
                      "one_kernel_us": round(float(np.median(t1[3:])) * 1e6, 2), "reps": args.sweep_reps}),
          flush=True)
    for b in sizes_b:
        n = b // 2
        x = d_flat[:n]
        c_cap, w_need = sz.sz_plan(n)
        with torch.cuda.stream(stream):
            def enc():  # one call: histogram, codebook and container
                sz.sz_compress(x, n, out, c_cap, size, cb, est, ws, w_need, stream)

            def enc2():  # the two-call path
                sz.sz_histogram_codebook(x, n, cb, None, ws, w_need, stream)
                sz.sz_encode(x, n, cb, out, c_cap, size, est, ws, w_need, stream)

            def dcd():
                sz.sz_decode(out, c_cap, dec, n, dst, ws, w_need, stream)

            enc2(); enc(); dcd()
            g_enc, g_enc2, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_enc2, stream=stream):
                enc2()
            with torch.cuda.graph(g_enc, stream=stream):
                enc()
            with torch.cuda.graph(g_dec, stream=stream):
                dcd()
            te, te2, td = [], [], []
            for _ in range(3 + args.sweep_reps):
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
                flush.fill_(1)
                ev[4].record(stream); g_enc2.replay(); ev[5].record(stream)
                flush.fill_(3)
                ev[0].record(stream); g_enc.replay(); ev[1].record(stream)
                flush.fill_(2)
                ev[2].record(stream); g_dec.replay(); ev[3].record(stream)
                stream.synchronize()
                te.append(ev[0].elapsed_time(ev[1]) / 1e3)
                te2.append(ev[4].elapsed_time(ev[5]) / 1e3)
                td.append(ev[2].elapsed_time(ev[3]) / 1e3)
            te, te2, td = float(np.median(te[3:])), float(np.median(te2[3:])), float(np.median(td[3:]))
            assert int(est.item()) == 0 and int(dst.item()) == 0, (b, int(est.item()), int(dst.item()))
            comp = int(size.item())
            ok = bool(torch.equal(dec[:n], x))
            del g_enc, g_enc2, g_dec
        line = {"sweep": "single stream, first bytes of llama3-8b-kv-32k", "bytes": b, "elems": n,
                "encode_us": round(te * 1e6, 2), "encode_two_call_us": round(te2 * 1e6, 2),
                "decode_us": round(td * 1e6, 2),
                "encode_gbs": round(b / te / 1e9, 2), "decode_gbs": round(b / td / 1e9, 2),
                "encode_roofline_frac": round((b + comp) / te / 1e9 / peak, 4),
                "decode_roofline_frac": round((b + comp) / td / 1e9 / peak, 4),
                "encode_roofline_frac_of_spec": round((b + comp) / te / 1e9 / SPEC_HBM_GBS, 4),
                "decode_roofline_frac_of_spec": round((b + comp) / td / 1e9 / SPEC_HBM_GBS, 4),
                "ratio": round(b / comp, 5), "round_trip": ok,
                "peak_gbs": peak, "peak_kind": peak_kind, "reps": args.sweep_reps,
                "timing": "CUDA graph replay between events, median; L2 flushed (512 MiB write) before each"}
        print(json.dumps(line), flush=True)


def single_streams(d_flat, sz, dev, peak, reps=10):
    """Mid-size single streams in the headline line: the first 16 and 64 MiB
    of the workload's buffer as ONE stream each, sz_compress and sz_decode
    captured in CUDA graphs and replayed between two events after a 512 MiB
    write that flushes L2 (median of `reps`), as in the latency sweep; also
    the frame, the same events around a graph of one tiny kernel."""
    import torch
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    n_max = (64 << 20) // 2
    cap, wsb = sz.sz_plan(n_max)
    out = torch.empty(cap, dtype=torch.uint8, device=dev)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    dec = torch.empty(n_max, dtype=torch.int16, device=dev)
    cb = torch.empty(16, dtype=torch.uint8, device=dev)
    size = torch.zeros(1, dtype=torch.int64, device=dev)
    est = torch.zeros(1, dtype=torch.int32, device=dev)
    dst = torch.zeros(1, dtype=torch.int32, device=dev)
    tiny = torch.zeros(4, dtype=torch.int32, device=dev)

    def timed(graphs):
        t = [[] for _ in graphs]
        for r in range(3 + reps):
            for i, g in enumerate(graphs):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                flush.fill_(r & 255)
                e0.record(stream); g.replay(); e1.record(stream)
                stream.synchronize()
                if r >= 3:
                    t[i].append(e0.elapsed_time(e1) * 1e3)
        return [float(np.median(v)) for v in t]

    res = {}
    with torch.cuda.stream(stream):
        g1 = torch.cuda.CUDAGraph()
        tiny.add_(1)
        with torch.cuda.graph(g1, stream=stream):
            tiny.add_(1)
        res["frame_one_kernel_us"] = round(timed([g1])[0], 2)
        del g1
        for mib in (16, 64):
            b = mib << 20
            n = b // 2
            x = d_flat[:n]
            c_cap, w_need = sz.sz_plan(n)

            def enc():
                sz.sz_compress(x, n, out, c_cap, size, cb, est, ws, w_need, stream)

            def dcd():
                sz.sz_decode(out, c_cap, dec, n, dst, ws, w_need, stream)

            enc(); dcd()
            ge, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(ge, stream=stream):
                enc()
            with torch.cuda.graph(gd, stream=stream):
                dcd()
            te, td = timed([ge, gd])
            stream.synchronize()
            comp = int(size.item())
            ok = int(est.item()) == 0 and int(dst.item()) == 0 and bool(torch.equal(dec[:n], x))
            res["%dMiB" % mib] = {"compress_us": round(te, 2), "decode_us": round(td, 2),
                                  "compress_frac": round((b + comp) / (te * 1e-6) / 1e9 / peak, 4),
                                  "decode_frac": round((b + comp) / (td * 1e-6) / 1e9 / peak, 4),
                                  "ratio": round(b / comp, 5), "round_trip": ok}
            del ge, gd
    res["timing"] = ("CUDA graph replay between events after a 512 MiB L2 flush, median of %d; fractions of the "
                     "peak over 2N + container bytes" % reps)
    return res


# ---------------------------------------------------------------- transfer
def run_transfer(args):
    """The cache handed from one place to another over a link: here PCIe
    through pinned host memory (the only link one GPU has), device-to-host
    and host-to-device copies on their own streams, chunk by chunk.  Raw:
    the BF16 values cross.  Compressed: each chunk is encoded before it
    crosses and decoded after (kernels overlapped with the other chunks'
    copies).  Device time from the first operation to the last."""
    import torch

    from lossless_bf16_kv_splitzip_b200.transfer import SplitZipChunks, host_transfer

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = workload_config(args.tensors)
    S, n = cfg["tensors"], cfg["elems_per_tensor"]
    h_in = torch.empty((S, n), dtype=torch.int16, pin_memory=True)
    host = h_in.numpy().view(np.uint16)
    if S % 2 == 0:
        kvgen.contiguous_cache(WORKLOAD, layers=S // 2, out=host)
    else:
        for k in range(S):
            host[k] = kvgen.contiguous_tensor(WORKLOAD, k // 2, k % 2)
    src = h_in.to(dev)
    del h_in, host
    out = torch.empty_like(src)
    staging = torch.empty(2 * S * n + 4096 * S, dtype=torch.uint8, pin_memory=True)
    codec = SplitZipChunks(src, out, args.transfer_chunk, dev)
    res = {}
    for name, cd in (("raw", None), ("compressed", codec)):
        times = []
        for r in range(1 + args.transfer_reps):
            out.zero_()
            t = host_transfer(cd, src, out, args.transfer_chunk, staging)
            torch.cuda.synchronize(dev)
            if r:
                times.append(t.seconds)
            assert torch.equal(out, src), name
            link = t.link_bytes
        if cd is not None:
            assert codec.statuses_ok()
        res[name] = (float(np.median(times)), link)
    t_raw, b_raw = res["raw"]
    t_c, b_c = res["compressed"]
    line = {"transfer": "GPU -> pinned host -> GPU (PCIe), %d chunks of %d tensors" % (len(codec.chunks),
                                                                                     args.transfer_chunk),
            "config": cfg, "raw_ms": round(t_raw * 1e3, 3), "compressed_ms": round(t_c * 1e3, 3),
            "speedup": round(t_raw / t_c, 4), "ratio": round(b_raw / b_c, 5),
            "raw_link_gbs": round(b_raw / t_raw / 1e9, 2), "compressed_link_gbs": round(b_c / t_c / 1e9, 2),
            "effective_gbs": round(b_raw / t_c / 1e9, 2), "round_trip": True, "reps": args.transfer_reps,
            "timing": "CUDA events, first operation to last, median of reps after one warm-up"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def host_facts():
    """Cores and CPU model of the host the CPU baseline runs on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


def job_config(cfg, world):
    """The workload's config plus how the job is spread over `world` GPUs:
    every rank codes its own copy of the workload (units are independent;
    no collective touches the data path)."""
    out = dict(cfg)
    if world == 1:
        out["parallelism"] = "1 GPU"
    else:
        out["parallelism"] = ("replicas x%d: each rank codes its own copy of the workload; the only "
                              "collectives are the timing barrier and a max all-reduce" % world)
    return out


def accumulate_chunks(inp, sz, dev, chunk_tokens=4096, page_chunks=4):
    """The workload's cache as it is written during prefill, one plan per
    prefill chunk for sz_histogram_accumulate_batched.  Contiguous
    workloads: every chunk of `chunk_tokens` tokens adds, for every (layer,
    K/V) tensor and head, its token slice (a contiguous run) to the tensor's
    histogram.  Paged: every request's pages arrive in `page_chunks` runs.
    Returns [(plan, page pointers, histogram row of each segment)]."""
    import torch
    out = []
    if inp.contiguous:
        S, n = inp.d_in.shape
        T = n // (kvgen.HEADS * kvgen.HEAD_DIM)
        base = inp.d_in.data_ptr()
        for c0 in range(0, T, chunk_tokens):
            t = min(chunk_tokens, T - c0)
            ptrs = [base + 2 * (k * n + (h * T + c0) * kvgen.HEAD_DIM) for k in range(S) for h in range(kvgen.HEADS)]
            rows = [k for k in range(S) for _ in range(kvgen.HEADS)]
            p = sz.BatchPlan([t * kvgen.HEAD_DIM] * len(ptrs), t * kvgen.HEAD_DIM, device=dev, buffers=False)
            out.append((p, torch.tensor(ptrs, dtype=torch.int64, device=dev),
                        torch.tensor(rows, dtype=torch.int32, device=dev)))
    else:
        b, P = inp.batch, kvgen.PAGE_ELEMS
        base = inp.pool_in.data_ptr()
        for c in range(page_chunks):
            lens, ptrs, rows = [], [], []
            for r in range(b.n_requests):
                slots = np.array_split(b.page_table[r], page_chunks)[c]
                if slots.size:
                    lens.append(int(slots.size) * P)
                    ptrs.extend(int(base + 2 * P * s_) for s_ in slots)
                    rows.append(r)
            p = sz.BatchPlan(lens, P, device=dev, buffers=False)
            out.append((p, torch.tensor(ptrs, dtype=torch.int64, device=dev),
                        torch.tensor(rows, dtype=torch.int32, device=dev)))
    return out


def time_events(fn, k, stream):
    """Mean device time (s) of fn() over k calls, CUDA events on `stream`."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
    for a0, a1 in ev:
        a0.record(stream)
        fn()
        a1.record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a0.elapsed_time(a1) for a0, a1 in ev])) / 1e3


def read_once_phase(inp, plan, sz, dev, stream, steps, peak):
    """The read-once encode: histograms accumulated while the cache is
    written (timed per prefill chunk), then per step the select of the exact
    codebooks and the one-pass encode.  Its containers must be the two-pass
    path's bytes.  Returns (dict, the one-pass plan, codebooks)."""
    import torch
    chunks = accumulate_chunks(inp, sz, dev)
    hists = torch.zeros((plan.n_segs, 256), dtype=torch.int32, device=dev)

    def accumulate():
        hists.zero_()
        for p, ptrs, rows in chunks:
            p.accumulate(ptrs, hists, rows, stream)

    accumulate()
    torch.cuda.synchronize()
    acc_ok = all(int(p.acc_status.abs().sum()) == 0 for p, _, _ in chunks)
    # per chunk: device time of each chunk's call, averaged
    t_acc = []
    for _ in range(3):
        for p, ptrs, rows in chunks:
            t_acc.append(time_events(lambda: p.accumulate(ptrs, hists, rows, stream), 1, stream))
    accumulate()  # the histograms again (the timing loop added the cache three more times)
    plan1 = sz.BatchPlan(plan.seg_elems, plan.page_elems, device=dev)
    cbs = torch.empty((plan.n_segs, 16), dtype=torch.uint8, device=dev)

    def step():
        sz.sz_select_codebook_batched(plan.n_segs, hists, cbs, None, stream)
        plan1.encode_one_pass(inp.in_ptrs, cbs, stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    same = bool(torch.equal(plan1.sizes, plan.sizes)) and int(plan1.enc_status.abs().sum()) == 0 and acc_ok
    same = same and bool(torch.equal(cbs, plan.codebooks[: plan.n_segs]))
    sizes = plan.sizes.cpu().numpy()
    for k in range(plan.n_segs):
        o, z = int(plan.out_offset[k]), int(sizes[k])
        same = same and bool(torch.equal(plan1.container[o: o + z], plan.container[o: o + z]))
    t1 = time_events(step, steps, stream)
    U, comp = inp.U, int(sizes.sum())
    chunk_bytes = U / len(chunks)
    ta = float(np.mean(t_acc))
    res = {"ms": round(t1 * 1e3, 4), "encode_gbs": round(U / t1 / 1e9, 2),
           "roofline_frac": round((U + comp) / t1 / 1e9 / peak, 4),
           "roofline_frac_of_spec": round((U + comp) / t1 / 1e9 / SPEC_HBM_GBS, 4),
           "same_containers_as_two_pass": same, "steps": steps,
           "launches": "select (1 block per codebook), one-pass encode, escape placement, overflow rescan",
           "accumulate": {"chunks": len(chunks), "ms_per_chunk": round(ta * 1e3, 4),
                          "chunk_bytes": int(chunk_bytes), "gbs": round(chunk_bytes / ta / 1e9, 1),
                          "roofline_frac": round(chunk_bytes / ta / 1e9 / peak, 4),
                          "what": ("per prefill chunk of 4096 tokens: every (layer, K/V) tensor's 8 head slices "
                                   "added to its histogram, one launch" if inp.contiguous else
                                   "per prefill chunk: a quarter of every request's pages added to its "
                                   "request's histogram, one launch")}}
    return res, plan1, cbs


def reuse_phase(inp, plan, plan1, cbs, stream, steps, peak):
    """Codebook reuse across layers: layer L's K and V tensors encoded with
    layer L-1's K and V codebooks (layer 0 keeps its own), one pass.
    Escapes, ratio and time beside the tensors' own codebooks."""
    import torch
    S = plan.n_segs
    prev = cbs.clone()
    prev[2:] = cbs[: S - 2]
    plan1.encode_one_pass(inp.in_ptrs, prev, stream)
    torch.cuda.synchronize()
    ok = int(plan1.enc_status.abs().sum()) == 0
    t = time_events(lambda: plan1.encode_one_pass(inp.in_ptrs, prev, stream), steps, stream)
    seg_n = np.array(plan.seg_elems, dtype=np.int64)
    sizes = plan1.sizes.cpu().numpy().astype(np.int64)
    esc = int(((sizes - (HEADER + seg_n + (seg_n + 1) // 2)) // 5).sum())
    comp = int(sizes.sum())
    return {"codebooks": "layer L-1's (K for K, V for V); layer 0 its own", "status_ok": ok,
            "escape_frac": round(esc / (inp.U // 2), 6), "ratio": round(inp.U / comp, 5),
            "ms": round(t * 1e3, 4), "encode_gbs": round(inp.U / t / 1e9, 2),
            "roofline_frac": round((inp.U + comp) / t / 1e9 / peak, 4)}


def two_pass_steps(inp, plan, stream, steps, warmup, flush=None, clocks=None, barrier=None):
    """Warm-up, then `steps` timed steps of histogram + select, encode and
    decode.  Returns per-step phase times (s) and the clock record."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]

    def step(ev=None):
        if flush is not None:  # an input that fits L2 is flushed out of it before every step
            flush.fill_(1)
        if ev is not None:
            ev[0].record(stream)
        plan.histogram(inp.in_ptrs, stream)
        if ev is not None:
            ev[1].record(stream)
        plan.encode_only(inp.in_ptrs, stream)
        if ev is not None:
            ev[2].record(stream)
        plan.decode(inp.out_ptrs, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    if int(plan.enc_status.abs().sum()) or int(plan.dec_status.abs().sum()):
        raise RuntimeError("device status: encode %s decode %s" % (plan.enc_status.tolist(), plan.dec_status.tolist()))
    if barrier:
        barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.25)  # let the sampler take its first reading
    for k in range(steps):
        step(evs[k])
    torch.cuda.synchronize()
    clock_info = clocks.stop() if clocks else None
    if barrier:
        barrier()
    t_hist = np.array([e[0].elapsed_time(e[1]) for e in evs]) / 1e3
    t_enc = np.array([e[1].elapsed_time(e[2]) for e in evs]) / 1e3
    t_dec = np.array([e[2].elapsed_time(e[3]) for e in evs]) / 1e3
    total_s = evs[0][0].elapsed_time(evs[-1][3]) / 1e3
    return t_hist, t_enc, t_dec, total_s, clock_info


def phase_fracs(U, comp, th, te, td, peak):
    return {"histogram+select": round(U / th / 1e9 / peak, 4),
            "encode_kernel": round((U + comp) / te / 1e9 / peak, 4),
            "encode_end_to_end": round((U + comp) / (th + te) / 1e9 / peak, 4),
            "decode": round((U + comp) / td / 1e9 / peak, 4)}


def other_workload(w, dev, sz, stream, steps, peak):
    """A compact line for another workload: ratio, escapes, phase fractions
    of the measured peak, the read-once encode, and for the paged batch the
    adversarial pass's worst-case bound."""
    import types

    import torch
    inp = Inputs(types.SimpleNamespace(workload=w, tensors=0), dev, sz)
    plan = inp.plan
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if inp.flush_l2 else None
    th, te, td, _, _ = two_pass_steps(inp, plan, stream, steps, 3, flush)
    th, te, td = float(th.mean()), float(te.mean()), float(td.mean())
    seg_n = np.array(plan.seg_elems, dtype=np.int64)
    sizes = plan.sizes.cpu().numpy().astype(np.int64)
    comp = int(sizes.sum())
    esc = int(((sizes - (HEADER + seg_n + (seg_n + 1) // 2)) // 5).sum())
    U = inp.U
    res = {"config": inp.cfg["workload"], "bytes": U, "ratio": round(U / comp, 5),
           "escape_frac": round(esc / (U // 2), 6), "round_trip": inp.round_trip_ok(), "steps": steps,
           "ms": {"histogram+select": round(th * 1e3, 4), "encode_kernel": round(te * 1e3, 4),
                  "decode": round(td * 1e3, 4)},
           "frac": phase_fracs(U, comp, th, te, td, peak)}
    ro, plan1, cbs = read_once_phase(inp, plan, sz, dev, stream, steps, peak)
    res["encode_read_once"] = {k: ro[k] for k in ("ms", "roofline_frac", "same_containers_as_two_pass")}
    res["encode_read_once"]["accumulate_frac"] = ro["accumulate"]["roofline_frac"]
    if inp.contiguous and w == 3:
        res["codebook_reuse"] = reuse_phase(inp, plan, plan1, cbs, stream, steps, peak)
    del plan1
    if w == 4:  # adversarial pass: uniform random 16-bit patterns in the same pages
        b = kvgen.paged_batch(adversarial=True)
        for r in range(b.n_requests):
            inp.pool_in[torch.from_numpy(b.page_table[r]).to(dev)] = torch.from_numpy(b.pages[r].view(np.int16)).to(dev)
        plan.encode(inp.in_ptrs, stream)
        torch.cuda.synchronize()
        sz_adv = plan.sizes.cpu().numpy().astype(np.int64)
        bound = HEADER + seg_n + (seg_n + 1) // 2 + 5 * (seg_n - (seg_n + 15) // 16)
        res["adversarial"] = {"status_ok": int(plan.enc_status.abs().sum()) == 0,
                              "within_bound": bool((sz_adv <= bound).all()),
                              "max_size_over_bound": round(float((sz_adv / bound).max()), 6),
                              "ratio": round(U / int(sz_adv.sum()), 5)}
    del inp, plan, flush
    torch.cuda.empty_cache()
    return res


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.sweep:
        if int(os.environ.get("RANK", "0")) == 0:
            run_sweep(args)
        return
    if args.transfer:
        if int(os.environ.get("RANK", "0")) == 0:
            run_transfer(args)
        return

    import torch
    import torch.distributed as dist

    import lossless_bf16_kv_splitzip_b200 as sz

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    inp = Inputs(args, dev, sz)
    cfg, plan, in_ptrs = inp.cfg, inp.plan, inp.in_ptrs
    U = inp.U  # uncompressed bytes per step on this rank
    seg_n = np.array(plan.seg_elems, dtype=np.int64)
    S = plan.n_segs
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if inp.flush_l2 else None
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    clocks = ClockSampler(vis.split(",")[local] if vis else str(local))

    t_hist, t_enc, t_dec, total_s, clock_info = two_pass_steps(inp, plan, stream, args.steps, args.warmup, flush,
                                                               clocks, barrier)
    ms_step = total_s / args.steps * 1e3
    if flush is not None:  # the flushes between steps are not the codec's time
        ms_step = float(np.mean(t_hist + t_enc + t_dec)) * 1e3
    if world > 1:
        t = torch.tensor([ms_step, t_hist.mean(), t_enc.mean(), t_dec.mean()], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step, th, te, td = t.tolist()
    else:
        th, te, td = float(t_hist.mean()), float(t_enc.mean()), float(t_dec.mean())

    # ---- results of the last step: sizes, ratio, statuses, round trip
    sizes = plan.sizes.cpu().numpy().astype(np.int64)
    assert int(plan.enc_status.abs().sum()) == 0 and int(plan.dec_status.abs().sum()) == 0
    comp = int(sizes.sum())
    esc = int(((sizes - (HEADER + seg_n + (seg_n + 1) // 2)) // 5).sum())
    round_trip_ok = inp.round_trip_ok()

    # ---- self-checks of the last step (bit-exactness against the oracle is
    # the parity tests' job): every tensor round-trips, and every container's
    # header states its length and escape count consistently
    hdr_ok = True
    for k in sorted({0, S - 1}):
        off = int(plan.out_offset[k])
        h = plan.container[off: off + HEADER].cpu().numpy()
        hn = int(h[8:16].view(np.uint64)[0])
        he = int(h[16:24].view(np.uint64)[0])
        nk = int(seg_n[k])
        hdr_ok &= bytes(h[:4]) == b"SZKV" and hn == nk and HEADER + nk + (nk + 1) // 2 + 5 * he == int(sizes[k])
    parity = {"decode_round_trip_all_units": round_trip_ok, "header_size_consistent": bool(hdr_ok)}

    # ---- roofline (algorithmic bytes / event time, per phase)
    peak, peak_kind = measured_peak()
    phases = {
        "histogram+select": (U, th),
        "encode_kernel": (U + comp, te),
        "decode": (comp + U, td),
    }
    roof = {}
    for name, (b, t) in phases.items():
        a = b / t / 1e9
        roof[name] = {"achieved": round(a, 1), "frac": round(a / peak, 4),
                      "frac_of_spec": round(a / SPEC_HBM_GBS, 4), "ms": round(t * 1e3, 4),
                      "algorithmic_bytes": b}
    dom = max(phases, key=lambda k: phases[k][1])
    enc_e2e_bytes = U + comp
    encode_s = th + te
    # the committed ncu summaries cover the headline workload only
    traffic = profiled_traffic(dom, S, 2 * kvgen.CONTIGUOUS[WORKLOAD][0]) if inp.workload == WORKLOAD else None
    roofline = {"bound": "hbm", "kernel": dom, "achieved": roof[dom]["achieved"], "peak": peak, "unit": "GB/s",
                "frac": roof[dom]["frac"], "traffic": traffic,
                "spec_peak": SPEC_HBM_GBS, "frac_of_spec": roof[dom]["frac_of_spec"],
                "peak_kind": peak_kind + " (copy, MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"}

    # ---- the read-once encode (histograms kept while the cache is written,
    # exact codebooks, one pass) and the cost of reusing the previous
    # layer's codebooks instead
    read_once = reuse = None
    k1 = max(1, min(args.steps, 50))
    if not args.no_one_pass:
        read_once, plan1, cbs = read_once_phase(inp, plan, sz, dev, stream, k1, peak)
        if inp.contiguous and S > 2:
            reuse = reuse_phase(inp, plan, plan1, cbs, stream, k1, peak)
        del plan1, cbs

    # ---- end to end: pinned host buffers, copies inside the timed region.
    # The cache goes up, is encoded, its containers come down and go up
    # again, are decoded and the BF16 values come down -- chunks of 4
    # tensors, uploads and downloads on their own streams so that both
    # directions of the link stay busy while the kernels run in between.
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0 and inp.contiguous:
        from lossless_bf16_kv_splitzip_b200.transfer import SplitZipChunks, host_round_trip
        h_in, d_in, d_out = inp.h_in, inp.d_in, inp.d_out
        per_chunk = 4
        rt = SplitZipChunks(d_in, d_out, per_chunk, dev)
        h_out = torch.empty(tuple(h_in.shape), dtype=torch.int16, pin_memory=True)
        staging = torch.empty(comp + 4096 * S + (1 << 20), dtype=torch.uint8, pin_memory=True)
        times = []
        for it in range(args.e2e_steps + 1):
            if it == args.e2e_steps:
                h_out[:, :8].zero_()  # the last pass must write every tensor again
            barrier()
            torch.cuda.synchronize(dev)
            t_rt, n_up, n_down = host_round_trip(rt, h_in, h_out, staging)
            if it > 0:  # the first pass warms the copy engines
                times.append(t_rt)
        assert torch.equal(h_out, h_in) and rt.statuses_ok()
        e2e_s = float(np.mean(times))
        if world > 1:
            t = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_s = t.item()
        e2e = {"value": round(world * U / e2e_s / 1e9, 3), "unit": "GB/s",
               "h2d_bytes_per_step": int(n_up), "d2h_bytes_per_step": int(n_down),
               "ms_per_step": round(e2e_s * 1e3, 2),
               "path": "pinned host -> upload -> encode -> download containers -> upload containers -> decode "
                       "-> download BF16, through the C ABI; %d chunks of %d tensors, uploads and downloads on "
                       "their own streams" % (len(rt.chunks), per_chunk)}
        del rt, staging, h_out

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(inp, args.cpu_seconds)
        cpu.update(host_facts())

    # ---- mid-size single streams and the other workloads, fewer steps
    # each (rank 0, one GPU)
    workloads = None
    streams = None
    if rank == 0 and world == 1 and not args.no_workloads and args.tensors <= 0:
        if inp.contiguous:
            streams = single_streams(inp.d_in.view(-1), sz, dev, peak)
        del inp, plan, flush
        torch.cuda.empty_cache()
        workloads = {}
        for w in (1, 3, 4):
            if w != args.workload:
                workloads[WORKLOAD_NAMES[w]] = other_workload(w, dev, sz, stream, min(args.steps, 10), peak)

    if rank == 0:
        value = world * U / (ms_step / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u16", "data": "synthetic", "config": job_config(cfg, world),
            "encode_gbs": round(U / encode_s / 1e9, 2), "decode_gbs": round(U / td / 1e9, 2),
            "encode_roofline_frac": round(enc_e2e_bytes / encode_s / 1e9 / peak, 4),
            "decode_roofline_frac": roof["decode"]["frac"],
            "encode_roofline_frac_of_spec": round(enc_e2e_bytes / encode_s / 1e9 / SPEC_HBM_GBS, 4),
            "decode_roofline_frac_of_spec": roof["decode"]["frac_of_spec"],
            "encode_read_once": read_once, "codebook_reuse": reuse, "single_streams": streams,
            "ratio": round(U / comp, 5), "escape_frac": round(esc / (U // 2), 6),
            "roofline": roofline, "roofline_phases": roof,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 4 * args.steps,  # hist, encode, esc_index, decode
            "clocks": clock_info, "parity": parity, "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
