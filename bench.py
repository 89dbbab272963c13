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
WORKLOAD = 2
HEADER = 48
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="splitzip", choices=["splitzip", "reference"])
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-one-pass", action="store_true")
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


def workload_config(tensors=0):
    layers, tokens = kvgen.CONTIGUOUS[WORKLOAD]
    n = kvgen.HEADS * tokens * kvgen.HEAD_DIM
    t = 2 * layers if tensors <= 0 else min(tensors, 2 * layers)
    return {
        "workload": "llama3-8b-kv-32k" if t == 2 * layers else "llama3-8b-kv-32k, first %d tensors" % t,
        "shape": "[%d layers][K,V][%d heads][%d tokens][%d dim] bf16" % (layers, kvgen.HEADS, tokens, kvgen.HEAD_DIM),
        "tensors": t,
        "elems_per_tensor": n,
        "bytes": 2 * t * n,
        "codebooks": "one per (layer, K/V) tensor",
        "seed": "0x%X" % (kvgen.SEED_BASE + WORKLOAD),
        "l2": "inputs (%d MiB) exceed the 126 MB L2; no flush between steps" % (2 * t * n >> 20),
    }


PROFILE_FILES = {
    "encode_kernel": "encode_kernel_llama3-8b-kv-32k-8tensors.md",
    "decode": "decode_kernel_llama3-8b-kv-32k-8tensors.md",
    "histogram+select": "hist_kernel_llama3-8b-kv-32k-8tensors.md",
}


def kernel_source_hash():
    import glob
    import hashlib
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "lossless_bf16_kv_splitzip_b200", "csrc", "*"))):
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(phase, tensors, total_tensors):
    """DRAM bytes per launch from the committed ncu summary of that kernel
    (dram__bytes_read.sum + dram__bytes_write.sum, scaled from the 8-tensor
    capture to the launch's tensor count); None when the kernel sources
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
        if fields.get("kernel_source_sha256") != kernel_source_hash():
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
    (layer, K/V) tensor of the workload, single-threaded."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    cfg = workload_config()
    n = cfg["elems_per_tensor"]
    cache = {}

    def tensor(i):
        if i not in cache:
            cache[i] = kvgen.contiguous_tensor(WORKLOAD, i // 2, i % 2)
        return cache[i]

    times = []
    for s in range(args.warmup + args.steps):
        x = tensor(s % cfg["tensors"])
        t0 = time.perf_counter()
        blob = oracle.encode(x)
        y = oracle.decode(blob, n)
        dt = time.perf_counter() - t0
        assert y[0] == x[0]
        if s >= args.warmup:
            times.append(dt)
        if len(cache) > 4:
            cache.pop(next(iter(cache)))
    per_step = float(np.mean(times))
    value = 2 * n / per_step / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_step * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "each step: oracle encode + decode of one 64 MiB (layer, K/V) tensor, "
                                   "tensors taken in order"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(host_cache, seconds):
    """The oracle as it stands (one thread) on the first tensors of the
    workload until about `seconds` of CPU work have run."""
    import oracle
    oracle.build()
    n = host_cache.shape[1]
    done, t_total = 0, 0.0
    while done < host_cache.shape[0] and t_total < seconds:
        x = host_cache[done].view(np.uint16)
        t0 = time.perf_counter()
        blob = oracle.encode(x)
        oracle.decode(blob, n)
        t_total += time.perf_counter() - t0
        done += 1
    return {"value": round(2 * n * done / t_total / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": "oracle encode + decode of the first %d of %d (layer, K/V) tensors (%.1f s)"
                      % (done, host_cache.shape[0], t_total)}


# ------------------------------------------------------------ latency sweep
def run_sweep(args):
    """Encode (histogram + codebook + container) and decode latency of one
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
    for b in sizes_b:
        n = b // 2
        x = d_flat[:n]
        c_cap, w_need = sz.sz_plan(n)
        with torch.cuda.stream(stream):
            def enc():
                sz.sz_histogram_codebook(x, n, cb, None, ws, w_need, stream)
                sz.sz_encode(x, n, cb, out, c_cap, size, est, ws, w_need, stream)

            def dcd():
                sz.sz_decode(out, c_cap, dec, n, dst, ws, w_need, stream)

            enc(); dcd()
            g_enc, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_enc, stream=stream):
                enc()
            with torch.cuda.graph(g_dec, stream=stream):
                dcd()
            te, td = [], []
            for _ in range(3 + args.sweep_reps):
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                flush.fill_(1)
                ev[0].record(stream); g_enc.replay(); ev[1].record(stream)
                flush.fill_(2)
                ev[2].record(stream); g_dec.replay(); ev[3].record(stream)
                stream.synchronize()
                te.append(ev[0].elapsed_time(ev[1]) / 1e3)
                td.append(ev[2].elapsed_time(ev[3]) / 1e3)
            te, td = float(np.median(te[3:])), float(np.median(td[3:]))
            assert int(est.item()) == 0 and int(dst.item()) == 0, (b, int(est.item()), int(dst.item()))
            comp = int(size.item())
            ok = bool(torch.equal(dec[:n], x))
            del g_enc, g_dec
        line = {"sweep": "single stream, first bytes of llama3-8b-kv-32k", "bytes": b, "elems": n,
                "encode_us": round(te * 1e6, 2), "decode_us": round(td * 1e6, 2),
                "encode_gbs": round(b / te / 1e9, 2), "decode_gbs": round(b / td / 1e9, 2),
                "encode_roofline_frac": round((b + comp) / te / 1e9 / peak, 4),
                "decode_roofline_frac": round((b + comp) / td / 1e9 / peak, 4),
                "ratio": round(b / comp, 5), "round_trip": ok,
                "peak_gbs": peak, "peak_kind": peak_kind, "reps": args.sweep_reps,
                "timing": "CUDA graph replay between events, median; L2 flushed (512 MiB write) before each"}
        print(json.dumps(line), flush=True)


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

    cfg = workload_config(args.tensors)
    S, n = cfg["tensors"], cfg["elems_per_tensor"]
    U = 2 * S * n  # uncompressed bytes per step on this rank

    # inputs: generated on the host straight into pinned memory, then resident in HBM
    h_in = torch.empty((S, n), dtype=torch.int16, pin_memory=True)
    host = h_in.numpy().view(np.uint16)
    if S % 2 == 0:
        kvgen.contiguous_cache(WORKLOAD, layers=S // 2, out=host)
    else:
        for k in range(S):
            host[k] = kvgen.contiguous_tensor(WORKLOAD, k // 2, k % 2)
    d_in = h_in.to(dev, non_blocking=False)
    d_out = torch.empty_like(d_in)
    plan = sz.BatchPlan([n] * S, n, device=dev)
    in_ptrs = torch.tensor([d_in.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=dev)
    out_ptrs = torch.tensor([d_out.data_ptr() + 2 * n * k for k in range(S)], dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        plan.histogram(in_ptrs, stream)
        if ev is not None:
            ev[1].record(stream)
        plan.encode_only(in_ptrs, stream)
        if ev is not None:
            ev[2].record(stream)
        plan.decode(out_ptrs, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if int(plan.enc_status.abs().sum()) or int(plan.dec_status.abs().sum()):
        raise RuntimeError("device status: encode %s decode %s" % (plan.enc_status.tolist(), plan.dec_status.tolist()))

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    clocks = ClockSampler(vis.split(",")[local] if vis else str(local))
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.25)  # let the sampler take its first reading
    for k in range(args.steps):
        step(evs[k])
    torch.cuda.synchronize(dev)
    clock_info = clocks.stop()
    barrier()

    t_hist = np.array([e[0].elapsed_time(e[1]) for e in evs]) / 1e3
    t_enc = np.array([e[1].elapsed_time(e[2]) for e in evs]) / 1e3
    t_dec = np.array([e[2].elapsed_time(e[3]) for e in evs]) / 1e3
    total_s = evs[0][0].elapsed_time(evs[-1][3]) / 1e3
    ms_step = total_s / args.steps * 1e3
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
    esc = int(((sizes - (HEADER + n + (n + 1) // 2)) // 5).sum())
    round_trip_ok = bool(torch.equal(d_out, d_in))

    # ---- self-checks of the last step (bit-exactness against the oracle is
    # the parity tests' job): every tensor round-trips, and every container's
    # header states its length and escape count consistently
    hdr_ok = True
    for k in (0, S - 1):
        off = int(plan.out_offset[k])
        h = plan.container[off: off + HEADER].cpu().numpy()
        hn = int(h[8:16].view(np.uint64)[0])
        he = int(h[16:24].view(np.uint64)[0])
        hdr_ok &= bytes(h[:4]) == b"SZKV" and hn == n and HEADER + n + (n + 1) // 2 + 5 * he == int(sizes[k])
    parity = {"decode_round_trip_all_tensors": round_trip_ok, "header_size_consistent": bool(hdr_ok)}

    # ---- roofline (algorithmic bytes / event time, per phase)
    peak, peak_kind = measured_peak()
    phases = {
        "histogram+select": (2 * S * n, th),
        "encode_kernel": (2 * S * n + comp, te),
        "decode": (comp + 2 * S * n, td),
    }
    roof = {}
    for name, (b, t) in phases.items():
        a = b / t / 1e9
        roof[name] = {"achieved": round(a, 1), "frac": round(a / peak, 4), "ms": round(t * 1e3, 4),
                      "algorithmic_bytes": b}
    dom = max(phases, key=lambda k: phases[k][1])
    enc_e2e_bytes = 2 * S * n + comp
    encode_s = th + te
    layers_full = kvgen.CONTIGUOUS[WORKLOAD][0]
    roofline = {"bound": "hbm", "kernel": dom, "achieved": roof[dom]["achieved"], "peak": peak, "unit": "GB/s",
                "frac": roof[dom]["frac"], "traffic": profiled_traffic(dom, S, 2 * layers_full),
                "peak_kind": peak_kind + " (copy, MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"}

    # ---- one pass with the codebooks kept from the timed steps (codebook
    # reuse): the input is read once; the containers must be the same bytes
    one_pass = None
    if not args.no_one_pass:
        plan1 = sz.BatchPlan([n] * S, n, device=dev)
        cbs = plan.codebooks.clone()
        for _ in range(3):
            plan1.encode_one_pass(in_ptrs, cbs, stream)
        torch.cuda.synchronize(dev)
        same = bool(torch.equal(plan1.sizes, plan.sizes)) and int(plan1.enc_status.abs().sum()) == 0
        for k in range(S):
            o, z = int(plan.out_offset[k]), int(sizes[k])
            same = same and bool(torch.equal(plan1.container[o: o + z], plan.container[o: o + z]))
        k1 = max(1, min(args.steps, 50))
        ev1 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k1)]
        for a0, a1 in ev1:
            a0.record(stream)
            plan1.encode_one_pass(in_ptrs, cbs, stream)
            a1.record(stream)
        torch.cuda.synchronize(dev)
        t1 = float(np.mean([a0.elapsed_time(a1) for a0, a1 in ev1])) / 1e3
        one_pass = {"encode_gbs": round(U / t1 / 1e9, 2), "ms": round(t1 * 1e3, 4),
                    "roofline_frac": round((2 * S * n + comp) / t1 / 1e9 / peak, 4),
                    "same_containers_as_two_pass": same, "steps": k1,
                    "codebooks": "kept from the two-pass encode of the same tensors",
                    "launches": "one-pass encode, escape placement, overflow rescan"}
        del plan1

    # ---- end to end: pinned host buffers, copies inside the timed region.
    # The cache goes up, is encoded, its containers come down and go up
    # again, are decoded and the BF16 values come down -- chunks of 4
    # tensors, uploads and downloads on their own streams so that both
    # directions of the link stay busy while the kernels run in between.
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        from lossless_bf16_kv_splitzip_b200.transfer import SplitZipChunks, host_round_trip
        per_chunk = 4
        rt = SplitZipChunks(d_in, d_out, per_chunk, dev)
        h_out = torch.empty((S, n), dtype=torch.int16, pin_memory=True)
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
        cpu = cpu_baseline(h_in.numpy(), args.cpu_seconds)

    if rank == 0:
        value = world * U / (ms_step / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u16", "data": "synthetic", "config": cfg,
            "encode_gbs": round(U / encode_s / 1e9, 2), "decode_gbs": round(U / td / 1e9, 2),
            "encode_roofline_frac": round(enc_e2e_bytes / encode_s / 1e9 / peak, 4),
            "decode_roofline_frac": roof["decode"]["frac"],
            "encode_one_pass": one_pass,
            "ratio": round(U / comp, 5), "escape_frac": round(esc / (S * n), 6),
            "roofline": roofline, "roofline_phases": roof,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 4 * args.steps,  # hist, encode, esc_index, decode
            "clocks": clock_info, "parity": parity,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
