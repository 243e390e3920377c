#!/usr/bin/env python
"""Benchmark of the TurboQuant packed-KV hot path on B200.

One step = one pass of the whole hot path over one batch of the workload:
quantize-append of the step's tokens (rotate, norm, encode, pack, store) and
then one paged decode step over the packed pages for every sequence.  The
default workload is the Llama-3-8B-shaped layer (32 q heads, 8 KV heads, D=128,
4-bit K and V, batch 32 x 8192 tokens): the step appends all 262,144 tokens
(4,194,304 rows) and decodes 32 queries over them.

Prints ONE JSON line (rank 0).  ``value`` is whole-step algorithmic HBM
throughput (append bytes + decode packed bytes, over the step time, summed over
ranks); the per-op breakdown (decode packed-KV GB/s, append Mrows/s) sits in
``decode`` and ``append``.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--config C]
       python bench.py --impl reference ...   (the CPU oracle, as it stands)
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TQ paged decode: packed-KV HBM GB/s (% of peak); quantize-append Mrows/s"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ("kv_cache_vector_append_b200/csrc/tq_append.cuh",
                  "kv_cache_vector_append_b200/csrc/tq_decode.cuh",
                  "kv_cache_vector_append_b200/csrc/tq_device.cuh")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2, help="workload index (see workloads.CONFIGS)")
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# bytes and units
# ---------------------------------------------------------------------------

def append_bytes(spec, n_tokens):
    """Algorithmic bytes of quantize-append: per (token, KV head) read 2 rows of D
    inputs, write slot_bytes; plus 8 bytes of slot_mapping per token."""
    d = spec.head_dim
    es = 4 if spec.dtype == "float32" else 2
    sb = (d * spec.k_bits + 7) // 8 + 4 + (d * spec.v_bits + 7) // 8 + 4
    return n_tokens * spec.num_kv_heads * (2 * d * es + sb) + 8 * n_tokens


def decode_bytes(spec, seq_lens):
    """Algorithmic bytes of paged decode: slot_bytes per (token, KV head), 4 bytes
    of block table per 16 tokens, q read and out written."""
    d = spec.head_dim
    es = 4 if spec.dtype == "float32" else 2
    sb = (d * spec.k_bits + 7) // 8 + 4 + (d * spec.v_bits + 7) // 8 + 4
    lens = np.asarray(seq_lens, dtype=np.int64)
    packed = int(lens.sum()) * spec.num_kv_heads * sb
    bt = int(((lens + 15) // 16).sum()) * 4
    return packed + bt + 2 * len(lens) * spec.num_q_heads * d * es, packed


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_name, config_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        e = j[config_name][kernel_name]
        return e["dram_bytes_per_launch"] if e.get("kernel_hash") == kernel_hash() else None
    except Exception:
        return None


# ---------------------------------------------------------------------------
# ranks (one process per GPU; replicas, no data-path collective)
# ---------------------------------------------------------------------------

def max_over_ranks(values, device):
    """Element-wise max of a list of floats over all ranks (identity when the
    process group is not initialised).  Device-measured times are combined this
    way: the job is as slow as its slowest rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_gbs(world, bytes_per_step, ms_per_step):
    """Whole-job throughput: every rank processes its own replica of the step."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clocks and clock-event reasons through NVML (read-only) in a
    background thread while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index, interval_s=0.002):
        self.gpu = gpu_index
        self.interval = interval_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None

    def _run(self):
        import pynvml
        h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        while not self._stop.is_set():
            try:
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.interval)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self._stop = None
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        sm = self.samples
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_step(wl, tables, n_append=1024, n_decode_tokens=2048, seq=0):
    """One bounded oracle step on the workload: quantize-append of n_append tokens
    of sequence `seq` into a page pool, then a decode step of that sequence over
    its first n_decode_tokens tokens.  Returns (seconds, algorithmic bytes, text)."""
    from oracle import tq_oracle as O
    spec = wl.spec
    kt, vt = tables
    seq = int(seq) % max(1, spec.batch)
    start = int(wl.seq_lens[:seq].astype(np.int64).sum())
    n_dec = int(min(n_decode_tokens, wl.seq_lens[seq]))
    n_app = int(min(n_append, n_dec))
    pages = np.zeros((wl.num_blocks, 16, spec.num_kv_heads, wl.slot_bytes), dtype=np.uint8)
    slots = wl.slot_mapping[start:start + n_dec]
    k = wl.k[start:start + n_dec].float().numpy()
    v = wl.v[start:start + n_dec].float().numpy()
    # the untimed part fills the decode range; the timed part re-appends n_app tokens
    pages = O.quantize_append(pages, slots, k, v, kt, vt, spec.sign_seed)
    t0 = time.perf_counter()
    c0 = time.process_time()
    pages = O.quantize_append(pages, slots[:n_app], k[:n_app], v[:n_app], kt, vt,
                              spec.sign_seed)
    q = wl.q[seq:seq + 1].float().numpy().astype(np.float64)
    O.paged_decode(q, pages, wl.block_table[seq:seq + 1], np.array([n_dec], dtype=np.int32),
                   kt, vt, spec.sign_seed, spec.scale)
    dt = time.perf_counter() - t0
    oracle_sample_step.cpu_seconds = time.process_time() - c0
    nbytes = append_bytes(spec, n_app) + decode_bytes(spec, [n_dec])[0]
    desc = (f"{n_app} tokens x {spec.num_kv_heads} KV heads appended + 1 sequence x {n_dec} "
            f"tokens x {spec.num_q_heads} q heads decoded")
    return dt, nbytes, desc


def cpu_baseline(wl, tables, min_seconds=10.0, max_samples=64):
    """The oracle timed on host cores over repeated bounded samples (one per
    sequence, cycling) until at least min_seconds of oracle work has run."""
    oracle_sample_step(wl, tables, 256, 512)   # warm caches
    total_t = total_b = total_cpu = 0.0
    n = 0
    desc = ""
    while n < max_samples and (total_t < min_seconds or n == 0):
        dt, nb, desc = oracle_sample_step(wl, tables, seq=n)
        total_t += dt
        total_b += nb
        total_cpu += oracle_sample_step.cpu_seconds
        n += 1
    return {"value": total_b / total_t / 1e9, "unit": "GB/s",
            "cores": effective_cores(total_cpu, total_t), "threads_available": blas_threads(),
            "kind": "oracle", "sample": f"{n} samples (sequences 0..{n - 1}, cycling) of: {desc}",
            "seconds": total_t}


def effective_cores(cpu_seconds, wall_seconds):
    """Host cores the oracle kept busy on average: process CPU time over wall time."""
    return round(max(1.0, cpu_seconds / wall_seconds), 1) if wall_seconds > 0 else 1.0


def oracle_tables(spec):
    from oracle import gen_codebooks as G
    kt = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(spec.head_dim, spec.k_bits)))
    vt = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(spec.head_dim, spec.v_bits)))
    return kt, vt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from kv_cache_vector_append_b200 import workloads as W
    spec = W.CONFIGS[args.config]
    wl = W.generate(spec)
    tables = oracle_tables(spec)
    for i in range(args.warmup):
        oracle_sample_step(wl, tables, seq=i)
    total_t = total_b = total_cpu = 0.0
    desc = ""
    for i in range(args.steps):
        dt, nb, desc = oracle_sample_step(wl, tables, seq=args.warmup + i)
        total_t += dt
        total_b += nb
        total_cpu += oracle_sample_step.cpu_seconds
    value = total_b / total_t / 1e9
    cores = effective_cores(total_cpu, total_t)
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": spec.name, "batch": spec.batch, "seq_len":
                       spec.seq_len or list(spec.seq_len_range), "head_dim": spec.head_dim,
                       "q_heads": spec.num_q_heads, "kv_heads": spec.num_kv_heads,
                       "k_bits": spec.k_bits, "v_bits": spec.v_bits,
                       "parallelism": "replicas" if args.gpus > 1 else "single"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores,
                             "threads_available": blas_threads(), "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args):
    import torch
    import torch.distributed as dist
    import kv_cache_vector_append_b200 as tq
    from kv_cache_vector_append_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    spec = W.CONFIGS[args.config]
    if args.batch:
        spec = spec.scaled(batch=args.batch)
    wl = W.generate(spec)
    step_idx = torch.from_numpy(wl.step_tokens)
    setup_idx = torch.from_numpy(wl.setup_tokens)
    cb = tq.load_codebooks(spec.head_dim, spec.k_bits, spec.v_bits, dev)
    pages = W.empty_pages(wl, device=dev)
    k_step = wl.k[step_idx].to(dev)
    v_step = wl.v[step_idx].to(dev)
    sm_step = torch.from_numpy(wl.slot_mapping[wl.step_tokens]).to(dev)
    q = wl.q.to(dev)
    out = torch.empty_like(q)
    bt = torch.from_numpy(wl.block_table).to(dev)
    sl = torch.from_numpy(wl.seq_lens).to(dev)
    if len(wl.setup_tokens):
        for s in range(0, len(wl.setup_tokens), 1 << 18):
            ii = setup_idx[s:s + (1 << 18)]
            tq.quantize_append(pages, torch.from_numpy(wl.slot_mapping[ii.numpy()]).to(dev),
                               wl.k[ii].to(dev), wl.v[ii].to(dev), cb, spec.sign_seed)
    ws_bytes = tq.decode_workspace_size(spec.batch, spec.num_q_heads, spec.num_kv_heads,
                                        spec.head_dim, wl.block_table.shape[1])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    tq.set_workspace(ws)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    n_step = len(wl.step_tokens)
    a_bytes = append_bytes(spec, n_step)
    d_bytes, d_packed = decode_bytes(spec, wl.seq_lens)
    step_bytes = a_bytes + d_bytes
    rows = 2 * n_step * spec.num_kv_heads

    def step():
        tq.quantize_append(pages, sm_step, k_step, v_step, cb, spec.sign_seed, stream)
        tq.paged_decode(out, q, pages, bt, sl, cb, spec.sign_seed, spec.scale, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if world == 1 else local) as clk:
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            tq.quantize_append(pages, sm_step, k_step, v_step, cb, spec.sign_seed, stream)
            ev[i][1].record(stream)
            tq.paged_decode(out, q, pages, bt, sl, cb, spec.sign_seed, spec.scale, stream)
            ev[i][2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    app_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in ev]))
    dec_ms = float(np.mean([b.elapsed_time(c) for _, b, c in ev]))
    total_ms, app_ms, dec_ms = max_over_ranks([total_ms, app_ms, dec_ms], dev)
    err = tq.get_device_error(stream)
    if err:
        raise RuntimeError(f"device error word {err:#x} during the bench")

    # ---- end to end through the public API, host buffers ----
    e2e = None
    if not args.no_e2e:
        k_h = wl.k[step_idx].pin_memory()
        v_h = wl.v[step_idx].pin_memory()
        sm_h = torch.from_numpy(wl.slot_mapping[wl.step_tokens]).pin_memory()
        q_h = wl.q.pin_memory()
        bt_h = torch.from_numpy(wl.block_table).pin_memory()
        sl_h = torch.from_numpy(wl.seq_lens).pin_memory()
        out_h = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (k_h, v_h, sm_h, q_h, bt_h, sl_h))
        d2h = out_h.numel() * out_h.element_size()

        def e2e_step():
            k_step.copy_(k_h, non_blocking=True)
            v_step.copy_(v_h, non_blocking=True)
            sm_step.copy_(sm_h, non_blocking=True)
            q.copy_(q_h, non_blocking=True)
            bt.copy_(bt_h, non_blocking=True)
            sl.copy_(sl_h, non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)

        for _ in range(max(args.warmup, 3)):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms, = max_over_ranks([e0.elapsed_time(e1)], dev)
        e2e = {"value": job_gbs(world, step_bytes, e2e_ms / args.steps), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / args.steps}

    if rank != 0:
        if world > 1:
            tq.set_workspace(None)
            dist.destroy_process_group()
        return 0

    peak, peak_kind = measured_peaks()
    ms_per_step = total_ms / args.steps
    value = job_gbs(world, step_bytes, ms_per_step)
    app_gbs = a_bytes / (app_ms * 1e-3) / 1e9
    dec_gbs = d_bytes / (dec_ms * 1e-3) / 1e9
    dec_packed_gbs = d_packed / (dec_ms * 1e-3) / 1e9
    dominant = "append" if app_ms >= dec_ms else "decode"
    dom_kernel = "append_kernel" if dominant == "append" else "decode_kernel"
    dom_gbs = app_gbs if dominant == "append" else dec_gbs
    traffic = ncu_traffic(dom_kernel, spec.name)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "dtype_detail": "f32 rotate/norm/encode; decode contractions f16 x f16 -> f32",
        "data": "synthetic",
        "config": {"workload": spec.name, "batch": spec.batch,
                   "seq_len": spec.seq_len or list(spec.seq_len_range),
                   "head_dim": spec.head_dim, "q_heads": spec.num_q_heads,
                   "kv_heads": spec.num_kv_heads, "k_bits": spec.k_bits, "v_bits": spec.v_bits,
                   "input_dtype": spec.dtype, "step_tokens_appended": n_step,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"inputs larger than L2 ({step_bytes / 1e6:.0f} MB touched per step)"},
        "append": {"ms": app_ms, "mrows_per_s": rows / (app_ms * 1e-3) / 1e6, "gbs": app_gbs,
                   "frac_of_peak": app_gbs / peak, "rows": rows, "bytes": a_bytes},
        "decode": {"ms": dec_ms, "packed_kv_gbs": dec_packed_gbs, "gbs": dec_gbs,
                   "frac_of_peak": dec_gbs / peak,
                   "tokens_per_s": spec.batch / (dec_ms * 1e-3),
                   "kv_tokens_scanned_per_s": float(np.sum(wl.seq_lens)) / (dec_ms * 1e-3),
                   "bytes": d_bytes, "packed_bytes": d_packed},
        "roofline": {"bound": "hbm", "kernel": dom_kernel, "achieved": dom_gbs, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": dom_gbs / peak,
                     "traffic": traffic},
        "roofline_decode": {"bound": "hbm", "kernel": "decode_kernel",
                            "achieved": dec_gbs, "peak": peak, "unit": "GB/s",
                            "frac": dec_gbs / peak,
                            "traffic": ncu_traffic("decode_kernel", spec.name)},
        "gpu_launches": 2 * args.steps,   # append_kernel + decode_kernel
        "clocks": clk.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, oracle_tables(spec))
    print(json.dumps(line), flush=True)
    if world > 1:
        tq.set_workspace(None)
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    raise SystemExit(main())
