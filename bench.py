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
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="skip the configs[3] and configs[4] legs of the default run")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# bytes and units
# ---------------------------------------------------------------------------

def append_bytes(spec, n_tokens, sb=None):
    """Algorithmic bytes of quantize-append: per (token, KV head) read 2 rows of D
    inputs, write slot_bytes (``sb``, default the plain slot); plus 8 bytes of
    slot_mapping per token."""
    d = spec.head_dim
    es = 4 if spec.dtype == "float32" else 2
    if sb is None:
        sb = (d * spec.k_bits + 7) // 8 + 4 + (d * spec.v_bits + 7) // 8 + 4
    return n_tokens * spec.num_kv_heads * (2 * d * es + sb) + 8 * n_tokens


def decode_bytes(spec, seq_lens, sb=None):
    """Algorithmic bytes of paged decode: slot_bytes (``sb``, default the plain slot)
    per (token, KV head), 4 bytes of block table per 16 tokens, q read and out written."""
    d = spec.head_dim
    es = 4 if spec.dtype == "float32" else 2
    if sb is None:
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


def code_text(src):
    """Kernel source without its // comments and blank lines: what the counters depend on."""
    lines = []
    for line in src.splitlines():
        code = line.split("//", 1)[0].rstrip()
        if code.strip():
            lines.append(code)
    return "\n".join(lines)


def kernel_hash():
    """Hash of the kernel sources' code (comments and blank lines ignored), keying the
    committed ncu traffic figures to the kernels they were taken on."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            h.update(code_text(f.read()).encode())
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

def oracle_sample_inputs(wl, seq, n_tokens=2048):
    """Inputs of one bounded oracle sample of the workload: the first n_tokens tokens of
    sequence `seq` (K, V, q as float arrays), appended into a compact page pool of their
    own (block b of the sequence in pool block b) and then decoded.  Plain arrays, so
    that they can go to a worker process."""
    spec = wl.spec
    seq = int(seq) % max(1, spec.batch)
    start = int(wl.seq_lens[:seq].astype(np.int64).sum())
    n_dec = int(min(n_tokens, wl.seq_lens[seq]))
    n_app = n_dec
    return {"k": wl.k[start:start + n_dec].float().numpy(),
            "v": wl.v[start:start + n_dec].float().numpy(),
            "q": wl.q[seq:seq + 1].float().numpy().astype(np.float64),
            "n_app": n_app, "n_dec": n_dec, "h_kv": spec.num_kv_heads,
            "slot_bytes": wl.slot_bytes, "head_dim": spec.head_dim, "k_bits": spec.k_bits,
            "v_bits": spec.v_bits, "sign_seed": spec.sign_seed, "scale": spec.scale,
            "bytes": append_bytes(spec, n_app) + decode_bytes(spec, [n_dec])[0]}


def oracle_sample_run(inp):
    """Run one sample through the oracle as it stands, all of it timed: quantize-append
    of the sample's tokens into an empty pool, then one decode step over them.
    Returns (wall seconds, CPU seconds, algorithmic bytes)."""
    from oracle import gen_codebooks as G
    from oracle import tq_oracle as O
    d = inp["head_dim"]
    kt = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, inp["k_bits"])))
    vt = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(d, inp["v_bits"])))
    n_dec, n_app = inp["n_dec"], inp["n_app"]
    nblk = (n_dec + 15) // 16
    slots = np.arange(n_dec, dtype=np.int64)
    t0 = time.perf_counter()
    c0 = time.process_time()
    pages = np.zeros((nblk, 16, inp["h_kv"], inp["slot_bytes"]), dtype=np.uint8)
    pages = O.quantize_append(pages, slots[:n_app], inp["k"][:n_app], inp["v"][:n_app], kt, vt,
                              inp["sign_seed"])
    O.paged_decode(inp["q"], pages, np.arange(nblk)[None], np.array([n_dec], dtype=np.int32),
                   kt, vt, inp["sign_seed"], inp["scale"])
    return time.perf_counter() - t0, time.process_time() - c0, inp["bytes"]


def _pool_worker(inp):
    """One sample in a worker process, on one BLAS thread."""
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            return oracle_sample_run(inp)
    except ImportError:
        return oracle_sample_run(inp)


def sample_desc(wl, inp):
    s = wl.spec
    return (f"{inp['n_app']} tokens x {s.num_kv_heads} KV heads appended + 1 sequence x "
            f"{inp['n_dec']} tokens x {s.num_q_heads} q heads decoded")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OraclePool:
    """The oracle on all host cores: one spawned worker process per core (spawn, so it
    is safe after CUDA has been initialised), each on one BLAS thread, each running
    whole samples."""

    def __init__(self, cores=None):
        import multiprocessing as mp
        self.cores = cores or host_cores()
        self.pool = mp.get_context("spawn").Pool(self.cores)

    def run(self, inputs):
        """Wall seconds, summed CPU seconds and bytes of running all inputs at once."""
        t0 = time.perf_counter()
        res = self.pool.map(_pool_worker, inputs, chunksize=1)
        wall = time.perf_counter() - t0
        return wall, sum(r[1] for r in res), sum(r[2] for r in res)

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(wl, min_seconds=10.0, max_samples=64):
    """The oracle timed on the host: on one core (samples one after another, one BLAS
    thread, until min_seconds) and on all cores (a spawned worker per core, a batch of
    samples per core, after a warm-up batch)."""
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except ImportError:
        limit = None
    oracle_sample_run(oracle_sample_inputs(wl, 0, 256))     # warm caches
    total_t = total_b = 0.0
    n = 0
    desc = ""
    while n < max_samples and (total_t < min_seconds or n == 0):
        inp = oracle_sample_inputs(wl, n)
        dt, _, nb = oracle_sample_run(inp)
        desc = sample_desc(wl, inp)
        total_t += dt
        total_b += nb
        n += 1
    if limit is not None:
        limit.unregister()
    single = {"value": total_b / total_t / 1e9, "cores": 1, "seconds": total_t,
              "sample": f"{n} samples (sequences 0..{n - 1}, cycling) of: {desc}"}
    pool = OraclePool()
    try:
        cores = pool.cores
        pool.run([oracle_sample_inputs(wl, i, 256) for i in range(cores)])   # warm-up
        per_core = max(1, int(round(min_seconds / max(total_t / n, 1e-3) / 2)))
        inputs = [oracle_sample_inputs(wl, i) for i in range(cores * per_core)]
        wall, cpu, nbytes = pool.run(inputs)
    finally:
        pool.close()
    return {"value": nbytes / wall / 1e9, "unit": "GB/s", "cores": cores,
            "cpu_seconds_per_wall_second": round(cpu / wall, 1), "kind": "oracle",
            "sample": f"{len(inputs)} samples ({per_core} per core, sequences cycling) of: "
                      f"{desc}", "seconds": wall, "single_core": single}


def oracle_tables(spec):
    from oracle import gen_codebooks as G
    kt = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(spec.head_dim, spec.k_bits)))
    vt = G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(spec.head_dim, spec.v_bits)))
    return kt, vt


def config_dict(spec, world, n_step_tokens, step_bytes):
    """The `config` object of the JSON line (the same in both arms)."""
    return {"workload": spec.name, "batch": spec.batch,
            "seq_len": spec.seq_len or list(spec.seq_len_range),
            "head_dim": spec.head_dim, "q_heads": spec.num_q_heads,
            "kv_heads": spec.num_kv_heads, "k_bits": spec.k_bits, "v_bits": spec.v_bits,
            "input_dtype": spec.dtype, "step_tokens_appended": int(n_step_tokens),
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": f"inputs larger than L2 ({step_bytes / 1e6:.0f} MB touched per step)"}


def step_shape(wl):
    """Tokens appended and algorithmic bytes of one full step of the workload."""
    n_step = len(wl.step_tokens)
    return n_step, append_bytes(wl.spec, n_step) + decode_bytes(wl.spec, wl.seq_lens)[0]


def run_reference(args):
    """The CPU oracle as it stands, on all host cores: each step is one batch of bounded
    samples of the workload, one per core, run at once."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from kv_cache_vector_append_b200 import workloads as W
    spec = W.CONFIGS[args.config]
    wl = W.generate(spec)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    n_step, step_bytes = step_shape(wl)
    pool = OraclePool()
    try:
        cores = pool.cores
        for i in range(args.warmup):
            pool.run([oracle_sample_inputs(wl, i * cores + j, 256) for j in range(cores)])
        total_t = total_b = total_cpu = 0.0
        inp = None
        for i in range(args.steps):
            inputs = [oracle_sample_inputs(wl, i * cores + j) for j in range(cores)]
            inp = inputs[0]
            wall, cpu, nb = pool.run(inputs)
            total_t += wall
            total_cpu += cpu
            total_b += nb
    finally:
        pool.close()
    value = total_b / total_t / 1e9
    desc = f"{cores} samples per step (one per core) of: {sample_desc(wl, inp)}"
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_dict(spec, world, n_step, step_bytes),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores,
                             "cpu_seconds_per_wall_second": round(total_cpu / total_t, 1),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def device_inputs(wl, dev):
    """The workload's step inputs, page pool (with the untimed setup tokens already
    appended) and decode inputs on the device."""
    import torch
    import kv_cache_vector_append_b200 as tq
    from kv_cache_vector_append_b200 import workloads as W
    spec = wl.spec
    step_idx = torch.from_numpy(wl.step_tokens)
    setup_idx = torch.from_numpy(wl.setup_tokens)
    cb = tq.load_codebooks(spec.head_dim, spec.k_bits, spec.v_bits, dev)
    pages = W.empty_pages(wl, device=dev)
    for s in range(0, len(wl.setup_tokens), 1 << 18):
        ii = setup_idx[s:s + (1 << 18)]
        tq.quantize_append(pages, torch.from_numpy(wl.slot_mapping[ii.numpy()]).to(dev),
                           wl.k[ii].to(dev), wl.v[ii].to(dev), cb, spec.sign_seed)
    return {"cb": cb, "pages": pages, "k": wl.k[step_idx].to(dev), "v": wl.v[step_idx].to(dev),
            "sm": torch.from_numpy(wl.slot_mapping[wl.step_tokens]).to(dev),
            "q": wl.q.to(dev), "out": torch.empty(wl.q.shape, dtype=wl.q.dtype, device=dev),
            "bt": torch.from_numpy(wl.block_table).to(dev),
            "sl": torch.from_numpy(wl.seq_lens).to(dev)}


def time_legs(spec, x, steps, stream, flush=None):
    """Mean ms of the append and of the decode over `steps` timed steps (CUDA events on
    the launching stream).  With `flush` (a device buffer larger than L2) the buffer is
    rewritten before every decode, outside its events."""
    import torch
    import kv_cache_vector_append_b200 as tq
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for i in range(steps):
        ev[i][0].record(stream)
        tq.quantize_append(x["pages"], x["sm"], x["k"], x["v"], x["cb"], spec.sign_seed, stream)
        ev[i][1].record(stream)
        if flush is not None:
            flush.add_(1)
        ev[i][2].record(stream)
        tq.paged_decode(x["out"], x["q"], x["pages"], x["bt"], x["sl"], x["cb"], spec.sign_seed,
                        spec.scale, stream)
        ev[i][3].record(stream)
    torch.cuda.synchronize()
    return (float(np.mean([e[0].elapsed_time(e[1]) for e in ev])),
            float(np.mean([e[2].elapsed_time(e[3]) for e in ev])))


def leg_summary(wl, app_ms, dec_ms, peak, sb=None):
    spec = wl.spec
    n_step = len(wl.step_tokens)
    a_bytes = append_bytes(spec, n_step, sb)
    d_bytes, d_packed = decode_bytes(spec, wl.seq_lens, sb)
    rows = 2 * n_step * spec.num_kv_heads
    return {"append": {"ms": app_ms, "mrows_per_s": rows / (app_ms * 1e-3) / 1e6,
                       "gbs": a_bytes / (app_ms * 1e-3) / 1e9,
                       "frac_of_peak": a_bytes / (app_ms * 1e-3) / 1e9 / peak, "rows": rows,
                       "bytes": a_bytes},
            "decode": {"ms": dec_ms, "packed_kv_gbs": d_packed / (dec_ms * 1e-3) / 1e9,
                       "gbs": d_bytes / (dec_ms * 1e-3) / 1e9,
                       "frac_of_peak": d_bytes / (dec_ms * 1e-3) / 1e9 / peak,
                       "tokens_per_s": spec.batch / (dec_ms * 1e-3),
                       "kv_tokens_scanned_per_s": float(np.sum(wl.seq_lens)) / (dec_ms * 1e-3),
                       "bytes": d_bytes, "packed_bytes": d_packed}}


def extra_config_legs(configs, dev, steps, warmup, peak):
    """Append and decode of other workloads on this GPU (timed like the main step,
    each in its own timed region): configs 3 and 4 by default.  configs[4]'s page pool
    (92 MB) fits in L2, so its decode is also timed with L2 rewritten before each
    launch."""
    import torch
    import kv_cache_vector_append_b200 as tq
    from kv_cache_vector_append_b200 import workloads as W
    stream = torch.cuda.current_stream(dev)
    res = {}
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    for c in configs:
        wl = W.generate(W.CONFIGS[c])
        spec = wl.spec
        x = device_inputs(wl, dev)
        ws = tq.decode_workspace_size(spec.batch, spec.num_q_heads, spec.num_kv_heads,
                                      spec.head_dim, wl.block_table.shape[1])
        ws_t = torch.empty(ws, dtype=torch.uint8, device=dev)
        tq.set_workspace(ws_t)
        time_legs(spec, x, max(warmup, 3), stream)
        app_ms, dec_ms = time_legs(spec, x, steps, stream)
        leg = leg_summary(wl, app_ms, dec_ms, peak)
        leg["step_tokens_appended"] = int(len(wl.step_tokens))
        if c == 4:
            flush = torch.zeros(4 * l2 // 4, dtype=torch.float32, device=dev)
            time_legs(spec, x, max(warmup, 3), stream, flush)
            _, dec_f = time_legs(spec, x, steps, stream, flush)
            leg["decode_l2_flushed"] = leg_summary(wl, app_ms, dec_f, peak)["decode"]
            leg["decode_l2_flushed"]["flush_bytes"] = int(flush.numel() * 4)
            del flush
        if tq.get_device_error(stream):
            raise RuntimeError(f"device error during the {spec.name} leg")
        tq.set_workspace(None)
        res[spec.name] = leg
        del x, ws_t
        torch.cuda.empty_cache()
    return res


def variant_legs(wl, x, dev, steps, warmup, peak):
    """The survey's next rows on the main workload, each in its own timed region:
    quantize-append and decode with the dense (QR) rotation (tcgen05 GEMM), the decode
    with a 64-token uncompressed hot window per sequence (bf16), and quantize-append and
    decode of keys that carry the QJL residual sketch."""
    import torch
    import kv_cache_vector_append_b200 as tq
    spec = wl.spec
    stream = torch.cuda.current_stream(dev)
    res = {}
    ev = lambda: torch.cuda.Event(enable_timing=True)   # noqa: E731
    if spec.head_dim in (64, 128):
        rot = tq.load_rotation(spec.head_dim, dev)

        def dense_step():
            tq.quantize_append_dense(x["pages"], x["sm"], x["k"], x["v"], x["cb"], rot, stream)
            tq.paged_decode_dense(x["out"], x["q"], x["pages"], x["bt"], x["sl"], x["cb"], rot,
                                  spec.scale, stream)
        for _ in range(max(warmup, 3)):
            dense_step()
        torch.cuda.synchronize(dev)
        e = [[ev() for _ in range(3)] for _ in range(steps)]
        for i in range(steps):
            e[i][0].record(stream)
            tq.quantize_append_dense(x["pages"], x["sm"], x["k"], x["v"], x["cb"], rot, stream)
            e[i][1].record(stream)
            tq.paged_decode_dense(x["out"], x["q"], x["pages"], x["bt"], x["sl"], x["cb"], rot,
                                  spec.scale, stream)
            e[i][2].record(stream)
        torch.cuda.synchronize(dev)
        app = float(np.mean([a.elapsed_time(b) for a, b, _ in e]))
        dec = float(np.mean([b.elapsed_time(c) for _, b, c in e]))
        leg = leg_summary(wl, app, dec, peak)
        n_rows = len(wl.step_tokens) * spec.num_kv_heads
        leg["append"]["tensor_tflops"] = 2 * 2 * n_rows * 2 * spec.head_dim ** 2 / (app * 1e-3) / 1e12
        res["dense_rotation"] = leg
        # the RHT pages again for the rest of the run
        tq.quantize_append(x["pages"], x["sm"], x["k"], x["v"], x["cb"], spec.sign_seed, stream)
    w = 64
    g = torch.Generator().manual_seed(7)
    hk = torch.randn(spec.batch, w, spec.num_kv_heads, spec.head_dim, generator=g).to(
        torch.bfloat16).to(dev)
    hv = torch.randn(spec.batch, w, spec.num_kv_heads, spec.head_dim, generator=g).to(
        torch.bfloat16).to(dev)
    hl = torch.full((spec.batch,), w, dtype=torch.int32, device=dev)
    for _ in range(max(warmup, 3)):
        tq.paged_decode_hot(x["out"], x["q"], x["pages"], x["bt"], x["sl"], hk, hv, hl, x["cb"],
                            spec.sign_seed, spec.scale, stream)
    torch.cuda.synchronize(dev)
    e0, e1 = ev(), ev()
    e0.record(stream)
    for _ in range(steps):
        tq.paged_decode_hot(x["out"], x["q"], x["pages"], x["bt"], x["sl"], hk, hv, hl, x["cb"],
                            spec.sign_seed, spec.scale, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dec = e0.elapsed_time(e1) / steps
    d_bytes, d_packed = decode_bytes(spec, wl.seq_lens)
    hot_bytes = 2 * spec.batch * w * spec.num_kv_heads * spec.head_dim * 2
    res["hot_window"] = {"window_tokens": w, "ms": dec,
                         "gbs": (d_bytes + hot_bytes) / (dec * 1e-3) / 1e9,
                         "frac_of_peak": (d_bytes + hot_bytes) / (dec * 1e-3) / 1e9 / peak}
    # keys that also carry the QJL sketch of their residual: their own page pool (the slot
    # is larger, its stride a multiple of 8)
    if spec.head_dim >= 128 and spec.k_bits <= 4:
        from kv_cache_vector_append_b200 import workloads as W
        sbq = tq.slot_bytes_qjl(spec.head_dim, spec.k_bits, spec.v_bits)
        qpages = W.empty_pages(wl, device=dev, slot_stride=(sbq + 7) // 8 * 8)
        qseed = spec.sign_seed + 1
        for _ in range(max(warmup, 3)):
            tq.quantize_append_qjl(qpages, x["sm"], x["k"], x["v"], x["cb"], spec.sign_seed,
                                   qseed, stream)
            tq.paged_decode_qjl(x["out"], x["q"], qpages, x["bt"], x["sl"], x["cb"],
                                spec.sign_seed, qseed, spec.scale, stream)
        torch.cuda.synchronize(dev)
        e = [[ev() for _ in range(3)] for _ in range(steps)]
        for i in range(steps):
            e[i][0].record(stream)
            tq.quantize_append_qjl(qpages, x["sm"], x["k"], x["v"], x["cb"], spec.sign_seed,
                                   qseed, stream)
            e[i][1].record(stream)
            tq.paged_decode_qjl(x["out"], x["q"], qpages, x["bt"], x["sl"], x["cb"],
                                spec.sign_seed, qseed, spec.scale, stream)
            e[i][2].record(stream)
        torch.cuda.synchronize(dev)
        app = float(np.mean([a.elapsed_time(b) for a, b, _ in e]))
        dec = float(np.mean([b.elapsed_time(c) for _, b, c in e]))
        res["qjl"] = dict(leg_summary(wl, app, dec, peak, sb=sbq), slot_bytes=sbq)
        del qpages
    if tq.get_device_error(stream):
        raise RuntimeError("device error during the variant legs")
    return res


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import kv_cache_vector_append_b200 as tq
    from kv_cache_vector_append_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
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
    x = device_inputs(wl, dev)
    cb, pages, k_step, v_step, sm_step = x["cb"], x["pages"], x["k"], x["v"], x["sm"]
    q, out, bt, sl = x["q"], x["out"], x["bt"], x["sl"]
    ws_bytes = tq.decode_workspace_size(spec.batch, spec.num_q_heads, spec.num_kv_heads,
                                        spec.head_dim, wl.block_table.shape[1])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    tq.set_workspace(ws)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    n_step, step_bytes = step_shape(wl)
    d_bytes, _ = decode_bytes(spec, wl.seq_lens)
    step_bytes = append_bytes(spec, n_step) + d_bytes

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
        step_idx = torch.from_numpy(wl.step_tokens)
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

    peak, peak_kind = measured_peaks()
    variants = None
    if not args.no_extra_configs:
        variants = variant_legs(wl, x, dev, args.steps, args.warmup, peak)
    extra = None
    if not args.no_extra_configs and args.config == 2 and not args.batch:
        tq.set_workspace(None)
        del x
        extra = extra_config_legs((3, 4), dev, args.steps, args.warmup, peak)
        tq.set_workspace(ws)

    if rank != 0:
        if world > 1:
            tq.set_workspace(None)
            dist.destroy_process_group()
        return 0

    ms_per_step = total_ms / args.steps
    value = job_gbs(world, step_bytes, ms_per_step)
    legs = leg_summary(wl, app_ms, dec_ms, peak)
    dominant = "append" if app_ms >= dec_ms else "decode"
    dom_kernel = "append_kernel" if dominant == "append" else "decode_kernel"
    dom_gbs = legs[dominant]["gbs"]
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32+f16",
        "dtype_detail": "append: f32 rotate/norm/encode; decode: f32 query rotation, softmax "
                        "and merge, score and value contractions on f16 x f16 -> f32 mma",
        "data": "synthetic",
        "config": config_dict(spec, world, n_step, step_bytes),
        "append": legs["append"], "decode": legs["decode"],
        "roofline": {"bound": "hbm", "kernel": dom_kernel, "achieved": dom_gbs, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": dom_gbs / peak,
                     "traffic": ncu_traffic(dom_kernel, spec.name)},
        "roofline_decode": {"bound": "hbm", "kernel": "decode_kernel",
                            "achieved": legs["decode"]["gbs"], "peak": peak, "unit": "GB/s",
                            "frac": legs["decode"]["gbs"] / peak,
                            "traffic": ncu_traffic("decode_kernel", spec.name)},
        # append_kernel (fast path) + its redo launch (returns at once unless flagged) +
        # decode_kernel, per step
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }
    if variants:
        line["variants"] = variants
    if extra:
        line["other_configs"] = extra
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)
    if world > 1:
        tq.set_workspace(None)
        dist.destroy_process_group()
    return 0


def launch_replicas(argv, n):
    """`--gpus N` run directly (no launcher): start N ranks, one process per GPU on
    this node, through torch.distributed.run, and return its exit code."""
    import random
    import subprocess
    port = 20000 + random.randrange(20000)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__)] + list(argv)
    return subprocess.run(cmd, timeout=3600).returncode


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_replicas(argv, args.gpus)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    raise SystemExit(main())
