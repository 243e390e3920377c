"""Write the fp32 Lloyd-Max codebook tables that both paths consume.

TEST INFRASTRUCTURE / OFFLINE TOOL: calls only ``oracle.tq_oracle``.  The
tables it writes are data files of the library (the fitted codebooks are built
once and shared, [turboquant_serve, "Codebook sharing"]); the library reads
them as bytes and never runs this script.

File format (little endian), one file per (D, bits):
    char[4]  magic "TQCB"
    u32      version (1)
    u32      D
    u32      bits
    u32      density id (0 = Beta-sphere, 1 = Gaussian approximation N(0, 1/D))
    u32      n_iter (iteration budget of Lloyd's iteration)
    u32      iterations actually run (< n_iter when a fixed point was reached)
    u32      reserved (0)
    f32[L]   centroids, ascending
    f32[L-1] boundaries, ascending

Usage: python -m oracle.gen_codebooks [--out DIR] [--jobs N]
"""

from __future__ import annotations

import argparse
import multiprocessing as mp
import os
import struct
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle import tq_oracle as O  # noqa: E402

MAGIC = b"TQCB"
VERSION = 1
N_ITER = 300_000
DIMS = (64, 128, 256)
BITS = (1, 2, 3, 4, 5, 6, 7, 8)
DEFAULT_OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "kv_cache_vector_append_b200", "codebooks")


KINDS = ("beta", "gauss")


def table_filename(dim: int, bits: int, kind: str = "beta") -> str:
    """beta_d<D>_b<bits>.tqcb: exact Beta-sphere density; gauss_d<D>_b<bits>.tqcb: its
    Gaussian approximation N(0, 1/D)."""
    if kind not in KINDS:
        raise ValueError(kind)
    return f"{kind}_d{dim}_b{bits}.tqcb"


def write_table(path: str, t: O.CodebookTable) -> None:
    with open(path, "wb") as f:
        f.write(MAGIC)
        f.write(struct.pack("<7I", VERSION, t.dim, t.bits, t.density_id, t.n_iter,
                            t.iterations_run, 0))
        f.write(np.asarray(t.centroids, dtype="<f4").tobytes())
        f.write(np.asarray(t.boundaries, dtype="<f4").tobytes())


def read_table(path: str) -> O.CodebookTable:
    """Oracle-side reader of a table file (independent of the library's reader)."""
    with open(path, "rb") as f:
        raw = f.read()
    if raw[:4] != MAGIC:
        raise ValueError(f"{path}: bad magic")
    version, dim, bits, dens, n_iter, iters, _ = struct.unpack_from("<7I", raw, 4)
    if version != VERSION:
        raise ValueError(f"{path}: unsupported version {version}")
    levels = 1 << bits
    off = 4 + 7 * 4
    c = np.frombuffer(raw, dtype="<f4", count=levels, offset=off).astype(np.float32)
    b = np.frombuffer(raw, dtype="<f4", count=levels - 1, offset=off + 4 * levels)
    return O.CodebookTable(dim=dim, bits=bits, density_id=dens, n_iter=n_iter,
                           iterations_run=iters, centroids=c, boundaries=b.astype(np.float32))


def build_table(dim: int, bits: int, n_iter: int = N_ITER, kind: str = "beta") -> O.CodebookTable:
    if kind == "beta":
        cb = O.lloyd_max_beta(dim, bits, n_iter)
        return O.to_fp32_table(cb, dim, bits, O.BetaSphereDensity.density_id)
    cb = O.lloyd_max_gaussian_dim(dim, bits, n_iter)
    return O.to_fp32_table(cb, dim, bits, O.GaussianDensity.density_id)


def _job(args):
    dim, bits, out, kind = args
    t = build_table(dim, bits, kind=kind)
    write_table(os.path.join(out, table_filename(dim, bits, kind)), t)
    return dim, bits, kind, t.iterations_run


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--out", default=DEFAULT_OUT)
    ap.add_argument("--jobs", type=int, default=os.cpu_count() or 1)
    ap.add_argument("--kind", choices=KINDS + ("all",), default="all")
    args = ap.parse_args(argv)
    os.makedirs(args.out, exist_ok=True)
    kinds = KINDS if args.kind == "all" else (args.kind,)
    jobs = [(d, b, args.out, k) for k in kinds for b in sorted(BITS, reverse=True) for d in DIMS]
    ctx = mp.get_context("spawn")
    with ctx.Pool(args.jobs) as pool:
        for dim, bits, kind, iters in pool.imap_unordered(_job, jobs):
            print(f"{kind:5s} D={dim:4d} bits={bits}: {iters} iterations")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
