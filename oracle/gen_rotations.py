"""Write the dense rotation tables that both paths consume.

TEST INFRASTRUCTURE / OFFLINE TOOL: calls only ``oracle.tq_oracle``.  The tables
are data files of the library ("a fixed random orthogonal matrix, seeded by
head_dim", turboquant_serve 0.1.2, "Rotation"); the library reads them as bytes and
never runs this script.

File format (little endian), one file per head dimension D (seed = D):
    char[4]   magic "TQRT"
    u32       version (1)
    u32       D
    u32       seed of the Gaussian draw (numpy PCG64)
    u16[D*D]  hi = bf16(H), row-major (H the float64 Haar matrix)
    u16[D*D]  lo = bf16(H - hi), row-major
The rotation is R = hi + lo (exact in float32).

Usage: python -m oracle.gen_rotations [--out DIR]
"""

from __future__ import annotations

import argparse
import os
import struct
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle import tq_oracle as O  # noqa: E402

MAGIC = b"TQRT"
VERSION = 1
DIMS = (64, 128, 256)
DEFAULT_OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "kv_cache_vector_append_b200", "rotations")


def table_filename(dim: int) -> str:
    return f"qr_d{dim}.tqrt"


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns of values already on the bf16 grid."""
    b = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype("<u2")


def write_table(path: str, rot: O.DenseRotation) -> None:
    with open(path, "wb") as f:
        f.write(MAGIC)
        f.write(struct.pack("<3I", VERSION, rot.dim, rot.seed))
        f.write(_bf16_bits(rot.hi).tobytes())
        f.write(_bf16_bits(rot.lo).tobytes())


def read_table(path: str):
    """(dim, seed, hi, lo) with hi, lo float64 [D, D] (oracle-side reader)."""
    with open(path, "rb") as f:
        raw = f.read()
    if raw[:4] != MAGIC:
        raise ValueError(f"{path}: bad magic")
    version, dim, seed = struct.unpack_from("<3I", raw, 4)
    if version != VERSION:
        raise ValueError(f"{path}: unsupported version {version}")
    n = dim * dim
    words = np.frombuffer(raw, dtype="<u2", count=2 * n, offset=16).astype(np.uint32) << 16
    vals = words.view(np.float32).astype(np.float64)
    return dim, seed, vals[:n].reshape(dim, dim), vals[n:].reshape(dim, dim)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--out", default=DEFAULT_OUT)
    args = ap.parse_args(argv)
    os.makedirs(args.out, exist_ok=True)
    for d in DIMS:
        write_table(os.path.join(args.out, table_filename(d)), O.dense_rotation(d, d))
        print(f"D={d}: {table_filename(d)}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
