"""Helpers shared by the GPU parity tests (CUDA path vs the CPU oracle)."""
import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from oracle import gen_codebooks as G
import os


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_vector_append_b200 as tq  # noqa: F401  (fails loudly if the library is missing)


def oracle_table(dim, bits, kind="beta"):
    return G.read_table(os.path.join(G.DEFAULT_OUT, G.table_filename(dim, bits, kind)))


def to_np_f64(t):
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def gpu_append(tq, wl, tokens=None, pages=None, slot_stride=None, fill=0, slot_mapping=None,
               kind="beta"):
    """Run tq_quantize_append for `tokens` (indices into the workload) on cuda:0."""
    from kv_cache_vector_append_b200 import workloads as W
    dev = "cuda"
    if pages is None:
        pages = W.empty_pages(wl, device=dev, fill=fill, slot_stride=slot_stride)
    idx = np.arange(wl.k.shape[0]) if tokens is None else np.asarray(tokens)
    it = torch.from_numpy(idx.astype(np.int64))
    k = wl.k[it].to(dev)
    v = wl.v[it].to(dev)
    sm = wl.slot_mapping[idx] if slot_mapping is None else slot_mapping
    sm = torch.from_numpy(np.ascontiguousarray(sm, dtype=np.int64)).to(dev)
    cb = tq.load_codebooks(wl.spec.head_dim, wl.spec.k_bits, wl.spec.v_bits, dev, kind)
    tq.quantize_append(pages, sm, k, v, cb, wl.spec.sign_seed)
    torch.cuda.synchronize()
    return pages, cb


def gpu_decode(tq, wl, pages, cb, out_dtype=None):
    dev = "cuda"
    q = wl.q.to(dev)
    out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=dev)
    bt = torch.from_numpy(wl.block_table).to(dev)
    sl = torch.from_numpy(wl.seq_lens).to(dev)
    tq.paged_decode(out, q, pages, bt, sl, cb, wl.spec.sign_seed, wl.spec.scale)
    torch.cuda.synchronize()
    return out


def decode_error(o_gpu, o_ref):
    """max over (b, h) of ||o_gpu - o_ref||_inf / ||o_ref||_2 (0/0 -> 0)."""
    diff = np.max(np.abs(o_gpu - o_ref), axis=-1)
    nrm = np.linalg.norm(o_ref, axis=-1)
    rel = np.where(nrm > 0, diff / np.where(nrm > 0, nrm, 1), diff)
    return float(np.max(rel)) if rel.size else 0.0
