"""Seeded synthetic workloads (inputs only; none of the method's arithmetic).

Shared by the tests, the bench and the smoke check: both the CUDA path and the
CPU oracle consume exactly these tensors.  Every draw comes from one seeded
``torch.Generator`` on the CPU, in a fixed order:

  1. per-(KV head, channel) key scales sigma = exp(0.5 * N(0,1)) (log-normal(0, 0.5)),
     when the workload asks for them, then for each KV head a seeded
     ``randperm(D)[:n_outliers]`` of outlier channels whose sigma is multiplied by
     ``outlier_factor``;
  2. sequence lengths (uniform integers when a range is given);
  3. a random permutation of the block pool (identity when asked), split into
     contiguous runs, one per sequence, in order;
  4. K = N(0,1) * sigma and V = N(0,1), token by token in sequence order, drawn
     in fp32 and rounded to the storage dtype;
  5. q = N(0,1) [B, H_q, D].

The shapes follow the model layers the pages name (Qwen2.5-0.5B/7B, Llama-3-8B);
no model weights or datasets are involved.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

BLOCK_SIZE = 16


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    head_dim: int
    num_q_heads: int
    num_kv_heads: int
    batch: int
    k_bits: int
    v_bits: int
    dtype: str                       # "float32" or "bfloat16"
    seq_len: int = 0                 # every sequence has this length ...
    seq_len_range: Optional[tuple] = None   # ... or lengths uniform in [lo, hi]
    channel_scales: bool = True
    n_outliers: int = 0
    outlier_factor: float = 1.0
    identity_blocks: bool = False
    seed: int = 0
    sign_seed: int = 0
    step: str = "fill"               # "fill" | "append_last" | "prefill_tail"
    tail_tokens: int = 0             # tokens appended by the step for "prefill_tail"

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.head_dim))

    def scaled(self, **kw) -> "WorkloadSpec":
        return replace(self, **kw)


CONFIGS = {
    0: WorkloadSpec("tiny-d128-k4v4", 128, 1, 1, 1, 4, 4, "float32", seq_len=256,
                    channel_scales=False, identity_blocks=True, seed=0),
    1: WorkloadSpec("qwen2.5-0.5b-layer-k8v8", 64, 14, 2, 8, 8, 8, "bfloat16", seq_len=4096,
                    n_outliers=4, outlier_factor=10.0, seed=1001),
    2: WorkloadSpec("llama3-8b-layer-k4v4", 128, 32, 8, 32, 4, 4, "bfloat16", seq_len=8192,
                    n_outliers=2, outlier_factor=20.0, seed=1002),
    3: WorkloadSpec("qwen2.5-7b-layer-k4v2", 128, 28, 4, 64, 4, 2, "bfloat16",
                    seq_len_range=(1024, 32768), n_outliers=2, outlier_factor=20.0, seed=1003,
                    step="append_last"),
    4: WorkloadSpec("llama3-8b-long-k3v2", 128, 32, 8, 1, 3, 2, "bfloat16", seq_len=131072,
                    n_outliers=2, outlier_factor=20.0, seed=1004, step="prefill_tail",
                    tail_tokens=16384),
}


@dataclass
class Workload:
    spec: WorkloadSpec
    seq_lens: np.ndarray            # int32 [B]
    block_table: np.ndarray         # int32 [B, max_blocks] (-1 past each sequence)
    num_blocks: int
    k: torch.Tensor                 # [T_total, H_kv, D] (tokens of seq 0, then seq 1, ...)
    v: torch.Tensor
    q: torch.Tensor                 # [B, H_q, D]
    token_seq: np.ndarray           # int32 [T_total]: sequence of each token
    token_pos: np.ndarray           # int32 [T_total]: position inside its sequence
    slot_mapping: np.ndarray        # int64 [T_total]
    step_tokens: np.ndarray         # int64 indices of the tokens the timed step appends
    setup_tokens: np.ndarray        # int64 indices appended before timing
    sigma: torch.Tensor = field(default=None)

    @property
    def slot_bytes(self) -> int:
        d = self.spec.head_dim
        return (d * self.spec.k_bits + 7) // 8 + 4 + (d * self.spec.v_bits + 7) // 8 + 4

    @property
    def torch_dtype(self):
        return torch.float32 if self.spec.dtype == "float32" else torch.bfloat16


def generate(spec: WorkloadSpec, chunk_tokens: int = 1 << 16) -> Workload:
    g = torch.Generator().manual_seed(spec.seed)
    d, h_kv, bsz = spec.head_dim, spec.num_kv_heads, spec.batch
    if spec.channel_scales:
        sigma = torch.exp(0.5 * torch.randn(h_kv, d, generator=g))
        for h in range(h_kv):
            if spec.n_outliers:
                ch = torch.randperm(d, generator=g)[:spec.n_outliers]
                sigma[h, ch] *= spec.outlier_factor
    else:
        sigma = torch.ones(h_kv, d)
    if spec.seq_len_range is not None:
        lo, hi = spec.seq_len_range
        lens = torch.randint(lo, hi + 1, (bsz,), generator=g).numpy().astype(np.int32)
    else:
        lens = np.full(bsz, spec.seq_len, dtype=np.int32)
    nblk = (lens.astype(np.int64) + BLOCK_SIZE - 1) // BLOCK_SIZE
    pool = max(1, int(nblk.sum()))
    order = np.arange(pool) if spec.identity_blocks else torch.randperm(pool, generator=g).numpy()
    max_blocks = max(1, int(nblk.max()) if bsz else 1)
    bt = np.full((bsz, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(bsz):
        bt[b, :nblk[b]] = order[off:off + nblk[b]]
        off += int(nblk[b])
    total = int(lens.astype(np.int64).sum())
    dt = torch.float32 if spec.dtype == "float32" else torch.bfloat16
    k = torch.empty(total, h_kv, d, dtype=dt)
    v = torch.empty(total, h_kv, d, dtype=dt)
    for s in range(0, total, chunk_tokens):
        n = min(chunk_tokens, total - s)
        k[s:s + n] = (torch.randn(n, h_kv, d, generator=g) * sigma).to(dt)
        v[s:s + n] = torch.randn(n, h_kv, d, generator=g).to(dt)
    q = torch.randn(bsz, spec.num_q_heads, d, generator=g).to(dt)
    token_seq = np.repeat(np.arange(bsz, dtype=np.int32), lens)
    starts = np.concatenate([[0], np.cumsum(lens.astype(np.int64))[:-1]]) if bsz else np.zeros(0)
    token_pos = (np.arange(total, dtype=np.int64) - np.repeat(starts, lens)).astype(np.int32)
    slot = bt[token_seq, token_pos // BLOCK_SIZE].astype(np.int64) * BLOCK_SIZE + token_pos % BLOCK_SIZE
    if spec.step == "fill":
        step_mask = np.ones(total, dtype=bool)
    elif spec.step == "append_last":
        step_mask = token_pos == lens[token_seq] - 1
    elif spec.step == "prefill_tail":
        step_mask = token_pos >= lens[token_seq] - spec.tail_tokens
    else:
        raise ValueError(spec.step)
    return Workload(spec=spec, seq_lens=lens, block_table=bt, num_blocks=pool, k=k, v=v, q=q,
                    token_seq=token_seq, token_pos=token_pos, slot_mapping=slot,
                    step_tokens=np.nonzero(step_mask)[0], setup_tokens=np.nonzero(~step_mask)[0],
                    sigma=sigma)


def empty_pages(wl: Workload, device="cpu", fill: int = 0, slot_stride: Optional[int] = None):
    """Zeroed (or ``fill``-ed) page pool [num_blocks, 16, H_kv, slot_stride] uint8."""
    stride = slot_stride or wl.slot_bytes
    return torch.full((wl.num_blocks, BLOCK_SIZE, wl.spec.num_kv_heads, stride), fill,
                      dtype=torch.uint8, device=device)
