"""Seeded synthetic inputs for the InfLLM-V2 sparse-attention path.

This module is shared by the tests, the benchmark and the oracle-side checks.
It only draws random numbers and packs them into tensors: it contains none of
the method's arithmetic (no pooling, scoring, selection or attention).

Workloads (sizes follow the InfLLM-V2 paper's GQA backbone, h_q=32, h_kv=2,
d=128, block B=64, |I|=96 selected blocks):

* ``tiny_1k``      n=1024, h_q=4, h_kv=1, d=64, |I|=5 (1 init + 2 local + 2 top-k),
                   Q,K,V ~ N(0,1), fp32 output.
* ``prefill_32k``  n=32768, h_q=32, h_kv=2, d=128, |I|=96.
* ``prefill_128k`` n=131072, same heads.
* ``decode_16x128k`` 16 sequences with a 131072-token prefix, one new token
                   per sequence per step.
* ``varlen_128k``  packed batch of 131072 tokens, lengths drawn from four
                   equally likely bands (0-4K, 4-12K, 12-24K, 24-32K).

For every workload except ``tiny_1k`` the keys carry a per-64-token-block
offset: K = N(0,1) + mu_b with mu_b ~ N(0, 0.5^2 I_d) drawn per
(sequence, kv head, block).  Q and V are N(0,1).  All draws use numpy's PCG64
in float32 and are rounded to bf16 (round to nearest even) by torch.
Draw order: Q, K noise, mu, V.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    h_q: int
    h_kv: int
    d: int
    n_init: int
    n_local: int
    top_k: int
    block_offset_std: float      # std of the per-block key offset mu_b (0: none)
    out_fp32: bool
    seqlen: int = 0               # prefill length (single sequence)
    batch: int = 1
    varlen_total: int = 0         # packed total for the varlen workload
    decode_steps: int = 0
    seed: int = 0

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def n_sel(self) -> int:
        return self.n_init + self.n_local + self.top_k


WORKLOADS: Dict[str, Workload] = {
    "tiny_1k": Workload("tiny_1k", 4, 1, 64, 1, 2, 2, 0.0, True, seqlen=1024, seed=1000),
    "prefill_32k": Workload("prefill_32k", 32, 2, 128, 1, 32, 63, 0.5, False, seqlen=32768, seed=1001),
    "prefill_128k": Workload("prefill_128k", 32, 2, 128, 1, 32, 63, 0.5, False, seqlen=131072, seed=1002),
    "decode_16x128k": Workload("decode_16x128k", 32, 2, 128, 1, 32, 63, 0.5, False, seqlen=131072,
                               batch=16, decode_steps=64, seed=1003),
    "varlen_128k": Workload("varlen_128k", 32, 2, 128, 1, 32, 63, 0.5, False, varlen_total=131072,
                            seed=1004),
}

# Sequence-length bands of the mixed-length fine-tuning data (0-4K, 4-12K,
# 12-24K, 24-32K); lengths are uniform inside a band.
LENGTH_BANDS = ((1, 4096), (4097, 12288), (12289, 24576), (24577, 32768))
DENSE_THRESHOLD = 8192
BLOCK = 64


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """float32 numpy array -> bf16 torch tensor (single RNE rounding)."""
    assert x.dtype == np.float32
    return torch.from_numpy(x).to(torch.bfloat16)


def varlen_lengths(total: int, seed: int) -> List[int]:
    """Lengths for the packed varlen batch: pick a band uniformly, then a
    length uniformly inside it, until the total is reached; the last length is
    cut so the lengths sum to exactly ``total``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens: List[int] = []
    acc = 0
    while acc < total:
        lo, hi = LENGTH_BANDS[int(rng.integers(0, len(LENGTH_BANDS)))]
        ln = int(rng.integers(lo, hi + 1))
        ln = min(ln, total - acc)
        lens.append(ln)
        acc += ln
    return lens


def _keys(rng: np.random.Generator, lens: List[int], h_kv: int, d: int, mu_std: float) -> np.ndarray:
    total = sum(lens)
    k = rng.standard_normal((total, h_kv, d), dtype=np.float32)
    if mu_std > 0.0:
        nblk = [(ln + BLOCK - 1) // BLOCK for ln in lens]
        mu = rng.standard_normal((sum(nblk), h_kv, d), dtype=np.float32) * np.float32(mu_std)
        row = 0
        b0 = 0
        for ln, nb in zip(lens, nblk):
            idx = np.arange(ln) // BLOCK + b0
            k[row:row + ln] += mu[idx]
            row += ln
            b0 += nb
    return k


def make_prefill(w: Workload, lens: Optional[List[int]] = None, seed: Optional[int] = None) -> dict:
    """Packed prefill inputs: Q [total,h_q,d], K/V [total,h_kv,d] bf16 (CPU),
    cu_seqlens int32 [batch+1]."""
    if lens is None:
        lens = varlen_lengths(w.varlen_total, w.seed) if w.varlen_total else [w.seqlen] * w.batch
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    total = sum(lens)
    q = rng.standard_normal((total, w.h_q, w.d), dtype=np.float32)
    Q = to_bf16(q)
    del q
    K = to_bf16(_keys(rng, lens, w.h_kv, w.d, w.block_offset_std))
    V = to_bf16(rng.standard_normal((total, w.h_kv, w.d), dtype=np.float32))
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    return {"Q": Q, "K": K, "V": V, "cu_seqlens": torch.from_numpy(cu), "lens": list(lens)}


def make_decode(w: Workload, prefix: Optional[int] = None, steps: Optional[int] = None,
                batch: Optional[int] = None) -> dict:
    """Decode inputs: a per-sequence prefix of ``prefix`` tokens plus ``steps``
    new tokens per sequence.  K/V hold prefix+steps rows per sequence
    ([batch, prefix+steps, h_kv, d]); rows past the prefix are the tokens the
    decode steps append, one per step.  q_steps is [steps, batch, h_q, d].
    The block offset of a new token continues the block structure (a fresh
    offset starts with every new 64-token block).  Sequence s uses its own
    seed (draw order: step queries, K noise, mu, V), so one sequence can be
    regenerated alone."""
    prefix = w.seqlen if prefix is None else prefix
    steps = w.decode_steps if steps is None else steps
    batch = w.batch if batch is None else batch
    Ks, Vs, Qs = [], [], []
    for s in range(batch):
        one = make_decode_sequence(w, s, prefix, steps)
        Qs.append(one["q_steps"])
        Ks.append(one["K"])
        Vs.append(one["V"])
    return {
        "K": torch.stack(Ks),                       # [batch, n, h_kv, d]
        "V": torch.stack(Vs),
        "q_steps": torch.stack(Qs, dim=1),          # [steps, batch, h_q, d]
        "prefix": prefix,
        "steps": steps,
    }


def make_decode_sequence(w: Workload, s: int, prefix: int, steps: int) -> dict:
    """One sequence of :func:`make_decode` (same values), without the others."""
    n = prefix + steps
    rng = np.random.Generator(np.random.PCG64(w.seed * 100 + s))
    # only the decoded tokens need queries (the prefix's queries are never used)
    Q = to_bf16(rng.standard_normal((steps, w.h_q, w.d), dtype=np.float32))
    K = to_bf16(_keys(rng, [n], w.h_kv, w.d, w.block_offset_std))
    V = to_bf16(rng.standard_normal((n, w.h_kv, w.d), dtype=np.float32))
    return {"K": K, "V": V, "q_steps": Q}


def sample_rows(total: int, count: int, seed: int) -> np.ndarray:
    """Uniform sample of row indices in [0, total), sorted, without repeats."""
    rng = np.random.Generator(np.random.PCG64(seed))
    count = min(count, total)
    return np.sort(rng.choice(total, size=count, replace=False))


def make_grad_out(total: int, h_q: int, d: int, seed: int) -> torch.Tensor:
    """A seeded upstream gradient dO [total, h_q, d] ~ N(0,1), bf16 (the
    backward's input; random draws only)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return to_bf16(rng.standard_normal((total, h_q, d), dtype=np.float32))
