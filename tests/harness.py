"""Shared helpers for the GPU parity tests: run the CUDA path through the
C ABI, and run the oracle on the same seeded inputs.  The two sides share
only the inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import infllm2_oracle as O
import trainable_block_sparse_pool_b200 as T

# Tolerances (bf16 inputs, fp32 accumulation): selected blocks bit-exact where
# the k-th and (k+1)-th candidate scores differ by more than 1e-4 relative;
# S_shared within 1e-4 relative on visible entries; attention outputs within
# 2e-2 max-abs and 2e-3 mean-abs.
S_RTOL = 1e-4
GAP_MIN = 1e-4
ATT_MAX_ABS = 2e-2
ATT_MEAN_ABS = 2e-3


def oracle_params(w) -> O.Params:
    return O.Params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k)


def lib_params(w) -> "T.Params":
    return T.default_params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k)


class DeviceRun:
    """Device buffers and the CUDA path's steps for one packed batch."""

    def __init__(self, data: dict, w, keep_scores: bool = True):
        self.w = w
        self.p = lib_params(w)
        self.lens = list(data["lens"])
        dev = torch.device("cuda")
        self.Q = data["Q"].to(dev)
        self.K = data["K"].to(dev)
        self.V = data["V"].to(dev)
        self.cu = data["cu_seqlens"].to(dev)
        self.vl = T.make_varlen(self.lens, self.cu, self.p)
        d = w.d
        self.Kc1 = torch.empty(w.h_kv, max(1, self.vl.total_c1), d, dtype=torch.bfloat16, device=dev)
        self.Kc2 = torch.empty(w.h_kv, max(1, self.vl.total_c2), d, dtype=torch.bfloat16, device=dev)
        self.ld = T.infllm2_scores_ld(self.vl, self.p)
        self.S = torch.zeros(w.h_kv, self.vl.total, self.ld, dtype=torch.float32, device=dev)
        self.idx = torch.empty(w.h_kv, self.vl.total, self.p.n_sel, dtype=torch.int32, device=dev)
        self.out = torch.empty(self.vl.total, w.h_q, d,
                               dtype=torch.float32 if w.out_fp32 else torch.bfloat16, device=dev)
        self.sws = torch.empty(max(256, T.infllm2_sparse_workspace_bytes(self.vl, w.h_q)), dtype=torch.uint8,
                               device=dev)

    def compress(self):
        T.infllm2_compress_k(self.K, self.vl, self.Kc1, self.Kc2, self.p)

    def scores(self):
        T.infllm2_shared_scores(self.Q, self.Kc1, self.Kc2, self.vl, self.w.h_kv, self.S, self.ld, self.p)

    def topk(self, S=None):
        T.infllm2_topk_blocks(self.S if S is None else S, self.ld, self.vl, self.w.h_kv, self.idx, self.p)

    def sparse(self, idx=None):
        T.infllm2_sparse_attn(self.Q, self.K, self.V, self.idx if idx is None else idx, self.vl, self.out, self.p,
                              workspace=self.sws)

    def dense(self):
        T.infllm2_dense_attn(self.Q, self.K, self.V, self.vl, self.out, self.p)

    def c1_offsets(self):
        o = [0]
        for n in self.lens:
            o.append(o[-1] + O.window_count(n, 32, 16))
        return o

    def c2_offsets(self):
        o = [0]
        for n in self.lens:
            o.append(o[-1] + O.window_count(n, 128, 64))
        return o


def oracle_sequences(data: dict, w, which=None, p=None):
    """fp64 oracle sequence objects (pooled keys included) for the sequences
    listed in `which` (all by default)."""
    p = oracle_params(w) if p is None else p
    cu = data["cu_seqlens"].tolist()
    seqs = {}
    for s in (range(len(data["lens"])) if which is None else which):
        a, b = cu[s], cu[s + 1]
        seqs[s] = O.Sequence1(O.to_f64(data["Q"][a:b]), O.to_f64(data["K"][a:b]), O.to_f64(data["V"][a:b]), p)
    return seqs


def default_index_rows(lens, w) -> np.ndarray:
    """A valid block list for every row (init + local + the lowest
    candidates): the selection a row gets when all its block scores tie.
    Used to fill rows whose attention output is not compared."""
    n_sel = w.n_sel
    rows = []
    for n in lens:
        t = np.arange(n)
        b_t = t // 64
        out = np.full((n, n_sel), -1, dtype=np.int32)
        for i in range(n):
            bt = int(b_t[i])
            if bt + 1 <= n_sel:
                out[i, :bt + 1] = np.arange(bt + 1)
            else:
                init = list(range(w.n_init))
                local = list(range(bt - w.n_local + 1, bt + 1))
                cand = list(range(w.n_init, w.n_init + w.top_k))
                out[i] = init + cand + local
        rows.append(out)
    return np.concatenate(rows, axis=0)


def seq_of_rows(lens, rows):
    cu = np.concatenate([[0], np.cumsum(lens)])
    s = np.searchsorted(cu, rows, side="right") - 1
    return s, rows - cu[s]
