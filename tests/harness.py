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


# A selection decided by a near tie (gap <= GAP_MIN) has several correct
# answers once the scores carry rounding error: such a list is checked for
# validity instead of equality.  TIE_TOL bounds how far (relative) a chosen
# block's oracle score may sit below an unchosen candidate's: the two scores
# each carry at most S_RTOL of relative error on the GPU side.
TIE_TOL = 2 * S_RTOL


def check_list_valid(lst, S_or: np.ndarray, t: int, p: O.Params, tol: float = TIE_TOL) -> None:
    """Assert that `lst` (one row's block list from the GPU) is a correct
    selection for the oracle's scores S_or of row t up to score error `tol`:
    ascending distinct blocks in [0, b_t], then -1 padding; the init blocks
    and the local run present; min(|I|, b_t + 1) entries; and no unchosen
    candidate scoring above a chosen one by more than tol (relative)."""
    lst = np.asarray(lst, dtype=np.int64)
    b_t = t // p.block
    valid = lst[lst >= 0]
    n = len(valid)
    assert (lst[n:] == -1).all() and (lst[:n] >= 0).all(), lst
    assert n == min(p.n_sel, b_t + 1), (n, b_t)
    assert (np.diff(valid) > 0).all() and valid[-1] <= b_t, lst
    init = set(range(min(p.n_init, b_t + 1)))
    local = set(range(max(0, b_t - p.n_local + 1), b_t + 1))
    chosen = set(valid.tolist())
    assert init <= chosen and local <= chosen, lst
    cand = [b for b in range(b_t + 1) if b not in init and b not in local]
    picked = [b for b in cand if b in chosen]
    assert len(picked) == min(p.top_k, len(cand))
    rest = [b for b in cand if b not in chosen]
    if picked and rest:
        bs = O.block_scores(S_or, t, p)
        lo = min(bs[b] for b in picked)
        hi = max(bs[b] for b in rest)
        assert lo >= hi * (1.0 - tol), (lo, hi)


def compare_lists(gpu_lists, S_rows, ts, p: O.Params):
    """Compare GPU block lists with the oracle's selection row by row:
    bit-exact where the oracle's top-k gap exceeds GAP_MIN, valid (see
    check_list_valid) elsewhere.  Returns (rows compared exactly, rows checked
    for validity, rows that differ where they must not)."""
    exact = tie = bad = 0
    for lst, S_or, t in zip(gpu_lists, S_rows, ts):
        sel = O.select_blocks(S_or, int(t), p)
        if O.topk_gap(S_or, int(t), p) > GAP_MIN:
            exact += 1
            bad += int(not np.array_equal(np.asarray(lst), sel))
        else:
            tie += 1
            check_list_valid(lst, S_or, int(t), p)
    return exact, tie, bad


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
