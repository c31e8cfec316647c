"""Plain fp64 CPU oracle of the InfLLM-V2 sparse-attention forward path (GQA).

TEST INFRASTRUCTURE ONLY.  This module is imported by ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``, nowhere else.  The product path (the CUDA library and its
binding) never calls it and shares no code with it.

It follows the method as described on these pages (cited by title + section):

* [blog]    "论文阅读：InfLLM-V2 — 把可训练稀疏注意力做成全注意力的'受限版本'"
            (xiaohongrsx.github.io paper-reading notes)
* [news]    "从密集到稀疏：InfLLM-V2 如何实现零参数开销的长文本高效处理" (dtcms.com)
* [top168]  top168.com article on InfLLM-V2 (Tsinghua / OpenBMB,
            arXiv 2509.24663), sections 三 (three-stage compression),
            四 (efficient implementation), 七 (implementation details)

Every formula on those pages was lost when they were extracted, so each step
below states the reading it takes.  Values are fp64; bf16 inputs convert to
fp64 exactly.  Pooled keys are rounded to bf16 (round to nearest even) because
the scoring contraction consumes them as bf16 operands.

Notation: n tokens in one sequence, h_q query heads, h_kv key/value heads,
G = h_q / h_kv, query head h belongs to kv group g = h // G, block size B=64,
stage-1 windows (l_C1=32, s_C1=16), coarse windows (l_C2=128, s_C2=64),
max-pool (kernel 5, stride 4, padding 1), |I| = n_init + n_local + top_k.

Parity status: every function below is pinned by ``tests/test_oracle.py``
(closed forms, invariants, brute force, a library routine, and the worked
example of the [blog] section "先看一个具体例子"); the attention backward by
central finite differences and, with every causal block selected, by fp64
autograd of dense causal attention.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# parameters
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Params:
    """Method parameters.  Defaults are the values the pages give:
    B=64 ([blog] "先看一个具体例子": 64 tokens per block), l_C1=B/2, s_C1=B/4,
    max-pool l=5 s=4 ([top168] §三), l_C2=4*l_C1, s_C2=4*s_C1 ([top168] §四),
    96 visible blocks = 1 init + 32 local + 63 top-k ([blog] worked example)."""
    block: int = 64
    c1_len: int = 32
    c1_stride: int = 16
    c2_len: int = 128
    c2_stride: int = 64
    pool_len: int = 5
    pool_stride: int = 4
    pool_pad: int = 1
    n_init: int = 1
    n_local: int = 32
    top_k: int = 63
    lse_mode: str = "approx"      # "approx": LSE from the coarse C2 scores; "exact": from C1
    scale: Optional[float] = None  # None: 1/sqrt(d)

    @property
    def n_sel(self) -> int:
        return self.n_init + self.n_local + self.top_k

    def softmax_scale(self, d: int) -> float:
        return (1.0 / math.sqrt(d)) if self.scale is None else float(self.scale)


# ----------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even)
# ----------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as
    fp64.  bf16 keeps 8 significant bits; its smallest normal is 2^-126 and
    its subnormal spacing is 2^-133."""
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x) & (x != 0.0)
    m, e = np.frexp(x[fin])                   # x = m * 2^e, 0.5 <= |m| < 1
    ulp_exp = np.maximum(e - 8, -133)         # weight of the last kept bit
    r = np.ldexp(np.rint(np.ldexp(x[fin], -ulp_exp)), ulp_exp)   # rint: ties to even
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    r = np.where(np.abs(r) > bf16_max, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


# ----------------------------------------------------------------------------
# step 1: stage-1 (and coarse) mean pooling of K   ([top168] §三, §四)
# ----------------------------------------------------------------------------
def window_count(n: int, length: int, stride: int) -> int:
    """Number of complete pooling windows [s*j, s*j+l-1] inside n tokens.
    Reading: partial windows at the end are dropped (no padding)."""
    return 0 if n < length else (n - length) // stride + 1


def pool_keys(K: np.ndarray, length: int, stride: int) -> np.ndarray:
    """Mean-pool the keys of one sequence over windows of ``length`` tokens
    taken every ``stride`` tokens ([top168] §三, first stage: mean pooling over
    consecutive key blocks with l_C1, s_C1; §四 the coarse C2 pooling uses the
    same operation with l_C2, s_C2 on the raw keys).

    K: [n, h_kv, d] fp64 (bf16-exact).  Returns [h_kv, count, d]: the exact
    mean of each window, rounded to bf16."""
    n, h_kv, d = K.shape
    cnt = window_count(n, length, stride)
    out = np.zeros((h_kv, cnt, d), dtype=np.float64)
    for j in range(cnt):
        win = K[j * stride: j * stride + length]           # [length, h_kv, d]
        out[:, j, :] = win.sum(axis=0) / length
    return bf16_round(out)


def visible_windows(t: int, length: int, stride: int) -> int:
    """How many pooled windows a query at position t may see.  Reading: a
    window is visible only when all of its tokens are at or before t
    (window j is visible iff stride*j + length - 1 <= t), so no future token
    leaks into a score."""
    if t < length - 1:
        return 0
    return (t - (length - 1)) // stride + 1


# ----------------------------------------------------------------------------
# step 2: compressed scores with the LSE approximation and the group sum
# ----------------------------------------------------------------------------
def _logsumexp(x: np.ndarray) -> float:
    if x.size == 0:
        return -math.inf
    m = float(np.max(x))
    return m + math.log(float(np.sum(np.exp(x - m))))


def group_lse(q_g: np.ndarray, Kc1_g: np.ndarray, Kc2_g: np.ndarray, t: int,
              p: Params, scale: float) -> np.ndarray:
    """Per-head softmax normaliser (log-sum-exp) of the stage-1 scores of one
    query token.

    [top168] §四: the per-head softmax must be normalised before the head-group
    sum, and the exact normaliser needs a second pass; the approximation takes
    it from the coarser scores S_C2 (l_C2 = 4 l_C1, s_C2 = 4 s_C1).
    Readings: no correction for the C2 scores having fewer terms (a constant
    per (head, token) shifts all of that row's scores alike); when no C2
    window is visible yet (t < l_C2 - 1) the exact log-sum-exp over the C1
    windows is used; when neither is visible the row is empty (-inf).

    q_g: [G, d] queries of the group's heads.  Returns [G]."""
    G = q_g.shape[0]
    n1 = visible_windows(t, p.c1_len, p.c1_stride)
    n2 = visible_windows(t, p.c2_len, p.c2_stride)
    out = np.empty(G, dtype=np.float64)
    for h in range(G):
        if p.lse_mode == "approx" and n2 > 0:
            s2 = (Kc2_g[:n2] @ q_g[h]) * scale
            out[h] = _logsumexp(s2)
        else:
            s1 = (Kc1_g[:n1] @ q_g[h]) * scale
            out[h] = _logsumexp(s1)
    return out


def shared_scores(q_g: np.ndarray, Kc1_g: np.ndarray, Kc2_g: np.ndarray, t: int,
                  p: Params, scale: float) -> np.ndarray:
    """S_shared of one (kv group, query token): for each visible stage-1
    window j, the sum over the group's G query heads of that head's softmax
    probability exp(s_hj - LSE_h) ([top168] §三 second stage: heads of a GQA
    group share one importance score, obtained by summing inside the group;
    §四: the group sum is fused with the score computation so only this
    reduced tensor is stored).  Returns [visible C1 windows]."""
    n1 = visible_windows(t, p.c1_len, p.c1_stride)
    lse = group_lse(q_g, Kc1_g, Kc2_g, t, p, scale)
    S = np.zeros(n1, dtype=np.float64)
    for h in range(q_g.shape[0]):
        s1 = (Kc1_g[:n1] @ q_g[h]) * scale
        S += np.exp(s1 - lse[h])
    return S


# ----------------------------------------------------------------------------
# step 3: max-pool to block scores, then init + local + top-k selection
# ----------------------------------------------------------------------------
def block_scores(S: np.ndarray, t: int, p: Params) -> np.ndarray:
    """Stage-3 max pooling ([top168] §三 third stage: max pooling with l=5,
    s=4, giving the same compression ratio as pooling by B at once; the block
    score comes from several sliding sub-blocks inside the block).
    Reading: padding 1, so block b takes the maximum over C1 windows
    [s*b - 1, s*b - 1 + l - 1] = [4b-1, 4b+3], exactly the five windows that
    overlap block b; windows outside the visible range are skipped.  Blocks
    with no visible window get -inf.  Returns scores for blocks 0..b_t."""
    b_t = t // p.block
    out = np.full(b_t + 1, -np.inf)
    for b in range(b_t + 1):
        lo = b * p.pool_stride - p.pool_pad
        hi = lo + p.pool_len - 1
        js = [j for j in range(lo, hi + 1) if 0 <= j < S.shape[0]]
        if js:
            out[b] = max(S[j] for j in js)
    return out


def select_blocks(S: np.ndarray, t: int, p: Params) -> np.ndarray:
    """Blocks attended by the query at position t, shared by its kv group
    ([top168] §七: a query in block b_i always attends a fixed set of initial
    blocks and of local blocks, and a top-k over the remaining blocks; the
    attended set is their union.  [blog] "先看一个具体例子": 1 initial block,
    the 32 most recent blocks ending at the query's own block, and top-k far
    blocks, 96 blocks in all).
    Readings: the local window includes the query's own block; ties in the
    top-k go to the lower block index; with fewer candidates than top_k all
    candidates are taken.  Returns |I| block indices, ascending, padded with
    -1."""
    b_t = t // p.block
    init = set(range(0, min(p.n_init, b_t + 1)))
    local = set(range(max(0, b_t - p.n_local + 1), b_t + 1))
    cand = [b for b in range(b_t + 1) if b not in init and b not in local]
    bs = block_scores(S, t, p)
    k = min(p.top_k, len(cand))
    order = sorted(cand, key=lambda b: (-bs[b], b))
    chosen = sorted(init | local | set(order[:k]))
    out = np.full(p.n_sel, -1, dtype=np.int64)
    out[:len(chosen)] = chosen
    return out


# ----------------------------------------------------------------------------
# step 4: block-sparse causal attention (and the dense causal path)
# ----------------------------------------------------------------------------
def attend(q_g: np.ndarray, K_g: np.ndarray, V_g: np.ndarray, t: int,
           keys: np.ndarray, scale: float) -> np.ndarray:
    """softmax(q k^T * scale) v over the listed key positions, per head.
    q_g [G, d]; K_g, V_g [n, d] of the group; keys: positions <= t."""
    if keys.size == 0:
        return np.zeros_like(q_g)
    s = (q_g @ K_g[keys].T) * scale                       # [G, nk]
    s = s - s.max(axis=1, keepdims=True)
    w = np.exp(s)
    w = w / w.sum(axis=1, keepdims=True)
    return w @ V_g[keys]


def sparse_keys(t: int, blocks: Sequence[int], block: int) -> np.ndarray:
    """Key positions u <= t whose block u // B is selected ([blog] "对齐计算图":
    selected and sliding attention are one sparse attention over the chosen
    blocks, causal inside the query's own block)."""
    keys: List[int] = []
    for b in sorted(int(x) for x in blocks if x >= 0):
        lo, hi = b * block, min(b * block + block - 1, t)
        keys.extend(range(lo, hi + 1))
    return np.asarray(keys, dtype=np.int64)


def dense_keys(t: int) -> np.ndarray:
    """All positions u <= t (dense causal attention, the short-sequence mode
    of the dense/sparse switch, [blog] "Dense-Sparse Switchable Attention")."""
    return np.arange(t + 1, dtype=np.int64)


# ----------------------------------------------------------------------------
# step 4, backward: gradients of the block-sparse attention over a fixed
# selection.  The method is trained end to end with no added parameters
# ([news] §二, [top168] §一): the block selection is a discrete choice with no
# gradient, and the loss reaches Q, K and V through the attention over the
# selected keys.  Reading: the gradient is that of attend() with the key set
# held fixed.
# ----------------------------------------------------------------------------
def attend_backward(q_g: np.ndarray, K_g: np.ndarray, V_g: np.ndarray, keys: np.ndarray,
                    dO_g: np.ndarray, scale: float):
    """Gradients of sum(dO_g * attend(q_g, K_g, V_g, t, keys, scale)) with
    respect to q_g [G, d] and to the rows K_g[keys], V_g[keys] ([nk, d] each),
    by the chain rule through O = P V, P = softmax(S), S = scale q K^T:
      dV = P^T dO,   dP = dO V^T,
      dS = P * (dP - rowsum(P * dP))      (the softmax Jacobian),
      dq = scale dS K,   dK = scale dS^T q."""
    G, d = q_g.shape
    if keys.size == 0:
        return np.zeros((G, d)), np.zeros((0, d)), np.zeros((0, d))
    Kk, Vk = K_g[keys], V_g[keys]
    s = (q_g @ Kk.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    P = np.exp(s)
    P = P / P.sum(axis=1, keepdims=True)
    dV = P.T @ dO_g
    dP = dO_g @ Vk.T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    return scale * (dS @ Kk), scale * (dS.T @ q_g), dV


def sparse_attention_backward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, blocks: np.ndarray,
                              dO: np.ndarray, p: "Params"):
    """Gradients of sum(dO * O) for one sequence, O[t, h] the block-sparse
    attention of token t, query head h over the keys of its group's selected
    blocks blocks[t, g] (-1 entries ignored), as sparse_keys() lists them.
    Q, dO [n, h_q, d]; K, V [n, h_kv, d]; returns dQ, dK, dV in fp64.  A key's
    gradient sums over the G heads of its group and every token whose
    selection holds it."""
    n, h_q, d = Q.shape
    h_kv = K.shape[1]
    G = h_q // h_kv
    scale = p.softmax_scale(d)
    dQ, dK, dV = np.zeros(Q.shape), np.zeros(K.shape), np.zeros(V.shape)
    for t in range(n):
        for g in range(h_kv):
            keys = sparse_keys(t, blocks[t, g], p.block)
            hs = slice(g * G, (g + 1) * G)
            dq, dk, dv = attend_backward(Q[t, hs], K[:, g], V[:, g], keys, dO[t, hs], scale)
            dQ[t, hs] = dq
            dK[keys, g] += dk                  # keys are distinct within one row
            dV[keys, g] += dv
    return dQ, dK, dV


def invert_block_lists(blocks: np.ndarray, n: int, block: int) -> List[List[List[int]]]:
    """For every kv group g and key block kb, the tokens t whose selection
    blocks[t, g] holds kb, ascending: the inverse of the block lists, the
    order in which a key-block-major backward visits its query rows."""
    h_kv = blocks.shape[1]
    nblk = (n + block - 1) // block
    inv: List[List[List[int]]] = [[[] for _ in range(nblk)] for _ in range(h_kv)]
    for t in range(n):
        for g in range(h_kv):
            for kb in blocks[t, g]:
                if kb >= 0:
                    inv[g][int(kb)].append(t)
    return inv


def key_block_gradients(Q: np.ndarray, K: np.ndarray, V: np.ndarray, blocks: np.ndarray,
                        dO: np.ndarray, p: "Params"):
    """dK and dV of sparse_attention_backward() gathered per key block instead
    of scattered per query row: for block kb of group g, the sum over the
    tokens that selected it of that row's contribution to the block's keys
    (only keys <= t count for token t).  Same result, no two rows writing
    one key at once."""
    n, h_q, d = Q.shape
    h_kv = K.shape[1]
    G = h_q // h_kv
    scale = p.softmax_scale(d)
    inv = invert_block_lists(blocks, n, p.block)
    dK, dV = np.zeros(K.shape), np.zeros(V.shape)
    for g in range(h_kv):
        hs = slice(g * G, (g + 1) * G)
        for kb, rows in enumerate(inv[g]):
            lo = kb * p.block
            for t in rows:
                keys = sparse_keys(t, blocks[t, g], p.block)
                _, dk, dv = attend_backward(Q[t, hs], K[:, g], V[:, g], keys, dO[t, hs], scale)
                mine = (keys >= lo) & (keys < lo + p.block)
                dK[keys[mine], g] += dk[mine]
                dV[keys[mine], g] += dv[mine]
    return dK, dV


def block_rows(blocks: np.ndarray, g: int, kb: int) -> np.ndarray:
    """The tokens t whose selection blocks[t, g] holds block kb, ascending."""
    return np.nonzero((blocks[:, g, :] == kb).any(axis=1))[0]


def one_block_gradients(Q: np.ndarray, K: np.ndarray, V: np.ndarray, blocks: np.ndarray, dO: np.ndarray,
                        p: "Params", g: int, kb: int):
    """dK and dV of the 64 keys of block kb of group g alone ([B, d] each,
    fewer rows for a partial last block): key_block_gradients() for one
    block, for checks that cannot afford every block."""
    n, h_q, d = Q.shape
    G = h_q // K.shape[1]
    scale = p.softmax_scale(d)
    lo, hi = kb * p.block, min(n, kb * p.block + p.block)
    hs = slice(g * G, (g + 1) * G)
    dk, dv = np.zeros((hi - lo, d)), np.zeros((hi - lo, d))
    for t in block_rows(blocks, g, kb):
        keys = sparse_keys(int(t), blocks[t, g], p.block)
        _, dkr, dvr = attend_backward(Q[t, hs], K[:, g], V[:, g], keys, dO[t, hs], scale)
        mine = (keys >= lo) & (keys < hi)
        dk[keys[mine] - lo] += dkr[mine]
        dv[keys[mine] - lo] += dvr[mine]
    return dk, dv


# ----------------------------------------------------------------------------
# per-sequence drivers
# ----------------------------------------------------------------------------
class Sequence1:
    """One sequence's inputs in fp64 plus its pooled keys.

    Q [n, h_q, d], K/V [n, h_kv, d] (bf16-exact fp64)."""

    def __init__(self, Q: np.ndarray, K: np.ndarray, V: np.ndarray, p: Params):
        self.Q, self.K, self.V, self.p = Q, K, V, p
        self.n, self.h_q, self.d = Q.shape
        self.h_kv = K.shape[1]
        self.G = self.h_q // self.h_kv
        self.scale = p.softmax_scale(self.d)
        self.Kc1 = pool_keys(K, p.c1_len, p.c1_stride)     # [h_kv, n_c1, d]
        self.Kc2 = pool_keys(K, p.c2_len, p.c2_stride)     # [h_kv, n_c2, d]

    def q_group(self, t: int, g: int) -> np.ndarray:
        return self.Q[t, g * self.G:(g + 1) * self.G, :]

    def shared_scores(self, t: int, g: int) -> np.ndarray:
        return shared_scores(self.q_group(t, g), self.Kc1[g], self.Kc2[g], t, self.p, self.scale)

    def select(self, t: int, g: int) -> np.ndarray:
        return select_blocks(self.shared_scores(t, g), t, self.p)

    def sparse_out(self, t: int, g: int, blocks: Sequence[int]) -> np.ndarray:
        keys = sparse_keys(t, blocks, self.p.block)
        return attend(self.q_group(t, g), self.K[:, g, :], self.V[:, g, :], t, keys, self.scale)

    def dense_out(self, t: int, g: int) -> np.ndarray:
        return attend(self.q_group(t, g), self.K[:, g, :], self.V[:, g, :], t, dense_keys(t), self.scale)


def decode_row(K_seq: np.ndarray, V_seq: np.ndarray, q_t: np.ndarray, p: Params):
    """One decode step: the new token at position t = len(K_seq) - 1 is row t
    of the prefill rule on the extended sequence ([news] §二.2.b: the sparse
    pattern serves prefill and decode alike), so this calls the pinned prefill
    functions.  K_seq, V_seq: [t+1, h_kv, d] including the new token;
    q_t: [h_q, d].  Returns (selected blocks [h_kv, |I|], output [h_q, d],
    scores per group, the pooled keys K_C1, K_C2)."""
    t = K_seq.shape[0] - 1
    h_q, d = q_t.shape
    h_kv = K_seq.shape[1]
    G = h_q // h_kv
    scale = p.softmax_scale(d)
    Kc1 = pool_keys(K_seq, p.c1_len, p.c1_stride)
    Kc2 = pool_keys(K_seq, p.c2_len, p.c2_stride)
    sel = np.empty((h_kv, p.n_sel), dtype=np.int64)
    out = np.empty((h_q, d))
    scores = []
    for g in range(h_kv):
        qg = q_t[g * G:(g + 1) * G]
        S = shared_scores(qg, Kc1[g], Kc2[g], t, p, scale)
        scores.append(S)
        sel[g] = select_blocks(S, t, p)
        keys = sparse_keys(t, sel[g], p.block)
        out[g * G:(g + 1) * G] = attend(qg, K_seq[:, g, :], V_seq[:, g, :], t, keys, scale)
    return sel, out, scores, Kc1, Kc2


def lse_rows_comparable(t: int, p: Params) -> bool:
    """Rows whose scores are defined by the approximation proper (at least one
    C2 window visible).  Earlier rows use the exact fallback; they never reach
    the top-k, because they have no candidate blocks."""
    return visible_windows(t, p.c2_len, p.c2_stride) > 0


def topk_gap(S: np.ndarray, t: int, p: Params) -> float:
    """Relative gap between the k-th and (k+1)-th largest candidate block
    scores of a row, (s_k - s_{k+1}) / s_k; +inf when every candidate is
    taken (the selection is then independent of the scores)."""
    b_t = t // p.block
    init = set(range(0, min(p.n_init, b_t + 1)))
    local = set(range(max(0, b_t - p.n_local + 1), b_t + 1))
    cand = [b for b in range(b_t + 1) if b not in init and b not in local]
    if len(cand) <= p.top_k:
        return math.inf
    bs = block_scores(S, t, p)
    v = np.sort(np.array([bs[b] for b in cand]))[::-1]
    k = p.top_k
    if v[k - 1] <= 0:
        return 0.0
    return float((v[k - 1] - v[k]) / v[k - 1])


def dense_route(length: int, threshold: int = 8192) -> bool:
    """The dense/sparse switch ([blog] "Dense-Sparse Switchable Attention";
    [news] §二.2.c: below a threshold such as 8K or 16K the dense path runs).
    Reading: dense when length <= 8192, else sparse; exactly one path runs."""
    return length <= threshold


def to_f64(x) -> np.ndarray:
    """torch bf16 / float tensor or numpy array -> fp64 numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)
