"""Pins for the fp64 oracle: closed forms, invariants, brute force, a library
routine and the pages' worked example.  None of these re-types an oracle
formula; each would fail on a plausible slip (a dropped term, a wrong sign,
index or window, a transposed operand, a wrong head-to-group map)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import infllm2_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_round_matches_library_on_fp32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    # exact halfway cases: a bf16 value plus half of its last place
    base = _bf16(rng.standard_normal(5000).astype(np.float32))
    m, e = np.frexp(base)
    ties = (base + np.ldexp(np.sign(base), e - 9)).astype(np.float32)
    for arr in (x, ties):
        ref = torch.from_numpy(arr).to(torch.bfloat16).to(torch.float64).numpy()
        np.testing.assert_array_equal(O.bf16_round(arr.astype(np.float64)), ref)


def test_bf16_round_hand_cases():
    cases = {
        1.0 + 2.0 ** -8: 1.0,                       # tie -> even (1.0)
        1.0 + 3 * 2.0 ** -8: 1.0 + 2.0 ** -6,       # tie -> even (odd last bit rounds up)
        1.0 + 2.0 ** -8 + 2.0 ** -30: 1.0 + 2.0 ** -7,   # just above a tie rounds up
        -(1.0 + 2.0 ** -8): -1.0,
        3.4e38: math.inf,                           # beyond the largest bf16 + half a place
        2.0 ** -140: 0.0,
        0.0: 0.0,
    }
    for x, want in cases.items():
        assert O.bf16_round(np.array([x]))[0] == want, x


# ---------------------------------------------------------------- pooling
def test_window_counts_and_visibility():
    # n=1024: 63 stage-1 windows (l=32, s=16) and 15 coarse windows (l=128, s=64)
    assert O.window_count(1024, 32, 16) == 63
    assert O.window_count(1024, 128, 64) == 15
    assert O.window_count(31, 32, 16) == 0
    assert O.window_count(32768, 32, 16) == 2047
    assert O.window_count(131072, 128, 64) == 2047
    # visibility = windows whose whole token range is <= t, by enumeration
    for (l, s) in ((32, 16), (128, 64)):
        for t in range(0, 700):
            brute = sum(1 for j in range(0, 100) if all(u <= t for u in range(s * j, s * j + l)))
            assert O.visible_windows(t, l, s) == brute


def test_pool_constant_blocks():
    # K constant inside each 64-token block: windows inside a block give its
    # value, a window over two blocks gives the average of the two.
    rng = np.random.default_rng(1)
    n, h, d = 512, 2, 8
    mu = _bf16(rng.standard_normal((n // 64, h, d)))
    K = np.repeat(mu, 64, axis=0)
    c1 = O.pool_keys(K, 32, 16)
    c2 = O.pool_keys(K, 128, 64)
    assert c1.shape == (h, 31, d) and c2.shape == (h, 7, d)
    for j in range(31):
        b0, b1 = (16 * j) // 64, (16 * j + 31) // 64
        want = mu[b0] if b0 == b1 else _bf16((mu[b0] + mu[b1]) / 2)
        np.testing.assert_array_equal(c1[:, j, :], want)
    for m in range(7):
        np.testing.assert_array_equal(c2[:, m, :], _bf16((mu[m] + mu[m + 1]) / 2))


def test_pool_mean_of_ramp():
    # K[u] = u (exact in bf16 for u < 256): window j of length l, stride s has
    # mean s*j + (l-1)/2.
    n = 256
    K = np.arange(n, dtype=np.float64).reshape(n, 1, 1)
    c1 = O.pool_keys(K, 32, 16)[0, :, 0]
    assert np.array_equal(c1, O.bf16_round(16 * np.arange(15) + 15.5))
    c2 = O.pool_keys(K, 128, 64)[0, :, 0]
    assert np.array_equal(c2, O.bf16_round(64 * np.arange(3) + 63.5))


# ---------------------------------------------------------------- scoring
def _seq(n, h_q, h_kv, d, seed, p=O.Params(), q_zero_heads=()):
    rng = np.random.default_rng(seed)
    Q = _bf16(rng.standard_normal((n, h_q, d)))
    for h in q_zero_heads:
        Q[:, h, :] = 0.0
    K = _bf16(rng.standard_normal((n, h_kv, d)))
    V = _bf16(rng.standard_normal((n, h_kv, d)))
    return O.Sequence1(Q, K, V, p)


def test_scores_with_zero_query_are_uniform():
    # q = 0: every score is 0, LSE = ln(#visible C2 windows), so each visible
    # C1 window gets G / #C2-windows; before any C2 window is visible the
    # exact normaliser over the C1 windows gives G / #C1-windows.
    s = _seq(600, 4, 1, 16, 2, q_zero_heads=range(4))
    for t in (31, 47, 126, 127, 128, 191, 192, 400, 599):
        S = s.shared_scores(t, 0)
        n1 = O.visible_windows(t, 32, 16)
        n2 = O.visible_windows(t, 128, 64)
        assert S.shape == (n1,)
        want = 4.0 / (n2 if n2 > 0 else n1)
        np.testing.assert_allclose(S, want, rtol=1e-14)
    assert s.shared_scores(30, 0).shape == (0,)


def test_head_to_group_map_is_contiguous():
    # h_q=4, h_kv=2: group 0 owns heads 0 and 1.  Zero exactly those.
    s = _seq(400, 4, 2, 16, 3, q_zero_heads=(0, 1))
    t = 300
    n2 = O.visible_windows(t, 128, 64)
    np.testing.assert_allclose(s.shared_scores(t, 0), 2.0 / n2, rtol=1e-14)
    assert np.ptp(s.shared_scores(t, 1)) > 1e-3


def test_exact_lse_rows_sum_to_group_size():
    # with the exact normaliser each head's probabilities sum to 1 over the
    # visible windows, so the group sum adds up to G
    p = O.Params(lse_mode="exact")
    s = _seq(700, 8, 2, 32, 4, p=p)
    for t in (31, 100, 333, 699):
        for g in range(2):
            assert abs(s.shared_scores(t, g).sum() - 4.0) < 1e-12


def test_scale_and_lse_by_hand():
    # d=64, scale 1/8.  Two C1 windows: k0 = 0, k1 = e_0; every head has
    # q = 8 e_0, so s = (0, 1).  Exact mode: S = G * (1, e) / (1 + e).
    d, G = 64, 3
    q = np.zeros((G, d)); q[:, 0] = 8.0
    Kc1 = np.zeros((2, d)); Kc1[1, 0] = 1.0
    p = O.Params(lse_mode="exact")
    S = O.shared_scores(q, Kc1, np.zeros((0, d)), 47, p, 1.0 / 8.0)
    e = math.e
    np.testing.assert_allclose(S, [G / (1 + e), G * e / (1 + e)], rtol=1e-14)
    # approximate mode: the normaliser comes from the C2 keys only.  One C2
    # window with k = 2 e_0 gives s2 = 2, LSE = 2, so S = G * (e^-2, e^-1).
    # At t=127 seven C1 windows are visible: k1 = e_0, the others 0.
    Kc2 = np.zeros((1, d)); Kc2[0, 0] = 2.0
    Kc1 = np.zeros((7, d)); Kc1[1, 0] = 1.0
    S = O.shared_scores(q, Kc1, Kc2, 127, O.Params(), 1.0 / 8.0)
    want = [G * math.exp(-2)] * 7
    want[1] = G * math.exp(-1)
    np.testing.assert_allclose(S, want, rtol=1e-14)


# ---------------------------------------------------------------- max-pool
def test_block_scores_match_token_overlap_definition():
    # Block b's score is the maximum over the visible C1 windows whose token
    # span [16j, 16j+31] overlaps the block's span [64b, 64b+63].
    rng = np.random.default_rng(5)
    p = O.Params()
    for t in (63, 64, 200, 777, 1023, 2047):
        n1 = O.visible_windows(t, 32, 16)
        S = rng.random(n1)
        bs = O.block_scores(S, t, p)
        assert bs.shape == (t // 64 + 1,)
        for b in range(t // 64 + 1):
            js = [j for j in range(n1) if 16 * j <= 64 * b + 63 and 16 * j + 31 >= 64 * b]
            want = max(S[j] for j in js) if js else -np.inf
            assert bs[b] == want
    # the max-pool compresses by 4 windows = 64 tokens = one block per output
    assert O.block_scores(np.ones(8191), 131071, p).shape == (2048,)


# ---------------------------------------------------------------- selection
def test_worked_example_32k():
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    p = O.Params()
    assert p.block == g["block"] and p.n_sel == g["n_selected_blocks"] and p.n_local == g["n_local"]
    rng = np.random.default_rng(6)
    for t in (g["token_1based"] - 1, g["token_1based"]):   # either reading of "the 20000th token"
        b_t = t // p.block
        assert b_t + 1 == g["block_1based"]
        S = rng.random(O.visible_windows(t, 32, 16))
        sel = O.select_blocks(S, t, p)
        assert len(sel) == g["n_selected_blocks"] and (sel >= 0).all()
        assert np.all(np.diff(sel) > 0)
        s1 = set((sel + 1).tolist())
        assert set(g["init_blocks_1based"]) <= s1
        assert set(range(g["local_first_block_1based"], g["local_last_block_1based"] + 1)) <= s1
        far = s1 - set(g["init_blocks_1based"]) - set(range(g["local_first_block_1based"], 314))
        assert len(far) == 63 and max(far) < g["local_first_block_1based"]
        assert len(sel) * p.block == g["visible_tokens"]


def test_topk_matches_bruteforce_subsets():
    # tiny parameters; scores drawn from a few values so ties are common.
    # The chosen far blocks must be the maximum-sum k-subset, ties broken
    # toward the lexicographically smallest index set.
    p = O.Params(n_init=1, n_local=2, top_k=3)
    rng = np.random.default_rng(7)
    for trial in range(200):
        t = int(rng.integers(64 * 5, 64 * 12))
        n1 = O.visible_windows(t, 32, 16)
        S = rng.integers(0, 4, n1).astype(np.float64)
        sel = set(O.select_blocks(S, t, p).tolist()) - {-1}
        b_t = t // 64
        bs = O.block_scores(S, t, p)
        cand = list(range(1, b_t - 1))
        best = max(itertools.combinations(cand, 3), key=lambda c: (sum(bs[b] for b in c), [-b for b in c]))
        assert sel == {0, b_t - 1, b_t} | set(best), (trial, t)


def test_topk_ties_take_lowest_blocks():
    # zero query: all block scores tie, so the top-k are the lowest candidates
    s = _seq(1024 * 8, 4, 1, 16, 8, q_zero_heads=range(4))
    p = s.p
    t = 8000
    sel = s.select(t, 0)
    b_t = t // 64
    want = [0] + list(range(1, 1 + p.top_k)) + list(range(b_t - 31, b_t + 1))
    assert sel.tolist() == want


def test_selected_count_and_always_selected():
    s = _seq(5000, 4, 1, 16, 9)
    for t in (0, 63, 64, 2111, 2112, 4000, 4999):
        sel = s.select(t, 0)
        b_t = t // 64
        valid = sel[sel >= 0]
        assert len(valid) == min(96, b_t + 1)
        assert 0 in valid
        assert set(range(max(0, b_t - 31), b_t + 1)) <= set(valid.tolist())
        assert (sel[len(valid):] == -1).all()


# ---------------------------------------------------------------- attention
def test_dense_matches_library_sdpa():
    rng = np.random.default_rng(10)
    n, h_q, h_kv, d = 200, 4, 2, 16
    s = _seq(n, h_q, h_kv, d, 10)
    G = h_q // h_kv
    q = torch.from_numpy(s.Q).permute(1, 0, 2)[None]
    k = torch.from_numpy(s.K).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    v = torch.from_numpy(s.V).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)[0].permute(1, 0, 2).numpy()
    for t in range(0, n, 7):
        for g in range(h_kv):
            np.testing.assert_allclose(s.dense_out(t, g), ref[t, g * G:(g + 1) * G], rtol=1e-12, atol=1e-13)


def test_sparse_equals_dense_when_every_block_is_selected():
    # |I| >= number of causal blocks -> sparse attention is dense attention
    p = O.Params(n_init=1, n_local=16, top_k=2)
    s = _seq(1024, 4, 1, 64, 11, p=p)
    for t in range(0, 1024, 13):
        sel = s.select(t, 0)
        assert sorted(sel[sel >= 0].tolist()) == list(range(t // 64 + 1))
        np.testing.assert_allclose(s.sparse_out(t, 0, sel), s.dense_out(t, 0), rtol=1e-13, atol=1e-14)


def test_zero_query_gives_mean_of_visible_values():
    s = _seq(3000, 4, 1, 16, 12, q_zero_heads=range(4))
    for t in (5, 64, 130, 2500, 2999):
        sel = s.select(t, 0)
        keys = [u for u in range(t + 1) if (u // 64) in set(sel.tolist())]
        want = s.V[keys, 0, :].mean(axis=0)
        out = s.sparse_out(t, 0, sel)
        for h in range(4):
            np.testing.assert_allclose(out[h], want, rtol=1e-12, atol=1e-14)


def test_dense_route_threshold():
    assert O.dense_route(8192) and not O.dense_route(8193) and O.dense_route(1)


# ---------------------------------------------------------------- attention backward
def _random_selection(rng, n, h_kv, n_sel, block=64):
    """A valid selection per (token, group): the token's own block plus a
    random subset of its earlier blocks, ascending, padded with -1."""
    out = np.full((n, h_kv, n_sel), -1, dtype=np.int64)
    for t in range(n):
        bt = t // block
        for g in range(h_kv):
            earlier = [b for b in range(bt) if rng.random() < 0.5][: n_sel - 1]
            sel = sorted(earlier + [bt])
            out[t, g, :len(sel)] = sel
    return out


def _sparse_forward(Q, K, V, blocks, p):
    n, h_q, d = Q.shape
    h_kv = K.shape[1]
    G = h_q // h_kv
    scale = p.softmax_scale(d)
    O_ = np.zeros(Q.shape)
    for t in range(n):
        for g in range(h_kv):
            keys = O.sparse_keys(t, blocks[t, g], p.block)
            O_[t, g * G:(g + 1) * G] = O.attend(Q[t, g * G:(g + 1) * G], K[:, g], V[:, g], t, keys, scale)
    return O_


def test_backward_matches_finite_differences():
    # central differences of sum(dO * O) on a small case with a random
    # (fixed) selection; the loss is smooth in Q, K and V
    rng = np.random.default_rng(30)
    n, h_q, h_kv, d = 160, 4, 2, 8
    p = O.Params(n_init=1, n_local=1, top_k=2)
    Q = rng.standard_normal((n, h_q, d))
    K = rng.standard_normal((n, h_kv, d))
    V = rng.standard_normal((n, h_kv, d))
    dO = rng.standard_normal((n, h_q, d))
    blocks = _random_selection(rng, n, h_kv, p.n_sel)
    dQ, dK, dV = O.sparse_attention_backward(Q, K, V, blocks, dO, p)
    eps = 1e-6

    def loss(Qx, Kx, Vx):
        return float((dO * _sparse_forward(Qx, Kx, Vx, blocks, p)).sum())

    for name, X, dX in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in X.shape)
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p = {"Q": (Xp, K, V), "K": (Q, Xp, V), "V": (Q, K, Xp)}[name]
            args_m = {"Q": (Xm, K, V), "K": (Q, Xm, V), "V": (Q, K, Xm)}[name]
            num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(num - dX[idx]) <= 1e-6 * max(1.0, abs(num)), (name, idx, num, dX[idx])


def test_backward_equals_dense_autograd_when_every_block_is_selected():
    # every causal block selected: the gradients are those of dense causal
    # GQA attention, here from fp64 autograd of the library routine
    rng = np.random.default_rng(31)
    n, h_q, h_kv, d = 200, 4, 2, 16
    p = O.Params(n_init=1, n_local=4, top_k=0)
    G = h_q // h_kv
    Q = rng.standard_normal((n, h_q, d))
    K = rng.standard_normal((n, h_kv, d))
    V = rng.standard_normal((n, h_kv, d))
    dO = rng.standard_normal((n, h_q, d))
    blocks = np.full((n, h_kv, p.n_sel), -1, dtype=np.int64)
    for t in range(n):
        blocks[t, :, :t // 64 + 1] = np.arange(t // 64 + 1)
    dQ, dK, dV = O.sparse_attention_backward(Q, K, V, blocks, dO, p)
    q = torch.from_numpy(Q).permute(1, 0, 2)[None].requires_grad_(True)
    k = torch.from_numpy(K).permute(1, 0, 2)[None].requires_grad_(True)
    v = torch.from_numpy(V).permute(1, 0, 2)[None].requires_grad_(True)
    out = torch.nn.functional.scaled_dot_product_attention(q, k.repeat_interleave(G, 1), v.repeat_interleave(G, 1),
                                                           is_causal=True)
    (out * torch.from_numpy(dO).permute(1, 0, 2)[None]).sum().backward()
    np.testing.assert_allclose(dQ, q.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, k.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, v.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_backward_value_gradient_sums_to_output_gradient():
    # the attention weights of a row sum to one, so the value gradients of a
    # group add up to the sum of its heads' output gradients over all tokens
    rng = np.random.default_rng(32)
    n, h_q, h_kv, d = 130, 4, 2, 8
    p = O.Params(n_init=1, n_local=1, top_k=1)
    Q = rng.standard_normal((n, h_q, d))
    K = rng.standard_normal((n, h_kv, d))
    V = rng.standard_normal((n, h_kv, d))
    dO = rng.standard_normal((n, h_q, d))
    blocks = _random_selection(rng, n, h_kv, p.n_sel)
    _, _, dV = O.sparse_attention_backward(Q, K, V, blocks, dO, p)
    G = h_q // h_kv
    for g in range(h_kv):
        np.testing.assert_allclose(dV[:, g].sum(axis=0), dO[:, g * G:(g + 1) * G].sum(axis=(0, 1)), rtol=1e-12,
                                   atol=1e-12)


def test_lse_approximation_cost_ratio():
    # [top168] §四: the coarse windows are 4x longer and 4x sparser, so the
    # approximation's coarse pass adds a quarter of a scoring pass (1.25x in
    # all) while the exact two-pass form doubles it (2x); counted here as
    # visible (token, window) products over a 128K sequence
    n = 131072
    fine = sum(O.visible_windows(t, 32, 16) for t in range(n))
    coarse = sum(O.visible_windows(t, 128, 64) for t in range(n))
    assert abs((fine + coarse) / fine - 1.25) < 2e-3
    assert (fine + fine) / fine == 2.0


def test_key_block_gradients_equal_row_scatter():
    # the key-block-major form (inverse lists) gives the row-major scatter's dK, dV
    rng = np.random.default_rng(33)
    n, h_q, h_kv, d = 300, 4, 2, 8
    p = O.Params(n_init=1, n_local=1, top_k=2)
    Q = rng.standard_normal((n, h_q, d))
    K = rng.standard_normal((n, h_kv, d))
    V = rng.standard_normal((n, h_kv, d))
    dO = rng.standard_normal((n, h_q, d))
    blocks = _random_selection(rng, n, h_kv, p.n_sel)
    _, dK, dV = O.sparse_attention_backward(Q, K, V, blocks, dO, p)
    dK2, dV2 = O.key_block_gradients(Q, K, V, blocks, dO, p)
    np.testing.assert_allclose(dK2, dK, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dV2, dV, rtol=1e-12, atol=1e-12)
    # every selected (token, block) pair appears once in the inverse lists
    inv = O.invert_block_lists(blocks, n, p.block)
    assert sum(len(r) for g in inv for r in g) == int((blocks >= 0).sum())


# ---------------------------------------------------------------- parity helpers
def _row_with_block_scores(t, values):
    """A C1 score row whose max-pooled block scores are exactly `values`
    ({block: score}; other blocks score 1e-9): block b's score is placed in
    window 4b+1, which lies in block b's pooling range [4b-1, 4b+3] only."""
    S = np.full(O.visible_windows(t, 32, 16), 1e-9)
    for b, v in values.items():
        S[4 * b + 1] = v
    return S


def test_topk_gap_hand_built_row():
    # n_init=1, n_local=2, top_k=2; t in block 9: init {0}, local {8, 9},
    # candidates {1..7}.  Candidate scores sorted: 0.9, 0.8 | 0.7, 0.5, ...
    # so the k-th is 0.8 and the (k+1)-th 0.7: gap = 0.1 / 0.8.
    p = O.Params(n_init=1, n_local=2, top_k=2)
    t = 9 * 64 + 63
    cand = {1: 0.5, 2: 0.9, 3: 0.3, 4: 0.8, 5: 0.1, 6: 0.7, 7: 0.2}
    S = _row_with_block_scores(t, cand)
    np.testing.assert_array_equal(O.block_scores(S, t, p)[1:8], [cand[b] for b in range(1, 8)])
    assert O.topk_gap(S, t, p) == pytest.approx(0.125, rel=1e-12)
    # init and local blocks are not candidates: large scores there change nothing
    S2 = _row_with_block_scores(t, {**cand, 0: 5.0, 8: 4.0, 9: 3.0})
    assert O.topk_gap(S2, t, p) == pytest.approx(0.125, rel=1e-12)
    # a tie at the boundary gives a zero gap; the gap is never negative
    S3 = _row_with_block_scores(t, {**cand, 6: 0.8})
    assert O.topk_gap(S3, t, p) == 0.0
    rng = np.random.default_rng(21)
    for _ in range(50):
        R = rng.random(O.visible_windows(t, 32, 16))
        assert O.topk_gap(R, t, p) >= 0.0


def test_topk_gap_infinite_when_every_candidate_is_taken():
    # block 4: init {0}, local {3, 4}, candidates {1, 2} = top_k: nothing to
    # choose, the gap is +inf; one more block makes it finite
    p = O.Params(n_init=1, n_local=2, top_k=2)
    rng = np.random.default_rng(22)
    t = 4 * 64 + 63
    assert O.topk_gap(rng.random(O.visible_windows(t, 32, 16)), t, p) == math.inf
    t = 5 * 64
    assert math.isfinite(O.topk_gap(rng.random(O.visible_windows(t, 32, 16)), t, p))
    # the default parameters: candidates exist only from block 1 + 32 + 63 = 96 on
    pd = O.Params()
    for t in (0, 2111, 96 * 64 - 1):
        assert O.topk_gap(rng.random(O.visible_windows(t, 32, 16)), t, pd) == math.inf
    t = 96 * 64
    assert math.isfinite(O.topk_gap(rng.random(O.visible_windows(t, 32, 16)), t, pd))


def test_lse_rows_comparable_boundary():
    # a row uses the coarse approximation from t = l_C2 - 1 = 127 on (its
    # first complete coarse window); before that the approximate and the
    # exact modes are the same computation, after it they differ
    p = O.Params()
    assert [O.lse_rows_comparable(t, p) for t in (0, 126, 127, 128, 5000)] == [False, False, True, True, True]
    pa, pe = O.Params(n_local=2, top_k=2), O.Params(n_local=2, top_k=2, lse_mode="exact")
    sa, se = _seq(400, 4, 1, 16, 23, p=pa), _seq(400, 4, 1, 16, 23, p=pe)
    for t in range(31, 400, 3):
        a, e = sa.shared_scores(t, 0), se.shared_scores(t, 0)
        if O.lse_rows_comparable(t, pa):
            assert np.abs(a - e).max() > 1e-6, t
        else:
            np.testing.assert_array_equal(a, e)
    # rows that are not comparable never reach the top-k: no candidates yet
    # (t < 127 lies in blocks 0 and 1, which are init or local)
    for t in range(127):
        assert O.topk_gap(np.ones(O.visible_windows(t, 32, 16)), t, O.Params(n_init=1, n_local=1, top_k=1)) == math.inf


def test_decode_row_is_row_t_of_the_prefill_rule():
    # decode of the token at t on the prefix K[:t+1] gives the selection and
    # output of row t of the prefill oracle on a LONGER sequence (causality:
    # later tokens change nothing for row t), and pooled keys that are the
    # prefix of the longer sequence's pooled keys
    p = O.Params(n_init=1, n_local=2, top_k=3)
    n, h_q, h_kv, d = 900, 4, 2, 16
    full = _seq(n, h_q, h_kv, d, 24, p=p)
    for t in (0, 31, 127, 128, 300, 511, 640, 899):
        sel, out, scores, Kc1, Kc2 = O.decode_row(full.K[:t + 1], full.V[:t + 1], full.Q[t], p)
        n1, n2 = O.window_count(t + 1, 32, 16), O.window_count(t + 1, 128, 64)
        assert Kc1.shape[1] == n1 and Kc2.shape[1] == n2
        np.testing.assert_array_equal(Kc1, full.Kc1[:, :n1])
        np.testing.assert_array_equal(Kc2, full.Kc2[:, :n2])
        for g in range(h_kv):
            np.testing.assert_array_equal(scores[g], full.shared_scores(t, g))
            np.testing.assert_array_equal(sel[g], full.select(t, g))
            np.testing.assert_allclose(out[g * 2:(g + 1) * 2], full.sparse_out(t, g, sel[g]), rtol=1e-13, atol=1e-15)
    # the last row of a sequence sees its own token: changing it changes the output
    t = 640
    V2 = full.V[:t + 1].copy()
    V2[t] += 1.0
    _, o1, _, _, _ = O.decode_row(full.K[:t + 1], full.V[:t + 1], full.Q[t], p)
    _, o2, _, _, _ = O.decode_row(full.K[:t + 1], V2, full.Q[t], p)
    assert np.abs(o1 - o2).min() > 0


def test_one_block_gradients_equal_the_key_block_form():
    # the per-block form used by sampled GPU checks equals the key-block-major
    # form over all blocks, block by block
    p = O.Params(n_init=1, n_local=2, top_k=2)
    rng = np.random.default_rng(31)
    n, h_q, h_kv, d = 330, 4, 2, 8
    Q = _bf16(rng.standard_normal((n, h_q, d)))
    K = _bf16(rng.standard_normal((n, h_kv, d)))
    V = _bf16(rng.standard_normal((n, h_kv, d)))
    dO = rng.standard_normal((n, h_q, d))
    blocks = _random_selection(rng, n, h_kv, p.n_sel)
    dK, dV = O.key_block_gradients(Q, K, V, blocks, dO, p)
    for g in range(h_kv):
        for kb in range((n + 63) // 64):
            dk, dv = O.one_block_gradients(Q, K, V, blocks, dO, p, g, kb)
            lo = 64 * kb
            np.testing.assert_allclose(dk, dK[lo:lo + dk.shape[0], g], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(dv, dV[lo:lo + dv.shape[0], g], rtol=1e-12, atol=1e-12)
    rows = O.block_rows(blocks, 0, 1)
    assert all(1 in blocks[t, 0] for t in rows) and len(rows) == sum(1 in blocks[t, 0] for t in range(n))
