"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Small cases compare every row; the 32K and 128K workloads run the full
CUDA path in the benchmark's launch configuration and compare a uniform
sample of rows that the oracle computes one by one."""
import dataclasses

import numpy as np
import pytest
import torch

from inputs import gen
from oracle import infllm2_oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu

VARLEN_SMALL = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="varlen_small", n_local=4, top_k=6, seed=7)
VARLEN_SMALL_LENS = [1000, 1057, 31, 127, 128, 200, 3000, 64, 1]
TINY_VARLEN = dataclasses.replace(gen.WORKLOADS["tiny_1k"], name="tiny_varlen", seed=8)
TINY_VARLEN_LENS = [333, 700, 1500, 17]


def _compare_pooled(run, seqs):
    c1o, c2o = run.c1_offsets(), run.c2_offsets()
    Kc1 = run.Kc1.float().cpu().numpy()
    Kc2 = run.Kc2.float().cpu().numpy()
    for s, seq in seqs.items():
        n1 = seq.Kc1.shape[1]
        n2 = seq.Kc2.shape[1]
        np.testing.assert_array_equal(Kc1[:, c1o[s]:c1o[s] + n1, :], seq.Kc1)
        np.testing.assert_array_equal(Kc2[:, c2o[s]:c2o[s] + n2, :], seq.Kc2)


def _check_rows(run, data, w, rows, seqs, S_gpu, idx_gpu, min_exact=0.85):
    """Scores (rel 1e-4 on visible entries of rows with a coarse window),
    selection (bit-exact where the top-k gap exceeds 1e-4) for the rows."""
    p = H.oracle_params(w)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    worst = 0.0
    ref_idx = {}
    lists, S_rows, ts = [], [], []
    for k, (row, s, t) in enumerate(zip(rows, sidx, tloc)):
        seq = seqs[int(s)]
        for g in range(w.h_kv):
            S_or = seq.shared_scores(int(t), g)
            n1 = S_or.shape[0]
            if O.lse_rows_comparable(int(t), p) and n1 > 0:
                got = S_gpu[g, k, :n1].astype(np.float64)
                rel = np.abs(got - S_or) / np.maximum(S_or, 1e-30)
                worst = max(worst, float(rel.max()))
            ref_idx[(int(row), g)] = O.select_blocks(S_or, int(t), p)
            lists.append(idx_gpu[g, k])
            S_rows.append(S_or)
            ts.append(int(t))
    assert worst <= H.S_RTOL, f"S_shared max relative error {worst:.3e}"
    exact, tie, bad = H.compare_lists(lists, S_rows, ts, p)
    print(f"[{w.name}] selection: {exact} rows bit-exact, {tie} near-tie rows valid, S_shared rel err {worst:.2e}")
    assert bad == 0, f"{bad} of {exact} selections differ"
    # a floor on the rows compared bit for bit, so that a regression that
    # narrows every gap cannot pass by skipping rows
    assert exact >= min_exact * (exact + tie), (exact, tie)
    return ref_idx


def _check_attention(run, w, rows, seqs, ref_idx):
    torch.cuda.synchronize()
    assert T_status() == 0, T_status()     # a device-side timeout or bounds record voids the output
    p = H.oracle_params(w)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    out = run.out.float().cpu().numpy()
    errs = []
    for row, s, t in zip(rows, sidx, tloc):
        seq = seqs[int(s)]
        for g in range(w.h_kv):
            o_ref = seq.sparse_out(int(t), g, ref_idx[(int(row), g)])
            o_gpu = out[int(row), g * w.group:(g + 1) * w.group, :]
            errs.append(np.abs(o_gpu - o_ref))
    e = np.concatenate([x.ravel() for x in errs])
    assert e.max() <= H.ATT_MAX_ABS and e.mean() <= H.ATT_MEAN_ABS, (e.max(), e.mean())
    return float(e.max()), float(e.mean())


def _full_case(w, lens, seed):
    data = gen.make_prefill(w, lens=lens, seed=seed)
    run = H.DeviceRun(data, w)
    run.compress()
    run.scores()
    run.topk()
    torch.cuda.synchronize()
    seqs = H.oracle_sequences(data, w)
    _compare_pooled(run, seqs)
    rows = np.arange(run.vl.total)
    S_gpu = run.S.cpu().numpy()
    idx_gpu = run.idx.cpu().numpy()
    ref_idx = _check_rows(run, data, w, rows, seqs, S_gpu, idx_gpu)

    # top-k alone, fed the oracle's scores rounded to fp32: bit-exact on every row
    p = H.oracle_params(w)
    S_in = np.zeros_like(S_gpu)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    want = np.empty_like(idx_gpu)
    for row, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            S_or = seqs[int(s)].shared_scores(int(t), g).astype(np.float32)
            S_in[g, row, :S_or.shape[0]] = S_or
            want[g, row] = O.select_blocks(S_or.astype(np.float64), int(t), p)
    S_dev = torch.from_numpy(S_in).cuda()
    run.topk(S_dev)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(run.idx.cpu().numpy(), want)

    # attention with the oracle's block lists fed to both sides
    idx_ref = np.stack([np.stack([ref_idx[(int(r), g)] for r in rows]) for g in range(w.h_kv)]).astype(np.int32)
    run.sparse(torch.from_numpy(idx_ref).cuda())
    torch.cuda.synchronize()
    _check_attention(run, w, rows, seqs, ref_idx)
    assert T_status() == 0


def T_status():
    import trainable_block_sparse_pool_b200 as T
    return T.infllm2_get_device_status()


def test_tiny_1k_full():
    w = gen.WORKLOADS["tiny_1k"]
    _full_case(w, [w.seqlen], w.seed)


def test_varlen_small_d128_g16():
    _full_case(VARLEN_SMALL, VARLEN_SMALL_LENS, VARLEN_SMALL.seed)


def test_varlen_tiny_d64_g4():
    _full_case(TINY_VARLEN, TINY_VARLEN_LENS, TINY_VARLEN.seed)


# The other supported group sizes and head dims.  G = 1 makes one LOCAL CTA
# (128 / G = 128 tokens) span two 64-token blocks, so its rows have
# different init/local sets; G = 2 and 8 exercise the remaining template
# cases of every kernel.
OTHER_GROUPS = [
    ("g1_d64", dict(h_q=4, h_kv=4, d=64)),
    ("g2_d128", dict(h_q=8, h_kv=4, d=128)),
    ("g8_d64", dict(h_q=16, h_kv=2, d=64)),
]
OTHER_LENS = [1300, 129, 2100, 64]


@pytest.mark.parametrize("name,shape", OTHER_GROUPS, ids=[g[0] for g in OTHER_GROUPS])
def test_varlen_group_sizes(name, shape):
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name=name, n_local=4, top_k=6, seed=31, **shape)
    _full_case(w, OTHER_LENS, w.seed)


def test_exact_lse_mode():
    # lse_mode EXACT: each head's log-sum-exp over the visible C1 windows
    # ([top168] §四's two-pass computation).  S_shared against the oracle's
    # exact variant on every row, and every row with a visible window sums
    # to G.
    import trainable_block_sparse_pool_b200 as T
    w = VARLEN_SMALL
    data = gen.make_prefill(w, lens=VARLEN_SMALL_LENS, seed=12)
    run = H.DeviceRun(data, w)
    run.p.lse_mode = T.LSE_EXACT
    run.compress()
    run.scores()
    torch.cuda.synchronize()
    op = dataclasses.replace(H.oracle_params(w), lse_mode="exact")
    seqs = H.oracle_sequences(data, w, p=op)
    S_gpu = run.S.cpu().numpy()
    rows = np.arange(run.vl.total)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    worst_rel, worst_sum, nrows = 0.0, 0.0, 0
    for row, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            S_or = seqs[int(s)].shared_scores(int(t), g)
            n1 = S_or.shape[0]
            if n1 == 0:
                continue
            got = S_gpu[g, row, :n1].astype(np.float64)
            worst_rel = max(worst_rel, float((np.abs(got - S_or) / np.maximum(S_or, 1e-30)).max()))
            worst_sum = max(worst_sum, abs(float(got.sum()) - w.group) / w.group)
            nrows += 1
    assert nrows > 0
    assert worst_rel <= H.S_RTOL, worst_rel
    assert worst_sum <= H.S_RTOL, worst_sum
    assert T_status() == 0


@pytest.mark.parametrize("name", ["varlen_small", "prefill_32k"])
def test_pooled_scores(name):
    # the max-pool's first step fused into the score kernel: the pairs give
    # the same lists as S_shared on every row (bit for bit), and the block
    # scores rebuilt from them match the oracle's max-pool at sampled rows
    import trainable_block_sparse_pool_b200 as T
    if name == "varlen_small":
        w = VARLEN_SMALL
        data = gen.make_prefill(w, lens=VARLEN_SMALL_LENS, seed=12)
    else:
        w = gen.WORKLOADS[name]
        data = gen.make_prefill(w)
    run = H.DeviceRun(data, w)
    run.compress()
    run.scores()
    run.topk()
    ldp = T.infllm2_pooled_ld(run.vl, run.p)
    P = torch.zeros(w.h_kv, run.vl.total, ldp, dtype=torch.float32, device="cuda")
    idx_p = torch.full_like(run.idx, -7)
    T.infllm2_pooled_scores(run.Q, run.Kc1, run.Kc2, run.vl, w.h_kv, P, ldp, run.p)
    T.infllm2_topk_blocks_pooled(P, ldp, run.vl, w.h_kv, idx_p, run.p)
    torch.cuda.synchronize()
    assert torch.equal(idx_p, run.idx)
    rows = gen.sample_rows(run.vl.total, 48, seed=w.seed + 23)
    P_cpu = P[:, torch.from_numpy(rows).cuda(), :].cpu().numpy().astype(np.float64)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    seqs = H.oracle_sequences(data, w, which=sorted(set(int(x) for x in sidx)))
    op = H.oracle_params(w)
    worst, n = 0.0, 0
    for k, (s, t) in enumerate(zip(sidx, tloc)):
        t = int(t)
        for g in range(w.h_kv):
            S_or = seqs[int(s)].shared_scores(t, g)
            ref = O.block_scores(S_or, t, op)
            # every block whose first window is visible has its pair
            nb = (S_or.shape[0] + 3) // 4
            for b in range(min(nb, ref.shape[0])):
                got = P_cpu[g, k, 2 * b]
                if b >= 1:
                    got = max(got, P_cpu[g, k, 2 * b - 1])
                worst = max(worst, abs(got - ref[b]) / max(abs(ref[b]), 1e-30))
                n += 1
    assert n > 0
    assert worst <= H.S_RTOL, worst
    assert T_status() == 0


def _sampled_case(name, n_rows, min_exact):
    w = gen.WORKLOADS[name]
    data = gen.make_prefill(w)
    run = H.DeviceRun(data, w)
    run.compress()
    run.scores()
    run.topk()
    torch.cuda.synchronize()
    seqs = H.oracle_sequences(data, w)
    _compare_pooled(run, seqs)
    rows = gen.sample_rows(run.vl.total, n_rows, seed=w.seed + 17)
    rows_t = torch.from_numpy(rows).cuda()
    S_gpu = run.S[:, rows_t, :].cpu().numpy()
    idx_gpu = run.idx[:, rows_t, :].cpu().numpy()
    ref_idx = _check_rows(run, data, w, rows, seqs, S_gpu, idx_gpu, min_exact=min_exact)
    # attention: oracle lists at the sampled rows, a valid default list elsewhere
    full = H.default_index_rows(run.lens, w)
    idx_all = np.stack([full.copy() for _ in range(w.h_kv)])
    for g in range(w.h_kv):
        for r in rows:
            idx_all[g, r] = ref_idx[(int(r), g)]
    run.sparse(torch.from_numpy(idx_all).cuda())
    torch.cuda.synchronize()
    _check_attention(run, w, rows, seqs, ref_idx)
    assert T_status() == 0


def test_prefill_32k_sampled():
    _sampled_case("prefill_32k", 128, 0.85)


def test_prefill_128k_sampled():
    _sampled_case("prefill_128k", 48, 0.8)


@pytest.mark.parametrize("with_s_out", [False, True], ids=["workspace", "s_shared_out"])
def test_select_blocks_entry_point(with_s_out):
    # the one-call selection (scores + max-pool + top-k) against the oracle on
    # every row of a ragged batch: with S_shared in the caller's workspace,
    # and with S_shared written out (then compared too)
    import trainable_block_sparse_pool_b200 as T
    w = VARLEN_SMALL
    data = gen.make_prefill(w, lens=VARLEN_SMALL_LENS, seed=13)
    run = H.DeviceRun(data, w)
    run.compress()
    run.idx.fill_(-7)
    if with_s_out:
        T.infllm2_select_blocks(run.Q, run.Kc1, run.Kc2, run.vl, w.h_kv, None, run.idx, run.S, run.p)
    else:
        ws = torch.empty(T.infllm2_select_workspace_bytes(run.vl, w.h_kv, run.p), dtype=torch.uint8, device="cuda")
        T.infllm2_select_blocks(run.Q, run.Kc1, run.Kc2, run.vl, w.h_kv, ws, run.idx, None, run.p)
    torch.cuda.synchronize()
    seqs = H.oracle_sequences(data, w)
    rows = np.arange(run.vl.total)
    p = H.oracle_params(w)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    idx_gpu = run.idx.cpu().numpy()
    S_gpu = run.S.cpu().numpy() if with_s_out else None
    lists, S_rows, ts, worst = [], [], [], 0.0
    for row, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            S_or = seqs[int(s)].shared_scores(int(t), g)
            lists.append(idx_gpu[g, row])
            S_rows.append(S_or)
            ts.append(int(t))
            if with_s_out and O.lse_rows_comparable(int(t), p) and S_or.shape[0] > 0:
                got = S_gpu[g, row, :S_or.shape[0]].astype(np.float64)
                worst = max(worst, float((np.abs(got - S_or) / np.maximum(S_or, 1e-30)).max()))
    exact, tie, bad = H.compare_lists(lists, S_rows, ts, p)
    print(f"[select_blocks] {exact} rows bit-exact, {tie} near-tie rows valid")
    assert bad == 0 and exact >= 0.85 * (exact + tie), (bad, exact, tie)
    assert worst <= H.S_RTOL, worst
    assert T_status() == 0


def test_sparse_attn_flags_lists_without_their_local_run():
    # a row whose list lacks one block of its local run (replaced by another
    # block of the same sequence, so every entry is still a valid block) is
    # reported through the device status word instead of silently giving a
    # result that is not the attention over the list
    import trainable_block_sparse_pool_b200 as T
    w = VARLEN_SMALL
    lens = [3000]
    data = gen.make_prefill(w, lens=lens, seed=14)
    run = H.DeviceRun(data, w)
    good = H.default_index_rows(lens, w)
    idx = np.stack([good.copy() for _ in range(w.h_kv)])
    T.infllm2_clear_device_status()
    run.sparse(torch.from_numpy(idx).cuda())
    assert T.infllm2_get_device_status() == 0
    t = 2900
    row = idx[1, t]
    b_t = t // 64
    assert b_t in row and 20 not in row
    bad = np.sort(np.where(row == b_t - 1, 20, row))
    idx[1, t] = bad
    run.sparse(torch.from_numpy(idx).cuda())
    assert T.infllm2_get_device_status() == -6
    T.infllm2_clear_device_status()
    assert T.infllm2_get_device_status() == 0


def test_deterministic_reruns():
    w = VARLEN_SMALL
    data = gen.make_prefill(w, lens=VARLEN_SMALL_LENS, seed=11)
    outs = []
    for _ in range(2):
        run = H.DeviceRun(data, w)
        run.compress(); run.scores(); run.topk(); run.sparse()
        torch.cuda.synchronize()
        outs.append((run.Kc1.cpu(), run.S.cpu(), run.idx.cpu(), run.out.cpu()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_bounded_wait_reports_timeout():
    import trainable_block_sparse_pool_b200 as T
    T.infllm2_clear_device_status()
    T.infllm2_debug_wait_timeout(50_000_000)   # 50 ms
    assert T.infllm2_get_device_status() == -5
    T.infllm2_clear_device_status()
    assert T.infllm2_get_device_status() == 0
