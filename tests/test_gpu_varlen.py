"""The dense/sparse switch on the packed 128K varlen workload: sequences of
at most 8192 tokens take the dense path, longer ones the sparse path
(pool, select, sparse attention).  Sampled rows of both against the oracle."""
import numpy as np
import pytest
import torch

from inputs import gen
from oracle import infllm2_oracle as O
from tests import harness as H
import trainable_block_sparse_pool_b200 as T

pytestmark = pytest.mark.gpu


def _sub(data, which):
    cu = data["cu_seqlens"].tolist()
    parts = {k: [data[k][cu[s]:cu[s + 1]] for s in which] for k in ("Q", "K", "V")}
    lens = [data["lens"][s] for s in which]
    c = np.zeros(len(lens) + 1, dtype=np.int32)
    c[1:] = np.cumsum(lens)
    return {"Q": torch.cat(parts["Q"]), "K": torch.cat(parts["K"]), "V": torch.cat(parts["V"]),
            "cu_seqlens": torch.from_numpy(c), "lens": lens}


def test_varlen_128k_dense_sparse_switch():
    w = gen.WORKLOADS["varlen_128k"]
    data = gen.make_prefill(w)
    dense_ids = [s for s, n in enumerate(data["lens"]) if O.dense_route(n)]
    sparse_ids = [s for s, n in enumerate(data["lens"]) if not O.dense_route(n)]
    assert dense_ids and sparse_ids
    op = H.oracle_params(w)
    errs = []
    # dense side
    dd = _sub(data, dense_ids)
    run = H.DeviceRun(dd, w)
    run.dense()
    torch.cuda.synchronize()
    rows = gen.sample_rows(run.vl.total, 40, seed=3)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    seqs = H.oracle_sequences(dd, w, which=sorted(set(int(s) for s in sidx)))
    out = run.out.float().cpu().numpy()
    for r, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            ref = seqs[int(s)].dense_out(int(t), g)
            errs.append(np.abs(out[r, g * w.group:(g + 1) * w.group] - ref).ravel())
    # sparse side
    sd = _sub(data, sparse_ids)
    run = H.DeviceRun(sd, w)
    run.compress(); run.scores(); run.topk()
    torch.cuda.synchronize()
    rows = gen.sample_rows(run.vl.total, 40, seed=4)
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    seqs = H.oracle_sequences(sd, w, which=sorted(set(int(s) for s in sidx)))
    idx_all = np.stack([H.default_index_rows(run.lens, w) for _ in range(w.h_kv)])
    gpu_idx = run.idx.cpu().numpy()
    lists, S_rows, ts = [], [], []
    for r, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            S = seqs[int(s)].shared_scores(int(t), g)
            idx_all[g, r] = O.select_blocks(S, int(t), op)
            lists.append(gpu_idx[g, r])
            S_rows.append(S)
            ts.append(int(t))
    exact, tie, bad = H.compare_lists(lists, S_rows, ts, op)
    print(f"[varlen_128k] selection: {exact} rows bit-exact, {tie} near-tie rows valid")
    assert bad == 0 and exact >= 0.8 * (exact + tie), (bad, exact, tie)
    run.sparse(torch.from_numpy(idx_all).cuda())
    torch.cuda.synchronize()
    out = run.out.float().cpu().numpy()
    for r, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            ref = seqs[int(s)].sparse_out(int(t), g, idx_all[g, r])
            errs.append(np.abs(out[r, g * w.group:(g + 1) * w.group] - ref).ravel())
    e = np.concatenate(errs)
    assert e.max() <= H.ATT_MAX_ABS and e.mean() <= H.ATT_MEAN_ABS, (e.max(), e.mean())
    assert T.infllm2_get_device_status() == 0
