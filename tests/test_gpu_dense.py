"""GPU parity of the dense causal path (the short-sequence side of the
dense/sparse switch) against the fp64 oracle."""
import dataclasses

import numpy as np
import pytest
import torch

from inputs import gen
from oracle import infllm2_oracle as O
from tests import harness as H

pytestmark = pytest.mark.gpu


def _dense_case(w, lens, seed, rows=None):
    data = gen.make_prefill(w, lens=lens, seed=seed)
    run = H.DeviceRun(data, w)
    run.dense()
    torch.cuda.synchronize()
    total = run.vl.total
    rows = np.arange(total) if rows is None else rows
    sidx, tloc = H.seq_of_rows(run.lens, rows)
    seqs = H.oracle_sequences(data, w, which=sorted(set(int(s) for s in sidx)))
    out = run.out.float().cpu().numpy()
    errs = []
    for row, s, t in zip(rows, sidx, tloc):
        for g in range(w.h_kv):
            ref = seqs[int(s)].dense_out(int(t), g)
            errs.append(np.abs(out[int(row), g * w.group:(g + 1) * w.group] - ref).ravel())
    e = np.concatenate(errs)
    assert e.max() <= H.ATT_MAX_ABS and e.mean() <= H.ATT_MEAN_ABS, (e.max(), e.mean())
    import trainable_block_sparse_pool_b200 as T
    assert T.infllm2_get_device_status() == 0


def test_dense_tiny_1k_full():
    w = gen.WORKLOADS["tiny_1k"]
    _dense_case(w, [w.seqlen], w.seed)


def test_dense_varlen_d128_g16():
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="dense_small", seed=21)
    _dense_case(w, [1, 77, 128, 129, 700, 1500], 21)


def test_dense_varlen_d64_g4():
    w = dataclasses.replace(gen.WORKLOADS["tiny_1k"], name="dense_tiny", seed=22)
    _dense_case(w, [5, 300, 1000, 2049], 22)


def test_dense_8k_sampled():
    # the longest sequences the switch sends to the dense path
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="dense_8k", seed=23)
    rows = gen.sample_rows(2 * 8192 + 4000, 96, seed=5)
    _dense_case(w, [8192, 4000, 8192], 23, rows=rows)


def test_sparse_equals_dense_when_every_block_is_selected():
    # |I| >= causal blocks: the sparse kernel must reproduce the dense one
    w = dataclasses.replace(gen.WORKLOADS["tiny_1k"], name="all_blocks", n_local=16, top_k=2, seed=24)
    data = gen.make_prefill(w, lens=[1024], seed=24)
    run = H.DeviceRun(data, w)
    run.compress(); run.scores(); run.topk(); run.sparse()
    sparse_out = run.out.clone()
    run.dense()
    torch.cuda.synchronize()
    d = (sparse_out - run.out).abs()
    # both kernels round P to bf16 (against different reference maxima), so
    # they agree to the attention tolerance, not bit for bit
    assert d.max().item() <= H.ATT_MAX_ABS and d.mean().item() <= H.ATT_MEAN_ABS, (d.max().item(), d.mean().item())
