"""GPU parity of the decode step (append, incremental pooled caches, one-row
selection and sparse attention) against the oracle's decode row, which is the
pinned prefill rule applied to the sequence extended by the new token."""
import dataclasses

import numpy as np
import pytest
import torch

from inputs import gen
from oracle import infllm2_oracle as O
from tests import harness as H
import trainable_block_sparse_pool_b200 as T

pytestmark = pytest.mark.gpu


class DecodeRun:
    def __init__(self, w, prefix, steps, batch):
        self.w = w
        self.data = gen.make_decode(w, prefix=prefix, steps=steps, batch=batch)
        self.p = H.lib_params(w)
        dev = torch.device("cuda")
        cap = prefix + steps
        self.k_cache = torch.zeros(batch, cap, w.h_kv, w.d, dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.zeros_like(self.k_cache)
        self.k_cache[:, :prefix] = self.data["K"][:, :prefix].to(dev)
        self.v_cache[:, :prefix] = self.data["V"][:, :prefix].to(dev)
        # rows past the prefix are not written yet: NaN there must never
        # reach an output (they are appended one per step)
        self.k_cache[:, prefix:] = float("nan")
        self.v_cache[:, prefix:] = float("nan")
        self.kc1 = torch.zeros(batch, w.h_kv, max(1, T.window_count(cap, 32, 16)), w.d, dtype=torch.bfloat16, device=dev)
        self.kc2 = torch.zeros(batch, w.h_kv, max(1, T.window_count(cap, 128, 64)), w.d, dtype=torch.bfloat16, device=dev)
        self.seq_len = torch.full((batch,), prefix, dtype=torch.int32, device=dev)
        self.st = T.make_decode_state(self.k_cache, self.v_cache, self.kc1, self.kc2, self.seq_len, w.h_q)
        self.ws = torch.empty(T.infllm2_decode_workspace_bytes(self.st, self.p), dtype=torch.uint8, device=dev)
        self.out = torch.empty(batch, w.h_q, w.d, dtype=torch.bfloat16, device=dev)
        self.prefix, self.steps, self.batch = prefix, steps, batch
        T.infllm2_decode_build_caches(self.st, self.p)

    def step(self, i):
        dev = torch.device("cuda")
        t = self.prefix + i
        q = self.data["q_steps"][i].to(dev)
        kn = self.data["K"][:, t].contiguous().to(dev)
        vn = self.data["V"][:, t].contiguous().to(dev)
        T.infllm2_decode_step(self.st, q, kn, vn, self.out, self.ws, self.p)


def _check_step(run, i, seqs, op, tally):
    """Row t = prefix + i of every listed sequence against the oracle's decode
    row: the block lists the step selected (read from the decode workspace)
    bit-exact where the top-k gap exceeds 1e-4, valid elsewhere; and the
    output against the oracle's attention over the GPU's own list (the same
    list as the oracle's wherever the lists are compared exactly)."""
    torch.cuda.synchronize()
    out = run.out.float().cpu().numpy()
    lists = T.infllm2_decode_block_lists(run.st, run.ws, run.p).cpu().numpy()
    t = run.prefix + i
    errs = []
    G = run.w.group
    for b in seqs:
        K = O.to_f64(run.data["K"][b, :t + 1])
        V = O.to_f64(run.data["V"][b, :t + 1])
        q = O.to_f64(run.data["q_steps"][i, b])
        sel, ref, scores, _, _ = O.decode_row(K, V, q, op)
        exact, tie, bad = H.compare_lists(lists[b], scores, [t] * run.w.h_kv, op)
        assert bad == 0, (b, t, lists[b], sel)
        tally["exact"] += exact
        tally["tie"] += tie
        for g in range(run.w.h_kv):
            keys = O.sparse_keys(t, lists[b, g], op.block)
            want = O.attend(q[g * G:(g + 1) * G], K[:, g], V[:, g], t, keys, op.softmax_scale(run.w.d))
            if np.array_equal(lists[b, g], sel[g]):
                np.testing.assert_allclose(want, ref[g * G:(g + 1) * G], rtol=0, atol=1e-12)
            errs.append(np.abs(out[b, g * G:(g + 1) * G] - want).ravel())
    return errs


def _run_case(w, prefix, steps, batch, check_every=1, seqs=None, min_exact=0.85):
    run = DecodeRun(w, prefix, steps, batch)
    op = H.oracle_params(w)
    seqs = list(range(batch)) if seqs is None else seqs
    errs, tally = [], {"exact": 0, "tie": 0}
    for i in range(steps):
        run.step(i)
        if i % check_every == 0 or i == steps - 1:
            errs += _check_step(run, i, seqs, op, tally)
    print(f"[{w.name}] decode selection: {tally['exact']} rows bit-exact, {tally['tie']} near-tie rows valid")
    assert tally["exact"] >= min_exact * (tally["exact"] + tally["tie"]), tally
    e = np.concatenate(errs)
    assert e.max() <= H.ATT_MAX_ABS and e.mean() <= H.ATT_MEAN_ABS, (e.max(), e.mean())
    # the pooled caches after the steps equal the oracle's pooling of the whole sequence
    torch.cuda.synchronize()
    assert run.seq_len.cpu().tolist() == [prefix + steps] * batch
    n = prefix + steps
    for b in seqs:
        K = O.to_f64(run.data["K"][b, :n])
        c1 = O.pool_keys(K, 32, 16)
        c2 = O.pool_keys(K, 128, 64)
        np.testing.assert_array_equal(run.kc1[b, :, :c1.shape[1]].float().cpu().numpy(), c1)
        np.testing.assert_array_equal(run.kc2[b, :, :c2.shape[1]].float().cpu().numpy(), c2)
    assert T.infllm2_get_device_status() == 0


def test_decode_small_d128_g16():
    # prefixes straddle the interesting boundaries: no coarse window yet,
    # fewer candidates than top_k, and a full selection
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="decode_small", n_local=4, top_k=6, seed=41)
    _run_case(w, prefix=100, steps=70, batch=1)
    _run_case(dataclasses.replace(w, seed=42), prefix=1500, steps=40, batch=3)


def test_decode_tiny_d64_g4():
    w = dataclasses.replace(gen.WORKLOADS["tiny_1k"], name="decode_tiny", seed=43)
    _run_case(w, prefix=900, steps=130, batch=2, check_every=3)


def test_decode_group_sizes():
    # G = 1 (d = 128) and G = 8 (d = 64): the remaining group sizes of the decode kernels
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="decode_g1", h_q=2, h_kv=2, n_local=4, top_k=6, seed=44)
    _run_case(w, prefix=1200, steps=20, batch=2, check_every=4)
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="decode_g8", h_q=16, h_kv=2, d=64, n_local=4, top_k=6,
                            seed=45)
    _run_case(w, prefix=2000, steps=20, batch=2, check_every=4)


def test_decode_many_groups():
    # 120 sequences x 4 groups: more (sequence, group) pairs than score CTAs in
    # one wave, so the score kernel cuts the flattened piece list into ranges
    # that cross from one group into the next
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="decode_many", h_q=16, h_kv=4, d=64, seed=46)
    _run_case(w, prefix=7000, steps=3, batch=120, check_every=2, seqs=[0, 57, 119])


def test_decode_16x128k_sampled():
    # the benchmark's decode workload: 16 sequences x 131072-token cache;
    # the oracle checks two sequences on the first and a later step
    w = gen.WORKLOADS["decode_16x128k"]
    run = DecodeRun(w, prefix=w.seqlen, steps=4, batch=w.batch)
    op = H.oracle_params(w)
    errs, tally = [], {"exact": 0, "tie": 0}
    for i in range(4):
        run.step(i)
        if i in (0, 3):
            errs += _check_step(run, i, [0, 5, 11, 15], op, tally)
    print(f"[{w.name}] decode selection: {tally['exact']} rows bit-exact, {tally['tie']} near-tie rows valid")
    assert tally["exact"] >= 0.6 * (tally["exact"] + tally["tie"]), tally
    e = np.concatenate(errs)
    assert e.max() <= H.ATT_MAX_ABS and e.mean() <= H.ATT_MEAN_ABS, (e.max(), e.mean())
    assert T.infllm2_get_device_status() == 0


def test_decode_more_than_256_sequences():
    # 300 short sequences: the score kernel counts the pieces of the batch in
    # chunks of 256 sequences, so sequences on both sides of the chunk
    # boundary (255, 256) and the last one are checked
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="decode_300", h_q=8, h_kv=2, d=64, n_local=4, top_k=6,
                            seed=47)
    _run_case(w, prefix=1500, steps=2, batch=300, check_every=1, seqs=[0, 128, 254, 255, 256, 257, 299])
