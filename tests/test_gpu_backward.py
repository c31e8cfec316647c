"""GPU parity of the backward of the block-sparse attention (dQ, dK, dV over
a fixed selection) against the fp64 oracle's chain rule
(oracle.sparse_attention_backward / one_block_gradients), on the GPU's own
block lists.  Forward and backward both run through the C ABI.

Tolerance.  The kernels take bf16 Q, K, V, dO (exact inputs to both sides)
and the bf16 forward output; they round P and dS to bf16 (unit roundoff
2^-9) before the gradient contractions and accumulate in fp32.  Each
gradient element is a sum of such terms, so its error is bounded by about
2^-8 of the sum of the terms' magnitudes; against the gradient's own scale
this is checked as max |err| <= 1e-2 * max |ref| and mean |err| <= 1e-2 *
mean |ref|, per tensor."""
import dataclasses

import numpy as np
import pytest
import torch

from inputs import gen
from oracle import infllm2_oracle as O
from tests import harness as H
import trainable_block_sparse_pool_b200 as T

pytestmark = pytest.mark.gpu

REL_MAX = 1e-2
REL_MEAN = 1e-2


def _forward_backward(w, data, seed):
    run = H.DeviceRun(data, w)
    run.compress()
    run.scores()
    run.topk()
    run.sparse()
    total = run.vl.total
    lse = run.sws[: total * w.h_q * 4].view(torch.float32).view(total, w.h_q).clone()
    dout = gen.make_grad_out(total, w.h_q, w.d, seed).cuda()
    ws = torch.empty(T.infllm2_sparse_backward_workspace_bytes(run.vl, w.h_q, w.h_kv, run.p), dtype=torch.uint8,
                     device="cuda")
    dQ = torch.full((total, w.h_q, w.d), float("nan"), dtype=torch.float32, device="cuda")
    dK = torch.full((total, w.h_kv, w.d), float("nan"), dtype=torch.float32, device="cuda")
    dV = torch.full_like(dK, float("nan"))
    T.infllm2_sparse_attn_backward(run.Q, run.K, run.V, run.out, dout, lse, run.idx, run.vl, dQ, dK, dV, ws, run.p)
    torch.cuda.synchronize()
    assert T.infllm2_get_device_status() == 0
    return run, dout, dQ, dK, dV, ws


def _rel(got, ref):
    e = np.abs(got - ref)
    return float(e.max() / max(np.abs(ref).max(), 1e-30)), float(e.mean() / max(np.abs(ref).mean(), 1e-30))


def _full_case(w, lens, seed):
    data = gen.make_prefill(w, lens=lens, seed=seed)
    run, dout, dQ, dK, dV, _ = _forward_backward(w, data, seed + 100)
    p = H.oracle_params(w)
    cu = data["cu_seqlens"].tolist()
    idx = run.idx.cpu().numpy()
    got = {"dQ": dQ.cpu().numpy(), "dK": dK.cpu().numpy(), "dV": dV.cpu().numpy()}
    ref = {k: np.zeros_like(v, dtype=np.float64) for k, v in got.items()}
    dO = O.to_f64(dout.cpu())
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        blocks = np.transpose(idx[:, a:b, :], (1, 0, 2)).astype(np.int64)
        q, k, v = (O.to_f64(data[x][a:b]) for x in ("Q", "K", "V"))
        ref["dQ"][a:b], ref["dK"][a:b], ref["dV"][a:b] = O.sparse_attention_backward(q, k, v, blocks, dO[a:b], p)
    for name in ("dQ", "dK", "dV"):
        assert np.isfinite(got[name]).all(), name
        rmax, rmean = _rel(got[name], ref[name])
        print(f"[{w.name}] {name}: max err / max |ref| = {rmax:.2e}, mean err / mean |ref| = {rmean:.2e}")
        assert rmax <= REL_MAX and rmean <= REL_MEAN, (name, rmax, rmean)


def test_backward_varlen_d128_g16():
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="bwd_varlen", n_local=4, top_k=6, seed=51)
    _full_case(w, [1000, 1057, 1, 200, 64, 3000, 129], 51)


def test_backward_varlen_d64_g8():
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="bwd_g8_d64", h_q=16, h_kv=2, d=64, n_local=4, top_k=6,
                            seed=52)
    _full_case(w, [700, 2100, 65], 52)


def test_backward_32k_sampled():
    # the bench's head shape and |I| = 96 at 32K: dQ at sampled rows, dK / dV
    # of a block in the middle (local and top-k rows) and of the last,
    # partial-causal block
    w = gen.WORKLOADS["prefill_32k"]
    data = gen.make_prefill(w)
    run, dout, dQ, dK, dV, _ = _forward_backward(w, data, 53)
    p = H.oracle_params(w)
    idx = run.idx.cpu().numpy()
    blocks = np.transpose(idx, (1, 0, 2)).astype(np.int64)
    seq = H.oracle_sequences(data, w)[0]
    dO = O.to_f64(dout.cpu())
    rows = gen.sample_rows(run.vl.total, 48, seed=54)
    got_q = dQ[torch.from_numpy(rows).cuda()].cpu().numpy()
    ref_q = np.zeros_like(got_q, dtype=np.float64)
    G = w.group
    for k, t in enumerate(rows):
        for g in range(w.h_kv):
            keys = O.sparse_keys(int(t), blocks[t, g], p.block)
            hs = slice(g * G, (g + 1) * G)
            ref_q[k, hs] = O.attend_backward(seq.Q[t, hs], seq.K[:, g], seq.V[:, g], keys, dO[t, hs],
                                             seq.scale)[0]
    rmax, rmean = _rel(got_q, ref_q)
    print(f"[prefill_32k] dQ (48 rows): {rmax:.2e}, {rmean:.2e}")
    assert rmax <= REL_MAX and rmean <= REL_MEAN
    gk, gv = dK.cpu().numpy(), dV.cpu().numpy()
    for g, kb in ((0, 250), (1, 511)):
        dk, dv = O.one_block_gradients(seq.Q, seq.K, seq.V, blocks, dO, p, g, kb)
        lo = 64 * kb
        for name, got, ref in (("dK", gk[lo:lo + 64, g], dk), ("dV", gv[lo:lo + 64, g], dv)):
            rmax, rmean = _rel(got, ref)
            print(f"[prefill_32k] {name} block {kb} group {g}: {rmax:.2e}, {rmean:.2e}")
            assert rmax <= REL_MAX and rmean <= REL_MEAN, (name, kb, rmax, rmean)


def test_backward_is_deterministic():
    w = dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="bwd_det", n_local=4, top_k=6, seed=55)
    data = gen.make_prefill(w, lens=[3000, 500], seed=55)
    outs = []
    for _ in range(2):
        _, _, dQ, dK, dV, _ = _forward_backward(w, data, 56)
        outs.append((dQ.cpu(), dK.cpu(), dV.cpu()))
    for x, y in zip(*outs):
        assert torch.equal(x, y)
