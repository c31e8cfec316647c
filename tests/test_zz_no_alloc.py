"""The allocation-free block selection (infllm2_select_blocks_noalloc) is for
callers that cannot allocate device memory when they select blocks: it keeps
S_shared in a fixed array inside the library instead of a caller-allocated
workspace.  It must pick exactly the blocks that infllm2_select_blocks
picks, on two calls in a row (the second call reuses the array the first one
left behind), and refuse problems larger than the array before launching.

This file is collected last so that a stop at the first failure has already
run every other test."""
import ctypes
import dataclasses

import pytest
import torch

from inputs import gen
from tests import harness as H
import trainable_block_sparse_pool_b200 as T


def _entry():
    L = T.lib()
    f = L.infllm2_select_blocks_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(T.Varlen), ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(T.Params), ctypes.c_void_p]
    return f


def test_noalloc_refuses_oversize_problems():
    f = _entry()
    vl = T.Varlen()
    vl.cu_seqlens = 0x1000
    vl.batch, vl.max_seqlen, vl.total = 1, 131072, 131072
    vl.total_c1, vl.total_c2 = 8191, 2047
    p = T.default_params()
    rc = f(0x1000, 0x1000, 0x1000, ctypes.byref(vl), 32, 2, 128, 0x1000, ctypes.byref(p), None)
    assert rc == -3


CASES = [
    (gen.WORKLOADS["tiny_1k"], [1024], 1000),
    (dataclasses.replace(gen.WORKLOADS["prefill_32k"], name="noalloc_varlen", n_local=4, top_k=6), [1000, 3000, 77],
     31),
]


@pytest.mark.gpu
@pytest.mark.parametrize("w,lens,seed", CASES)
def test_noalloc_matches_workspace_entry_point(w, lens, seed):
    f = _entry()
    data = gen.make_prefill(w, lens=lens, seed=seed)
    run = H.DeviceRun(data, w)
    run.compress()
    ws = torch.empty(T.infllm2_select_workspace_bytes(run.vl, w.h_kv, run.p), dtype=torch.uint8, device="cuda")
    T.infllm2_select_blocks(run.Q, run.Kc1, run.Kc2, run.vl, w.h_kv, ws, run.idx, None, run.p)
    ref = run.idx.clone()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        got = torch.full_like(ref, -7)
        rc = f(run.Q.data_ptr(), run.Kc1.data_ptr(), run.Kc2.data_ptr(), ctypes.byref(run.vl), w.h_q, w.h_kv, w.d,
               got.data_ptr(), ctypes.byref(run.p), stream)
        assert rc == 0, T.lib().infllm2_status_string(rc)
        torch.cuda.synchronize()
        # block indices are integers: the tolerance is exact equality
        assert torch.equal(got, ref)
    assert T.infllm2_get_device_status() == 0
