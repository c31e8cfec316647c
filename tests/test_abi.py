"""The C-ABI library builds, loads without a GPU, exports every entry
point that include/*.h declare, and rejects bad arguments on the host
before launching anything."""
import ctypes
import os
import re

import pytest

import trainable_block_sparse_pool_b200 as T
from trainable_block_sparse_pool_b200 import build as B

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADERS = [os.path.join(INCLUDE, f) for f in sorted(os.listdir(INCLUDE)) if f.endswith(".h")]


@pytest.fixture(scope="module")
def L():
    B.build()
    return T.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(infllm2_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n


def test_defaults_follow_the_pages(L):
    p = T.default_params()
    assert (p.block_size, p.c1_len, p.c1_stride, p.c2_len, p.c2_stride) == (64, 32, 16, 128, 64)
    assert (p.pool_len, p.pool_stride, p.pool_pad) == (5, 4, 1)
    assert (p.n_init, p.n_local, p.top_k, p.n_sel) == (1, 32, 63, 96)
    assert p.dense_threshold == 8192


def test_window_count_and_ld(L):
    assert T.window_count(1024, 32, 16) == 63
    assert T.window_count(1024, 128, 64) == 15
    assert T.window_count(31, 32, 16) == 0
    vl = T.Varlen()
    vl.max_seqlen = 131072
    assert T.infllm2_scores_ld(vl) == 8192      # 8191 windows rounded up to a multiple of 4
    # pooled pairs: 2 * ceil(8191 / 4) = 4096, already a multiple of 4
    assert T.infllm2_pooled_ld(vl) == 4096
    vl.max_seqlen = 1024                        # 63 windows: 16 groups, 32 floats
    assert T.infllm2_pooled_ld(vl) == 32
    vl.max_seqlen = 100                         # 5 windows: 2 groups, 4 floats
    assert T.infllm2_pooled_ld(vl) == 4


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert L.infllm2_status_string(code)


def _vl(batch=1, max_seqlen=1024, total=1024):
    vl = T.Varlen()
    vl.cu_seqlens = 0x1000
    vl.batch, vl.max_seqlen, vl.total = batch, max_seqlen, total
    vl.total_c1, vl.total_c2 = 63, 15
    return vl


def test_argument_errors_are_caught_on_host(L):
    p = T.default_params()
    vl = _vl()
    by = ctypes.byref
    # null pointers
    assert L.infllm2_compress_k(None, by(vl), 1, 64, 0x1000, 0x1000, by(p), None) == -1
    # misaligned pointer
    assert L.infllm2_compress_k(0x1008, by(vl), 1, 64, 0x1000, 0x1000, by(p), None) == -1
    # unsupported head dim and group size
    assert L.infllm2_shared_scores(0x1000, 0x1000, 0x1000, by(vl), 4, 1, 96, 0x1000, 64, by(p), None) == -2
    assert L.infllm2_shared_scores(0x1000, 0x1000, 0x1000, by(vl), 6, 2, 64, 0x1000, 64, by(p), None) == -2
    assert L.infllm2_shared_scores(0x1000, 0x1000, 0x1000, by(vl), 5, 2, 64, 0x1000, 64, by(p), None) == -1
    # ld too small
    assert L.infllm2_shared_scores(0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 60, by(p), None) == -1
    # the pooled pairs' ld is checked against infllm2_pooled_ld (32 floats here) and must be a multiple of 4
    assert L.infllm2_pooled_scores(0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 28, by(p), None) == -1
    assert L.infllm2_pooled_scores(0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 34, by(p), None) == -1
    assert L.infllm2_topk_blocks_pooled(0x1000, 28, by(vl), 1, 0x1000, by(p), None) == -1
    assert L.infllm2_topk_blocks_pooled(None, 32, by(vl), 1, 0x1000, by(p), None) == -1
    # unsupported pooling geometry
    q = T.default_params(c1_len=48)
    assert L.infllm2_topk_blocks(0x1000, 64, by(vl), 1, 0x1000, by(q), None) == -2
    q = T.default_params(n_local=0)
    assert L.infllm2_topk_blocks(0x1000, 64, by(vl), 1, 0x1000, by(q), None) == -1
    # workspace too small
    assert L.infllm2_select_blocks(0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 16, 0x1000, None, by(p),
                                   None) == -3
    # bad output dtype
    ws = T.infllm2_sparse_workspace_bytes(vl, 4)
    assert L.infllm2_sparse_attn(0x1000, 0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 7, 0x1000, ws, by(p),
                                 None) == -1
    # sparse workspace missing, misaligned or too small
    assert L.infllm2_sparse_attn(0x1000, 0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 0, None, ws, by(p),
                                 None) == -1
    assert L.infllm2_sparse_attn(0x1000, 0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 0, 0x1008, ws, by(p),
                                 None) == -1
    assert L.infllm2_sparse_attn(0x1000, 0x1000, 0x1000, 0x1000, by(vl), 4, 1, 64, 0x1000, 0, 0x1000, ws - 4, by(p),
                                 None) == -3
    # inconsistent varlen
    bad = _vl(batch=0)
    assert L.infllm2_dense_attn(0x1000, 0x1000, 0x1000, by(bad), 4, 1, 64, 0x1000, 0, by(p), None) == -1
    bad = _vl(max_seqlen=2048, total=1024)
    assert L.infllm2_dense_attn(0x1000, 0x1000, 0x1000, by(bad), 4, 1, 64, 0x1000, 0, by(p), None) == -1
    assert L.infllm2_debug_wait_timeout(0, None) == -1


def test_workspace_size(L):
    vl = _vl(max_seqlen=131072, total=131072)
    assert T.infllm2_select_workspace_bytes(vl, 2) == 2 * 131072 * 8192 * 4
    # one fp32 log-sum-exp per (token, query head)
    assert T.infllm2_sparse_workspace_bytes(vl, 32) == 131072 * 32 * 4


def _decode_state(batch, capacity, h_q=32, h_kv=2, d=128):
    st = T.DecodeState()
    st.k_cache = st.v_cache = st.k_c1 = st.k_c2 = st.seq_len = 0x1000
    st.batch, st.capacity, st.h_q, st.h_kv, st.d = batch, capacity, h_q, h_kv, d
    return st


def test_decode_plan_limits(L):
    # the host-side decode plan: supported shapes get a workspace, the
    # documented limits (candidate keys of one selection in shared memory;
    # batch * h_kv and pieces in 16 bits) and the exact LSE give 0
    p = T.default_params()
    by = ctypes.byref
    ws = L.infllm2_decode_workspace_bytes(by(_decode_state(16, 131072 + 64)), by(p))
    assert ws > 0 and ws % 256 == 0
    # at least, per (b, g): the block scores of 2049 blocks and the 96-entry block list
    assert ws >= 32 * (2049 * 4 + 96 * 4)
    assert L.infllm2_decode_workspace_bytes(by(_decode_state(1, 1441792)), by(p)) > 0
    assert L.infllm2_decode_workspace_bytes(by(_decode_state(1, 1441792 + 64)), by(p)) == 0
    assert L.infllm2_decode_workspace_bytes(by(_decode_state(32767, 4096)), by(p)) > 0
    assert L.infllm2_decode_workspace_bytes(by(_decode_state(32768, 4096)), by(p)) == 0   # 65536 (b, g) pairs
    q = T.default_params(lse_mode=T.LSE_EXACT)
    assert L.infllm2_decode_workspace_bytes(by(_decode_state(16, 131072 + 64)), by(q)) == 0
    # a step with too small a workspace is refused on the host
    st = _decode_state(16, 131072 + 64)
    assert L.infllm2_decode_step(by(st), 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, ws - 256, by(p), None) == -3
