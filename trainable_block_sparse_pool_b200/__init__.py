"""Python binding of libinfllm2 (InfLLM-V2 sparse-attention forward path for
GQA on sm_100a).

Argument marshalling only: every function below forwards torch tensors'
device pointers and the current CUDA stream to the C ABI declared in
``include/infllm2.h`` and raises :class:`InfLLM2Error` on a non-zero status.
All arithmetic happens in the CUDA library; there is no fallback path.  If
the shared library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

from . import build as _build

__all__ = [
    "InfLLM2Error", "Params", "Varlen", "lib", "default_params", "make_varlen", "window_count",
    "infllm2_compress_k", "infllm2_shared_scores", "infllm2_topk_blocks", "infllm2_select_blocks",
    "infllm2_pooled_ld", "infllm2_pooled_scores", "infllm2_topk_blocks_pooled",
    "infllm2_select_workspace_bytes", "infllm2_scores_ld", "infllm2_sparse_workspace_bytes", "infllm2_sparse_attn",
    "infllm2_dense_attn",
    "infllm2_get_device_status", "infllm2_clear_device_status", "infllm2_debug_wait_timeout",
    "infllm2_probe_l2_gather",
    "DecodeState", "make_decode_state", "infllm2_decode_workspace_bytes", "infllm2_decode_build_caches",
    "infllm2_decode_step", "OUT_BF16", "OUT_F32", "LSE_APPROX", "LSE_EXACT",
]

LSE_APPROX = 0
LSE_EXACT = 1
OUT_BF16 = 0
OUT_F32 = 1


class InfLLM2Error(RuntimeError):
    pass


class Params(ctypes.Structure):
    _fields_ = [
        ("block_size", ctypes.c_int32), ("c1_len", ctypes.c_int32), ("c1_stride", ctypes.c_int32),
        ("c2_len", ctypes.c_int32), ("c2_stride", ctypes.c_int32), ("pool_len", ctypes.c_int32),
        ("pool_stride", ctypes.c_int32), ("pool_pad", ctypes.c_int32), ("n_init", ctypes.c_int32),
        ("n_local", ctypes.c_int32), ("top_k", ctypes.c_int32), ("scale", ctypes.c_float),
        ("lse_mode", ctypes.c_int32), ("dense_threshold", ctypes.c_int32),
    ]

    @property
    def n_sel(self) -> int:
        return self.n_init + self.n_local + self.top_k


class Varlen(ctypes.Structure):
    _fields_ = [
        ("cu_seqlens", ctypes.c_void_p), ("batch", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
        ("total", ctypes.c_int64), ("total_c1", ctypes.c_int64), ("total_c2", ctypes.c_int64),
    ]


class DecodeState(ctypes.Structure):
    _fields_ = [
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("k_c1", ctypes.c_void_p),
        ("k_c2", ctypes.c_void_p), ("seq_len", ctypes.c_void_p), ("batch", ctypes.c_int32),
        ("capacity", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_kv", ctypes.c_int32), ("d", ctypes.c_int32),
    ]


_LIB = None
_P = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load libinfllm2.so from the package directory (raises if absent)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = _build.LIB_PATH
    if not os.path.exists(path):
        raise InfLLM2Error(f"{path} is not built: run trainable_block_sparse_pool_b200.build.build()")
    L = ctypes.CDLL(path)
    pp, vp = ctypes.POINTER(Params), ctypes.POINTER(Varlen)
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    sig = {
        "infllm2_default_params": (Params, []),
        "infllm2_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "infllm2_window_count": (i64, [i64, i32, i32]),
        "infllm2_scores_ld": (i64, [vp, pp]),
        "infllm2_compress_k": (ctypes.c_int, [_P, vp, i32, i32, _P, _P, pp, _P]),
        "infllm2_shared_scores": (ctypes.c_int, [_P, _P, _P, vp, i32, i32, i32, _P, i64, pp, _P]),
        "infllm2_topk_blocks": (ctypes.c_int, [_P, i64, vp, i32, _P, pp, _P]),
        "infllm2_pooled_ld": (i64, [vp, pp]),
        "infllm2_pooled_scores": (ctypes.c_int, [_P, _P, _P, vp, i32, i32, i32, _P, i64, pp, _P]),
        "infllm2_topk_blocks_pooled": (ctypes.c_int, [_P, i64, vp, i32, _P, pp, _P]),
        "infllm2_select_workspace_bytes": (ctypes.c_size_t, [vp, i32, pp]),
        "infllm2_select_blocks": (ctypes.c_int, [_P, _P, _P, vp, i32, i32, i32, _P, ctypes.c_size_t, _P, _P, pp, _P]),
        "infllm2_sparse_workspace_bytes": (ctypes.c_size_t, [vp, i32]),
        "infllm2_sparse_attn": (ctypes.c_int, [_P, _P, _P, _P, vp, i32, i32, i32, _P, i32, _P, ctypes.c_size_t, pp,
                                                _P]),
        "infllm2_dense_attn": (ctypes.c_int, [_P, _P, _P, vp, i32, i32, i32, _P, i32, pp, _P]),
        "infllm2_sparse_backward_workspace_bytes": (ctypes.c_size_t, [vp, i32, i32, pp]),
        "infllm2_sparse_attn_backward": (ctypes.c_int, [_P, _P, _P, _P, i32, _P, _P, _P, vp, i32, i32, i32, _P, _P, _P,
                                                         _P, ctypes.c_size_t, pp, _P]),
        "infllm2_get_device_status": (ctypes.c_int, []),
        "infllm2_clear_device_status": (ctypes.c_int, []),
        "infllm2_debug_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, _P]),
        "infllm2_probe_l2_gather": (ctypes.c_int, [_P, _P, i64, i32, i32, i32, i32, _P]),
        "infllm2_decode_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(DecodeState), pp]),
        "infllm2_decode_block_idx_offset": (i64, [ctypes.POINTER(DecodeState), pp]),
        "infllm2_decode_build_caches": (ctypes.c_int, [ctypes.POINTER(DecodeState), pp, _P]),
        "infllm2_decode_step": (ctypes.c_int, [ctypes.POINTER(DecodeState), _P, _P, _P, _P, _P, ctypes.c_size_t, pp,
                                                _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _LIB = L
    return L


def _check(name: str, rc: int) -> None:
    if rc != 0:
        msg = lib().infllm2_status_string(rc).decode()
        raise InfLLM2Error(f"{name} failed ({rc}): {msg}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise InfLLM2Error("tensors passed to libinfllm2 must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def default_params(**overrides) -> Params:
    p = lib().infllm2_default_params()
    for k, v in overrides.items():
        setattr(p, k, v)
    return p


def window_count(n: int, length: int, stride: int) -> int:
    return int(lib().infllm2_window_count(n, length, stride))


def make_varlen(lens: Sequence[int], cu_seqlens: torch.Tensor, params: Optional[Params] = None) -> Varlen:
    """Varlen geometry from the host list of lengths and the device
    cu_seqlens tensor (int32, batch+1).  Keeps a reference to the tensor."""
    p = params or default_params()
    lens = [int(x) for x in lens]
    vl = Varlen()
    vl.cu_seqlens = cu_seqlens.data_ptr()
    vl.batch = len(lens)
    vl.max_seqlen = max(lens) if lens else 0
    vl.total = sum(lens)
    vl.total_c1 = sum(window_count(n, p.c1_len, p.c1_stride) for n in lens)
    vl.total_c2 = sum(window_count(n, p.c2_len, p.c2_stride) for n in lens)
    vl._keep = cu_seqlens  # noqa: SLF001  (keeps the device buffer alive)
    return vl


def infllm2_scores_ld(vl: Varlen, params: Optional[Params] = None) -> int:
    return int(lib().infllm2_scores_ld(ctypes.byref(vl), ctypes.byref(params or default_params())))


def infllm2_select_workspace_bytes(vl: Varlen, h_kv: int, params: Optional[Params] = None) -> int:
    return int(lib().infllm2_select_workspace_bytes(ctypes.byref(vl), h_kv, ctypes.byref(params or default_params())))


def infllm2_compress_k(K: torch.Tensor, vl: Varlen, K_c1: torch.Tensor, K_c2: torch.Tensor,
                       params: Optional[Params] = None, stream=None) -> None:
    h_kv, d = K.shape[1], K.shape[2]
    rc = lib().infllm2_compress_k(_ptr(K), ctypes.byref(vl), h_kv, d, _ptr(K_c1), _ptr(K_c2),
                                  ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_compress_k", rc)


def infllm2_shared_scores(Q: torch.Tensor, K_c1: torch.Tensor, K_c2: torch.Tensor, vl: Varlen, h_kv: int,
                          S: torch.Tensor, ld: int, params: Optional[Params] = None, stream=None) -> None:
    h_q, d = Q.shape[1], Q.shape[2]
    rc = lib().infllm2_shared_scores(_ptr(Q), _ptr(K_c1), _ptr(K_c2), ctypes.byref(vl), h_q, h_kv, d, _ptr(S), ld,
                                     ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_shared_scores", rc)


def infllm2_topk_blocks(S: torch.Tensor, ld: int, vl: Varlen, h_kv: int, block_idx: torch.Tensor,
                        params: Optional[Params] = None, stream=None) -> None:
    rc = lib().infllm2_topk_blocks(_ptr(S), ld, ctypes.byref(vl), h_kv, _ptr(block_idx),
                                   ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_topk_blocks", rc)


def infllm2_pooled_ld(vl: Varlen, params: Optional[Params] = None) -> int:
    return int(lib().infllm2_pooled_ld(ctypes.byref(vl), ctypes.byref(params or default_params())))


def infllm2_pooled_scores(Q: torch.Tensor, K_c1: torch.Tensor, K_c2: torch.Tensor, vl: Varlen, h_kv: int,
                          P: torch.Tensor, ldp: int, params: Optional[Params] = None, stream=None) -> None:
    h_q, d = Q.shape[1], Q.shape[2]
    rc = lib().infllm2_pooled_scores(_ptr(Q), _ptr(K_c1), _ptr(K_c2), ctypes.byref(vl), h_q, h_kv, d, _ptr(P), ldp,
                                     ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_pooled_scores", rc)


def infllm2_topk_blocks_pooled(P: torch.Tensor, ldp: int, vl: Varlen, h_kv: int, block_idx: torch.Tensor,
                               params: Optional[Params] = None, stream=None) -> None:
    rc = lib().infllm2_topk_blocks_pooled(_ptr(P), ldp, ctypes.byref(vl), h_kv, _ptr(block_idx),
                                          ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_topk_blocks_pooled", rc)


def infllm2_select_blocks(Q: torch.Tensor, K_c1: torch.Tensor, K_c2: torch.Tensor, vl: Varlen, h_kv: int,
                          workspace: Optional[torch.Tensor], block_idx: torch.Tensor,
                          s_shared_out: Optional[torch.Tensor] = None, params: Optional[Params] = None,
                          stream=None) -> None:
    h_q, d = Q.shape[1], Q.shape[2]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib().infllm2_select_blocks(_ptr(Q), _ptr(K_c1), _ptr(K_c2), ctypes.byref(vl), h_q, h_kv, d,
                                     _ptr(workspace), ws_bytes, _ptr(block_idx), _ptr(s_shared_out),
                                     ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_select_blocks", rc)


def infllm2_sparse_workspace_bytes(vl: Varlen, h_q: int) -> int:
    return lib().infllm2_sparse_workspace_bytes(ctypes.byref(vl), h_q)


def infllm2_sparse_attn(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, block_idx: torch.Tensor, vl: Varlen,
                        out: torch.Tensor, params: Optional[Params] = None, stream=None,
                        workspace: Optional[torch.Tensor] = None) -> None:
    """`workspace`: a device byte tensor of at least infllm2_sparse_workspace_bytes(vl, h_q) bytes; one is
    allocated for the call when it is None."""
    h_q, d = Q.shape[1], Q.shape[2]
    h_kv = K.shape[1]
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    need = infllm2_sparse_workspace_bytes(vl, h_q)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=Q.device)
    rc = lib().infllm2_sparse_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(block_idx), ctypes.byref(vl), h_q, h_kv, d,
                                   _ptr(out), od, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_sparse_attn", rc)


def infllm2_sparse_backward_workspace_bytes(vl: Varlen, h_q: int, h_kv: int, params: Optional[Params] = None) -> int:
    return int(lib().infllm2_sparse_backward_workspace_bytes(ctypes.byref(vl), h_q, h_kv,
                                                             ctypes.byref(params or default_params())))


def infllm2_sparse_attn_backward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, out: torch.Tensor,
                                 dout: torch.Tensor, lse: torch.Tensor, block_idx: torch.Tensor, vl: Varlen,
                                 dQ: torch.Tensor, dK: torch.Tensor, dV: torch.Tensor, workspace: torch.Tensor,
                                 params: Optional[Params] = None, stream=None) -> None:
    """Gradients of the block-sparse attention (fp32 dQ, dK, dV).  `lse`: fp32 [total, h_q], the first
    total * h_q floats of the workspace infllm2_sparse_attn used."""
    h_q, d = Q.shape[1], Q.shape[2]
    h_kv = K.shape[1]
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    rc = lib().infllm2_sparse_attn_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(out), od, _ptr(dout), _ptr(lse),
                                            _ptr(block_idx), ctypes.byref(vl), h_q, h_kv, d, _ptr(dQ), _ptr(dK),
                                            _ptr(dV), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                            ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_sparse_attn_backward", rc)


def infllm2_probe_l2_gather(K: torch.Tensor, V: torch.Tensor, nblk: int, tiles: int, producers: int,
                            stream=None) -> None:
    """L2 gather bandwidth probe with the sparse attention's tile shape (K, V: [rows, h_kv, 128] bf16)."""
    rc = lib().infllm2_probe_l2_gather(_ptr(K), _ptr(V), K.shape[0], K.shape[1], nblk, tiles, producers,
                                       _stream(stream))
    _check("infllm2_probe_l2_gather", rc)


def infllm2_dense_attn(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, vl: Varlen, out: torch.Tensor,
                       params: Optional[Params] = None, stream=None) -> None:
    h_q, d = Q.shape[1], Q.shape[2]
    h_kv = K.shape[1]
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    rc = lib().infllm2_dense_attn(_ptr(Q), _ptr(K), _ptr(V), ctypes.byref(vl), h_q, h_kv, d, _ptr(out), od,
                                  ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_dense_attn", rc)


def infllm2_get_device_status() -> int:
    return int(lib().infllm2_get_device_status())


def infllm2_clear_device_status() -> None:
    _check("infllm2_clear_device_status", lib().infllm2_clear_device_status())


def infllm2_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    _check("infllm2_debug_wait_timeout", lib().infllm2_debug_wait_timeout(limit_ns, _stream(stream)))


def make_decode_state(k_cache: torch.Tensor, v_cache: torch.Tensor, k_c1: torch.Tensor, k_c2: torch.Tensor,
                      seq_len: torch.Tensor, h_q: int) -> DecodeState:
    """Decode state over caller-owned device tensors: caches [batch, capacity,
    h_kv, d], pooled caches [batch, h_kv, cap, d], seq_len int32 [batch]."""
    st = DecodeState()
    st.k_cache, st.v_cache = _ptr(k_cache), _ptr(v_cache)
    st.k_c1, st.k_c2, st.seq_len = _ptr(k_c1), _ptr(k_c2), _ptr(seq_len)
    st.batch, st.capacity, st.h_kv, st.d = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2], k_cache.shape[3]
    st.h_q = h_q
    st._keep = (k_cache, v_cache, k_c1, k_c2, seq_len)  # noqa: SLF001
    return st


def infllm2_decode_workspace_bytes(st: DecodeState, params: Optional[Params] = None) -> int:
    return int(lib().infllm2_decode_workspace_bytes(ctypes.byref(st), ctypes.byref(params or default_params())))


def infllm2_decode_block_lists(st: DecodeState, workspace: torch.Tensor, params: Optional[Params] = None) -> torch.Tensor:
    """View of the block lists the last decode step on `workspace` selected:
    int32 [batch, h_kv, n_sel], ascending, -1 padded (read after the step)."""
    params = params or default_params()
    off = int(lib().infllm2_decode_block_idx_offset(ctypes.byref(st), ctypes.byref(params)))
    if off < 0:
        raise InfLLM2Error("infllm2_decode_block_idx_offset: invalid or unsupported decode state")
    n = st.batch * st.h_kv * params.n_sel
    if off + 4 * n > workspace.numel() * workspace.element_size():
        raise InfLLM2Error("decode workspace smaller than its block lists")
    return workspace.view(torch.uint8)[off:off + 4 * n].view(torch.int32).view(st.batch, st.h_kv, params.n_sel)


def infllm2_decode_build_caches(st: DecodeState, params: Optional[Params] = None, stream=None) -> None:
    rc = lib().infllm2_decode_build_caches(ctypes.byref(st), ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_decode_build_caches", rc)


def infllm2_decode_step(st: DecodeState, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                        out: torch.Tensor, workspace: torch.Tensor, params: Optional[Params] = None,
                        stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib().infllm2_decode_step(ctypes.byref(st), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(workspace),
                                   ws_bytes, ctypes.byref(params or default_params()), _stream(stream))
    _check("infllm2_decode_step", rc)
