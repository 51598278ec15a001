"""ctypes binding of libkvc (include/kvc.h): argument marshalling only.

Every function here has the name of a C entry point, takes torch tensors for
device buffers and numpy/sequence objects for host arrays, passes their
addresses and the current CUDA stream through, and raises KvcError on a
non-zero status.  There is no Python or CPU implementation behind any of
them: if libkvc.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvc.so")

KVC_F32, KVC_BF16 = 0, 1
# kvc_status
KVC_OK, KVC_ERR_INVALID_ARG, KVC_ERR_UNSUPPORTED, KVC_ERR_WORKSPACE, KVC_ERR_CUDA, KVC_ERR_DEVICE_CHECK = range(6)

# entry points declared in include/kvc.h, with their ctypes signatures
_c_int, _c_i64, _c_u64, _c_sz, _c_f, _c_p = (ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t,
                                             ctypes.c_float, ctypes.c_void_p)
SIGNATURES = {
    "kvc_version": (_c_int, []),
    "kvc_launch_count": (_c_i64, []),
    "kvc_check_workspace": (_c_int, [_c_p, _c_p]),
    "kvc_status_string": (ctypes.c_char_p, [_c_int]),
    "kvc_last_error": (ctypes.c_char_p, []),
    "kvc_cache_bytes": (_c_u64, [_c_int, _c_i64, _c_int, _c_int, _c_int]),
    "kvc_budget_offsets": (_c_i64, [_c_int, _c_p, _c_int, _c_p]),
    "kvc_pyramid_budgets": (_c_i64, [_c_int, _c_int, _c_int, _c_p]),
    "kvc_score_window_workspace_size": (_c_sz, [_c_int, _c_int, _c_p, _c_int, _c_int, _c_int, _c_int]),
    "kvc_score_window": (_c_int, [_c_int, _c_int, _c_p, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_f,
                                  _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "kvc_compress_window": (_c_int, [_c_int, _c_int, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _c_int, _c_f, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz,
                                     _c_p]),
    "kvc_select_topk": (_c_int, [_c_int, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_p, _c_p, _c_p]),
    "kvc_gather_kv": (_c_int, [_c_int, _c_int, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_p, _c_p, _c_p,
                               _c_p, _c_p, _c_p]),
    "kvc_tsp_workspace_size": (_c_sz, [_c_int, _c_int]),
    "kvc_tsp_select_gather": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, _c_p, _c_int, _c_p,
                                       _c_p, _c_p, _c_sz, _c_p]),
    "kvc_tsp_select_gather_static": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, _c_p, _c_int,
                                              _c_p, _c_p, _c_p]),
    "kvc_gather_kv_q8": (_c_int, [_c_int, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_p, _c_p, _c_p, _c_p, _c_p,
                                  _c_p, _c_p, _c_i64, _c_p]),
    "kvc_gqa_decode_attn_q8": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_f, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i64,
                                        _c_i64, _c_p, _c_p, _c_int, _c_p, _c_p, _c_sz, _c_p]),
    "kvc_freekv_workspace_size": (_c_sz, [_c_int, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "kvc_freekv_step": (_c_int, [_c_int, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_f,
                                 _c_f, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "kvc_xkv_workspace_size": (_c_sz, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "kvc_xkv_factorize": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, _c_p, _c_int, _c_p, _c_p,
                                   _c_p, _c_sz, _c_p]),
    "kvc_xkv_reconstruct": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, _c_p,
                                     _c_p, _c_p, _c_p]),
    "kvc_gqa_decode_workspace_size": (_c_sz, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "kvc_gqa_decode_attn": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_f, _c_p, _c_p, _c_p, _c_i64, _c_p,
                                     _c_p, _c_int, _c_p, _c_p, _c_sz, _c_p]),
}

_lib = None


class KvcError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libkvc.so (once) and declare its prototypes."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m kv_cache_compression_score_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status: int) -> None:
    if status != 0:
        L = lib()
        raise KvcError(status, f"{L.kvc_status_string(status).decode()}: {L.kvc_last_error().decode()}")


def _dptr(t):
    """Device address of a torch tensor (None -> NULL)."""
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _host_i32(a):
    """(keep-alive array, address) of a host int32 array."""
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.int32))
    return arr, arr.ctypes.data_as(ctypes.c_void_p)


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(getattr(stream, "cuda_stream", stream))


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return KVC_F32
    if t.dtype == torch.bfloat16:
        return KVC_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ host side
def kvc_version() -> int:
    return lib().kvc_version()


def kvc_launch_count() -> int:
    """Kernels this library has enqueued in this process (graph captures count once)."""
    return int(lib().kvc_launch_count())


def kvc_check_workspace(ws, stream=None) -> int:
    """Status of a workspace's device error word after waiting for the stream:
    KVC_OK (0) or KVC_ERR_DEVICE_CHECK (5); other failures raise KvcError."""
    st = int(lib().kvc_check_workspace(_dptr(ws), _stream(stream)))
    if st not in (KVC_OK, KVC_ERR_DEVICE_CHECK):
        _check(st)
    return st


def kvc_cache_bytes(L: int, S: int, n_kv: int, d_h: int, b: int) -> int:
    return int(lib().kvc_cache_bytes(L, S, n_kv, d_h, b))


def kvc_budget_offsets(seqlens, budget: int) -> np.ndarray:
    sl, p = _host_i32(seqlens)
    out = np.zeros(len(sl) + 1, dtype=np.int32)
    total = lib().kvc_budget_offsets(len(sl), p, budget, out.ctypes.data_as(ctypes.c_void_p))
    if total < 0:
        raise KvcError(1, "kvc_budget_offsets: invalid input")
    return out


def kvc_pyramid_budgets(L: int, avg_budget: int, min_budget: int) -> np.ndarray:
    """Per-layer PyramidKV budgets (host helper of the library)."""
    out = np.zeros(max(L, 1), dtype=np.int32)
    total = lib().kvc_pyramid_budgets(L, avg_budget, min_budget, out.ctypes.data_as(ctypes.c_void_p))
    if total < 0:
        raise KvcError(1, "kvc_pyramid_budgets: invalid input")
    return out


def kvc_score_window_workspace_size(dt: int, seqlens, n_h: int, n_kv: int, d_h: int, w: int) -> int:
    sl, p = _host_i32(seqlens)
    return int(lib().kvc_score_window_workspace_size(dt, len(sl), p, n_h, n_kv, d_h, w))


def kvc_tsp_workspace_size(S: int, w: int) -> int:
    return int(lib().kvc_tsp_workspace_size(S, w))


def kvc_gqa_decode_workspace_size(batch: int, n_h: int, n_kv: int, d_h: int, max_kv_len: int) -> int:
    return int(lib().kvc_gqa_decode_workspace_size(batch, n_h, n_kv, d_h, max_kv_len))


# ---------------------------------------------------------------- device ops
def kvc_score_window(q_win, k, seqlens, cu_seqlens, n_h: int, n_kv: int, w: int, pool_k: int, scale: float,
                     scores, scores_raw, ws, stream=None) -> None:
    sl, p = _host_i32(seqlens)
    _check(lib().kvc_score_window(dtype_code(k), len(sl), p, _dptr(cu_seqlens), n_h, n_kv, k.shape[-1], w, pool_k,
                                  scale, _dptr(q_win), _dptr(k), _dptr(scores), _dptr(scores_raw), _dptr(ws),
                                  ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def kvc_compress_window(q_win, k, v, seqlens, cu_seqlens, cu_budget, n_h: int, n_kv: int, w: int, pool_k: int,
                        budget: int, scale: float, scores, scores_raw, idx, k_out, v_out, ws, stream=None) -> None:
    """Score, select and gather in one call (one launch where the fused path applies)."""
    sl, p = _host_i32(seqlens)
    _check(lib().kvc_compress_window(dtype_code(k), len(sl), p, _dptr(cu_seqlens), _dptr(cu_budget), n_h, n_kv,
                                     k.shape[-1], w, pool_k, budget, scale, _dptr(q_win), _dptr(k), _dptr(v),
                                     _dptr(scores), _dptr(scores_raw), _dptr(idx), _dptr(k_out), _dptr(v_out),
                                     _dptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def kvc_select_topk(seqlens, cu_seqlens, cu_budget, n_kv: int, w: int, budget: int, scores, idx,
                    stream=None) -> None:
    sl, p = _host_i32(seqlens)
    _check(lib().kvc_select_topk(len(sl), p, _dptr(cu_seqlens), _dptr(cu_budget), n_kv, w, budget, _dptr(scores),
                                 _dptr(idx), _stream(stream)))


def kvc_gather_kv(seqlens, cu_seqlens, cu_budget, budget: int, idx, k, v, k_out, v_out, stream=None) -> None:
    sl, p = _host_i32(seqlens)
    _check(lib().kvc_gather_kv(dtype_code(k), len(sl), p, _dptr(cu_seqlens), _dptr(cu_budget), k.shape[1],
                               k.shape[2], budget, _dptr(idx), _dptr(k), _dptr(v), _dptr(k_out), _dptr(v_out),
                               _stream(stream)))


def kvc_tsp_select_gather(scores_raw, w: int, pool_k: int, k_tsp: int, hidden, idx_out, hidden_out, ws,
                          stream=None) -> None:
    n_rows, S = scores_raw.shape
    _check(lib().kvc_tsp_select_gather(dtype_code(hidden), S, n_rows, w, pool_k, k_tsp, _dptr(scores_raw),
                                       _dptr(hidden), hidden.shape[1], _dptr(idx_out), _dptr(hidden_out), _dptr(ws),
                                       ws.numel() * ws.element_size(), _stream(stream)))


def kvc_tsp_select_gather_static(scores_raw, w: int, pool_k: int, k_tsp: int, hidden, idx_out, hidden_out,
                                 stream=None) -> None:
    """Token-selective propagation without a caller workspace (library-owned scratch)."""
    n_rows, S = scores_raw.shape
    _check(lib().kvc_tsp_select_gather_static(dtype_code(hidden), S, n_rows, w, pool_k, k_tsp, _dptr(scores_raw),
                                              _dptr(hidden), hidden.shape[1], _dptr(idx_out), _dptr(hidden_out),
                                              _stream(stream)))


def kvc_gqa_decode_attn(q, k_c, v_c, kv_row_offset, kv_len, max_kv_len: int, scale: float, out, ws,
                        stream=None) -> None:
    batch, n_h, d_h = q.shape
    _check(lib().kvc_gqa_decode_attn(dtype_code(q), batch, n_h, k_c.shape[1], d_h, scale, _dptr(q), _dptr(k_c),
                                     _dptr(v_c), k_c.shape[0], _dptr(kv_row_offset), _dptr(kv_len), max_kv_len,
                                     _dptr(out),
                                     _dptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def kvc_gather_kv_q8(seqlens, cu_seqlens, cu_budget, budget: int, idx, k, v, k_q, v_q, k_scale, v_scale,
                     stream=None) -> None:
    """Gather the retained rows of bf16 caches and quantise each (slot, head) vector to int8 + a float32 scale."""
    sl, p = _host_i32(seqlens)
    _check(lib().kvc_gather_kv_q8(len(sl), p, _dptr(cu_seqlens), _dptr(cu_budget), k.shape[1], k.shape[2], budget,
                                  _dptr(idx), _dptr(k), _dptr(v), _dptr(k_q), _dptr(v_q), _dptr(k_scale),
                                  _dptr(v_scale), k_scale.shape[1], _stream(stream)))


def kvc_gqa_decode_attn_q8(q, k_q, v_q, k_scale, v_scale, kv_row_offset, kv_len, max_kv_len: int, scale: float, out,
                           ws, stream=None) -> None:
    batch, n_h, d_h = q.shape
    _check(lib().kvc_gqa_decode_attn_q8(batch, n_h, k_q.shape[1], d_h, scale, _dptr(q), _dptr(k_q), _dptr(v_q),
                                        _dptr(k_scale), _dptr(v_scale), k_scale.shape[1], k_q.shape[0],
                                        _dptr(kv_row_offset), _dptr(kv_len), max_kv_len, _dptr(out), _dptr(ws),
                                        ws.numel() * ws.element_size(), _stream(stream)))


def kvc_freekv_workspace_size(seqlens, n_h: int, n_kv: int, d_h: int, w: int, budget: int) -> int:
    sl, p = _host_i32(seqlens)
    return int(lib().kvc_freekv_workspace_size(len(sl), p, n_h, n_kv, d_h, w, budget))


def kvc_freekv_step(seqlens, cu_seqlens, cu_budget, n_h: int, w: int, pool_k: int, budget: int, tau: float,
                    scale: float, q_cur, q_prev, k, v, idx, k_c, v_c, reselected, out, ws, stream=None) -> None:
    """One FreeKV decode step: re-select the heads whose query drifted, then decode."""
    sl, p = _host_i32(seqlens)
    _check(lib().kvc_freekv_step(len(sl), p, _dptr(cu_seqlens), _dptr(cu_budget), n_h, k.shape[1], k.shape[2], w,
                                 pool_k, budget, tau, scale, _dptr(q_cur), _dptr(q_prev), _dptr(k), _dptr(v),
                                 _dptr(idx), _dptr(k_c), _dptr(v_c), _dptr(reselected), _dptr(out), _dptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)))


def kvc_xkv_workspace_size(S: int, n_kv: int, d_h: int, W: int, r: int) -> int:
    return int(lib().kvc_xkv_workspace_size(S, n_kv, d_h, W, r))


def kvc_xkv_factorize(k_layers, r: int, iters: int, v0, basis, blocks, ws, stream=None) -> None:
    """xKV factorisation of the keys of W layers (list of bf16 [S, n_kv, d_h]
    tensors): writes basis (A, [n_kv, S, r], float32 or bf16) and blocks (Vt,
    float32 [n_kv, r, W d_h])."""
    S, n_kv, d_h = k_layers[0].shape
    ptrs = (ctypes.c_void_p * len(k_layers))(*[t.data_ptr() for t in k_layers])
    _check(lib().kvc_xkv_factorize(S, n_kv, d_h, len(k_layers), r, iters, ptrs, _dptr(v0), dtype_code(basis),
                                   _dptr(basis), _dptr(blocks), _dptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)))


def kvc_xkv_reconstruct(W: int, layer: int, basis, blocks, idx, out, stream=None) -> None:
    """Rows idx ([n_kv, n_sel] int32) of layer `layer` into out (bf16 [n_sel, n_kv, d_h])."""
    n_kv, S, r = basis.shape
    n_sel = idx.shape[1]
    d_h = out.shape[2]
    _check(lib().kvc_xkv_reconstruct(S, n_kv, d_h, W, r, layer, n_sel, dtype_code(basis), _dptr(basis),
                                     _dptr(blocks), _dptr(idx), _dptr(out), _stream(stream)))
