"""Host-side checks of the C ABI that need no GPU: the library loads, every
entry point declared in include/kvc.h is exported and bound, the host helpers
compute what the pages fix, and invalid arguments are rejected before any
CUDA call."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

from kv_cache_compression_score_b200 import build as kbuild
from kv_cache_compression_score_b200 import kvc
from oracle import kvc_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvc.h")
INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kvc.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvc_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound(L):
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
        assert n in kvc.SIGNATURES, f"{n} has no binding"
    assert set(kvc.SIGNATURES) == set(names)


def test_version_and_status_strings(L):
    assert kvc.kvc_version() >= 100
    assert L.kvc_status_string(0) == b"KVC_OK"
    assert L.kvc_status_string(3) == b"KVC_ERR_WORKSPACE"


def test_cache_bytes_matches_worked_example(L):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "cache_bytes.json")))
    for c in g["cases"]:
        assert c.get("n_seqs", 1) * kvc.kvc_cache_bytes(c["L"], c["S"], c["n_kv"], c["d_h"], c["b"]) == c["bytes"]
    assert kvc.kvc_cache_bytes(-1, 4, 1, 1, 1) == 0


def test_budget_offsets(L):
    lens = [100, 3, 50, 0, 7]
    np.testing.assert_array_equal(kvc.kvc_budget_offsets(lens, 20), O.budget_offsets(lens, 20))
    with pytest.raises(kvc.KvcError):
        kvc.kvc_budget_offsets([5, -1], 3)


def test_pyramid_budgets_host_helper(L):
    for args in [(32, 3276, 1000), (32, 2048, 2048), (1, 500, 100), (7, 300, 32), (2, 64, 0)]:
        np.testing.assert_array_equal(kvc.kvc_pyramid_budgets(*args), O.pyramid_budgets(*args))
    for bad in [(0, 10, 5), (4, 10, 11), (4, 10, -1)]:
        with pytest.raises(kvc.KvcError):
            kvc.kvc_pyramid_budgets(*bad)


def test_workspace_sizes(L):
    sl = np.array([32768], dtype=np.int32)
    n = kvc.kvc_score_window_workspace_size(kvc.KVC_BF16, sl, 32, 8, 128, 32)
    assert n >= 8 * 32768 * 4                                   # holds the raw scores
    assert kvc.kvc_score_window_workspace_size(kvc.KVC_BF16, sl, 32, 8, 96, 32) == 0   # d_h unsupported
    assert kvc.kvc_score_window_workspace_size(kvc.KVC_BF16, np.array([16], np.int32), 32, 8, 128, 32) == 0
    assert kvc.kvc_tsp_workspace_size(32768, 32) >= (32768 - 32) * 4
    assert kvc.kvc_tsp_workspace_size(10, 11) == 0
    assert kvc.kvc_gqa_decode_workspace_size(16, 32, 8, 128, 2048) > 0
    assert kvc.kvc_gqa_decode_workspace_size(16, 24, 8, 128, 2048) == 0   # G = 3


P16 = ctypes.c_void_p(1 << 20)     # aligned fake device address (never dereferenced: calls fail first)
P8 = ctypes.c_void_p((1 << 20) + 8)


def _score(L, **kw):
    a = dict(dt=kvc.KVC_BF16, n_seqs=1, sl=np.array([64], np.int32), cu=P16, n_h=4, n_kv=2, d_h=128, w=8,
             pool_k=7, scale=0.0, q=P16, k=P16, sc=P16, raw=None, ws=P16, ws_bytes=1 << 30)
    a.update(kw)
    return L.kvc_score_window(a["dt"], a["n_seqs"], a["sl"].ctypes.data_as(ctypes.c_void_p), a["cu"], a["n_h"],
                              a["n_kv"], a["d_h"], a["w"], a["pool_k"], a["scale"], a["q"], a["k"], a["sc"],
                              a["raw"], a["ws"], a["ws_bytes"], None)


def test_score_window_rejects_before_launch(L):
    assert _score(L, pool_k=4) == INVALID
    assert _score(L, pool_k=33) == INVALID
    assert _score(L, d_h=96) == UNSUPPORTED
    assert _score(L, dt=7) == UNSUPPORTED
    assert _score(L, n_h=6, n_kv=4) == INVALID
    assert _score(L, w=65) == INVALID                     # sequence shorter than the window
    assert _score(L, n_h=16, n_kv=1, w=32) == UNSUPPORTED  # 512-row window block
    assert _score(L, q=None) == INVALID
    assert _score(L, k=P8) == INVALID
    assert _score(L, raw=P8) == INVALID
    assert _score(L, ws_bytes=16) == WORKSPACE
    assert _score(L, n_seqs=0) == INVALID


def test_select_gather_decode_tsp_reject_before_launch(L):
    sl = np.array([100, 40], np.int32)
    slp = sl.ctypes.data_as(ctypes.c_void_p)
    # budget below the window
    assert L.kvc_select_topk(2, slp, P16, P16, 8, 32, 31, P16, P16, None) == INVALID
    assert b"window" in L.kvc_last_error()
    assert L.kvc_select_topk(2, slp, None, P16, 8, 32, 64, P16, P16, None) == INVALID
    assert L.kvc_select_topk(2, slp, P16, P16, 8, 32, 64, P8, P16, None) == INVALID
    # gather: row bytes must be a multiple of 16
    assert L.kvc_gather_kv(kvc.KVC_BF16, 2, slp, P16, P16, 8, 4, 64, P16, P16, P16, P16, P16, None) == UNSUPPORTED
    assert L.kvc_gather_kv(kvc.KVC_BF16, 2, slp, P16, P16, 8, 128, 64, P16, P16, P8, P16, P16, None) == INVALID
    # decode: group of 3, odd head dim, small workspace
    assert L.kvc_gqa_decode_attn(kvc.KVC_BF16, 2, 24, 8, 128, 0.0, P16, P16, P16, 200, P16, P16, 100, P16, P16,
                                 1 << 30, None) == UNSUPPORTED
    assert L.kvc_gqa_decode_attn(kvc.KVC_BF16, 2, 32, 8, 80, 0.0, P16, P16, P16, 200, P16, P16, 100, P16, P16,
                                 1 << 30, None) == UNSUPPORTED
    assert L.kvc_gqa_decode_attn(kvc.KVC_BF16, 2, 32, 8, 128, 0.0, P16, P16, P16, 200, P16, P16, 100, P16, P16, 8,
                                 None) == WORKSPACE
    assert L.kvc_gqa_decode_attn(kvc.KVC_BF16, 2, 32, 8, 128, 0.0, P16, P16, P16, 0, P16, P16, 100, P16, P16,
                                 1 << 30, None) == INVALID
    # TSP: k_tsp beyond the prefix, even pool
    assert L.kvc_tsp_select_gather(kvc.KVC_BF16, 100, 8, 32, 7, 69, P16, P16, 4096, P16, P16, P16, 1 << 20,
                                   None) == INVALID
    assert L.kvc_tsp_select_gather(kvc.KVC_BF16, 100, 8, 32, 6, 10, P16, P16, 4096, P16, P16, P16, 1 << 20,
                                   None) == INVALID
    assert L.kvc_tsp_select_gather(kvc.KVC_BF16, 100, 8, 32, 7, 10, P16, P16, 4, P16, P16, P16, 1 << 20,
                                   None) == UNSUPPORTED


def test_xkv_rejects_before_launch(L):
    ptrs = (ctypes.c_void_p * 8)(*([P16.value] * 8))
    ws_ok = kvc.kvc_xkv_workspace_size(256, 2, 128, 4, 64)
    assert ws_ok >= 2 * 512 * 512 * 4                    # holds the Gram matrices
    assert kvc.kvc_xkv_workspace_size(256, 2, 128, 5, 64) == 0     # W d_h = 640 > 512
    assert kvc.kvc_xkv_workspace_size(256, 2, 96, 2, 16) == 0      # d_h unsupported
    assert kvc.kvc_xkv_workspace_size(40, 2, 128, 2, 64) == 0      # r > S

    def fac(S=256, n_kv=2, d=128, W=4, r=64, iters=8, kl=ptrs, v0=P16, bdt=kvc.KVC_BF16, basis=P16, ws_b=ws_ok):
        return L.kvc_xkv_factorize(S, n_kv, d, W, r, iters, kl, v0, bdt, basis, P16, P16, ws_b, None)

    assert fac(r=48) == UNSUPPORTED
    assert fac(W=9) == UNSUPPORTED
    assert fac(iters=0) == INVALID
    assert fac(bdt=7) == UNSUPPORTED
    assert fac(kl=None) == INVALID
    assert fac(kl=(ctypes.c_void_p * 8)(*([P8.value] * 8))) == INVALID
    assert fac(v0=None) == INVALID
    assert fac(basis=P8) == INVALID
    assert fac(ws_b=64) == WORKSPACE
    assert fac(S=32, r=64) == INVALID

    def rec(layer=0, n_sel=10, r=64, idx=P16):
        return L.kvc_xkv_reconstruct(256, 2, 128, 4, r, layer, n_sel, kvc.KVC_BF16, P16, P16, idx, P16, None)

    assert rec(layer=4) == INVALID
    assert rec(layer=-1) == INVALID
    assert rec(n_sel=-1) == INVALID
    assert rec(r=8) == UNSUPPORTED
    assert rec(idx=P8) == INVALID
    assert rec(n_sel=0) == 0                               # nothing to do, nothing launched


def test_check_workspace_and_launch_count_need_no_gpu_to_validate(L):
    """kvc_check_workspace rejects a NULL workspace before any CUDA call; the
    launch counter is readable without a device."""
    with pytest.raises(kvc.KvcError) as e:
        kvc.kvc_check_workspace(None, stream=0)
    assert e.value.status == kvc.KVC_ERR_INVALID_ARG
    assert L.kvc_status_string(kvc.KVC_ERR_DEVICE_CHECK) == b"KVC_ERR_DEVICE_CHECK"
    assert kvc.kvc_launch_count() >= 0


def test_compress_window_rejects_before_launch(L):
    """kvc_compress_window validates the selection and gather arguments as well
    as the scoring ones, before anything is launched."""
    sl = np.array([300, 100], np.int32)
    slp = sl.ctypes.data_as(ctypes.c_void_p)
    ws_ok = kvc.kvc_score_window_workspace_size(kvc.KVC_BF16, sl, 32, 8, 128, 32)
    assert ws_ok > 0

    def call(budget=64, cu_budget=P16, v=P16, idx=P16, k_out=P16, v_out=P16, ws_bytes=ws_ok, pool_k=7, w=32,
             dt=kvc.KVC_BF16):
        return L.kvc_compress_window(dt, 2, slp, P16, cu_budget, 32, 8, 128, w, pool_k, budget, 0.0, P16, P16, v,
                                     P16, None, idx, k_out, v_out, P16, ws_bytes, None)

    assert call(budget=31) == INVALID and b"window" in L.kvc_last_error()
    assert call(cu_budget=None) == INVALID
    assert call(v=None) == INVALID
    assert call(idx=P8) == INVALID
    assert call(k_out=None) == INVALID
    assert call(v_out=P8) == INVALID
    assert call(pool_k=6) == INVALID
    assert call(w=101) == INVALID                        # the second sequence is shorter than the window
    assert call(ws_bytes=64) == WORKSPACE
    assert call(dt=5) == UNSUPPORTED


def test_int8_cache_calls_reject_before_launch(L):
    """kvc_gather_kv_q8 and kvc_gqa_decode_attn_q8 validate every argument
    before anything is launched (each call below has exactly one bad one)."""
    sl = np.array([100, 40], np.int32)
    slp = sl.ctypes.data_as(ctypes.c_void_p)

    def gq(n_seqs=2, cu=P16, n_kv=8, d_h=128, budget=64, k_q=P16, pitch=104):
        return L.kvc_gather_kv_q8(n_seqs, slp, cu, P16, n_kv, d_h, budget, P16, P16, P16, k_q, P16, P16, P16, pitch,
                                  None)

    assert gq(n_seqs=0) == INVALID
    assert gq(n_kv=0) == INVALID
    assert gq(d_h=96) == UNSUPPORTED
    assert gq(budget=-1) == INVALID
    assert gq(cu=None) == INVALID
    assert gq(k_q=P8) == INVALID
    assert gq(pitch=103) == INVALID and b"scale_pitch" in L.kvc_last_error()   # 64 + 40 compact rows
    assert gq(budget=0) == 0                               # no compact rows: nothing to do, nothing launched

    def dq(batch=2, n_h=32, d_h=128, q=P16, kv_len=P16, pitch=200, rows=200, ws_bytes=1 << 30):
        return L.kvc_gqa_decode_attn_q8(batch, n_h, 8, d_h, 0.0, q, P16, P16, P16, P16, pitch, rows, P16, kv_len, 100,
                                        P16, P16, ws_bytes, None)

    assert dq(batch=0) == INVALID
    assert dq(n_h=24) == UNSUPPORTED                       # GQA group 3
    assert dq(d_h=80) == UNSUPPORTED
    assert dq(q=P8) == INVALID
    assert dq(kv_len=None) == INVALID
    assert dq(rows=0) == INVALID
    assert dq(pitch=199) == INVALID
    assert dq(ws_bytes=8) == WORKSPACE


def test_freekv_step_rejects_before_launch(L):
    """kvc_freekv_step and its workspace query validate before any launch."""
    sl = np.array([300, 100], np.int32)
    slp = sl.ctypes.data_as(ctypes.c_void_p)
    ws_ok = L.kvc_freekv_workspace_size(2, slp, 32, 8, 128, 32, 64)
    assert ws_ok > 0
    assert L.kvc_freekv_workspace_size(2, slp, 32, 8, 128, 32, 31) == 0     # budget below the window
    assert L.kvc_freekv_workspace_size(2, slp, 32, 8, 128, 101, 128) == 0   # a sequence shorter than w
    assert L.kvc_freekv_workspace_size(2, slp, 24, 8, 128, 32, 64) == 0     # GQA group 3
    assert L.kvc_freekv_workspace_size(2, slp, 32, 8, 96, 32, 64) == 0      # d_h

    def fk(pool_k=7, budget=64, cu_budget=P16, q_prev=P16, out=P16, ws_bytes=ws_ok):
        return L.kvc_freekv_step(2, slp, P16, cu_budget, 32, 8, 128, 32, pool_k, budget, 0.9, 0.0, P16, q_prev,
                                 P16, P16, P16, P16, P16, P16, out, P16, ws_bytes, None)

    assert fk(pool_k=6) == INVALID
    assert fk(pool_k=33) == INVALID
    assert fk(budget=31) == INVALID and b"window" in L.kvc_last_error()
    assert fk(cu_budget=None) == INVALID
    assert fk(q_prev=P8) == INVALID
    assert fk(out=None) == INVALID
    assert fk(ws_bytes=ws_ok - 1) == WORKSPACE


def test_tsp_static_rejects_before_launch(L):
    """The no-allocation TSP entry point checks its size limit and every
    argument before it resolves its scratch or launches anything."""
    def ts(S=1000, w=32, pool_k=7, k_tsp=100, D=4096, hidden=P16, dt=kvc.KVC_BF16):
        return L.kvc_tsp_select_gather_static(dt, S, 8, w, pool_k, k_tsp, P16, hidden, D, P16, P16, None)

    assert ts(S=262144 + 33) == UNSUPPORTED and b"workspace" in L.kvc_last_error()   # S - w = 262,145
    assert ts(dt=7) == UNSUPPORTED
    assert ts(w=1001) == INVALID
    assert ts(pool_k=8) == INVALID
    assert ts(k_tsp=969) == INVALID                        # beyond the prefix S - w = 968
    assert ts(D=4) == UNSUPPORTED                          # 8-byte rows
    assert ts(hidden=P8) == INVALID
