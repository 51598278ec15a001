"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Sizes: small cases that span several key tiles and chunks with ragged tails,
plus the edge cases (prefix of length 0, budget == window, budget >= length,
empty decode caches, aliased cache offsets, pool size 1)."""
import numpy as np
import pytest
import torch

from kv_cache_compression_score_b200 import synth
from kv_cache_compression_score_b200.runner import Compressor, TspSelector, from_device, to_device
from oracle import kvc_oracle as O
from parity_helpers import (assert_scores_close, assert_selection_matches, run_and_check_compress,
                            run_and_check_decode)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from kv_cache_compression_score_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


# ------------------------------------------------------------------ scoring
def test_small_fp32_layer_s2048_whole_path():
    """One layer, n_h 4, n_kv 2, d_h 64, S 2048, fp32, w 32, pool 7, B 256."""
    r = run_and_check_compress("f32", [2048], 4, 2, 64, 32, 7, 256, seed=1001)
    assert r["n_diff"] == 0
    # then one decode query over the retained cache (256 rows per KV head)
    q = synth.decode_queries(1001 + 8, 1, 4, 64, "f32")
    run_and_check_decode("f32", q, from_device(r["comp"].buf.k_c), from_device(r["comp"].buf.v_c), [0], [256], 2)


@pytest.mark.parametrize("lengths", [[1000, 300, 129, 32, 777], [4097]])
def test_bf16_tensor_core_ragged(lengths):
    """G*w = 128 rows: tensor-core kernels; ragged tails inside key tiles."""
    run_and_check_compress("bf16", lengths, 32, 8, 128, 32, 7, 200, seed=1234)


def test_bf16_tensor_core_split_launches():
    """20 sequences x 8 KV heads = 160 work items: more than fit on the GPU at
    once, so the two passes and the pool run as separate launches."""
    lengths = synth.ragged_lengths(4242, 20, 40, 700).tolist()
    run_and_check_compress("bf16", lengths, 32, 8, 128, 32, 7, 96, seed=4243)


def test_bf16_fused_repeated_calls():
    """The single cooperative launch, three times on the same workspace: its
    arrival counters must come back to zero after every call."""
    run_and_check_compress("bf16", [3000, 1500], 32, 8, 128, 32, 7, 300, seed=4244, repeat=3)


def test_check_workspace_reads_the_device_error_word():
    """kvc_check_workspace: clear after a healthy call; KVC_ERR_DEVICE_CHECK
    once the error word is nonzero (planted from the host, no fault)."""
    from kv_cache_compression_score_b200 import kvc
    r = run_and_check_compress("bf16", [600], 32, 8, 128, 32, 7, 100, seed=4245)
    ws = r["comp"].buf.ws
    assert kvc.kvc_check_workspace(ws) == kvc.KVC_OK
    ws[:4].view(torch.int32).fill_(1)
    assert kvc.kvc_check_workspace(ws) == kvc.KVC_ERR_DEVICE_CHECK
    ws[:4].view(torch.int32).fill_(0)
    assert kvc.kvc_check_workspace(ws) == kvc.KVC_OK


def test_fused_wait_gives_up_and_reports():
    """A cross-CTA wait that can never complete (its arrival counter planted
    far below zero from the host: no fault, no trap) gives up after its time
    limit; the call returns, the device error word reads back as
    KVC_ERR_DEVICE_CHECK, the counters are left at zero, and the context stays
    usable: a rerun on the re-zeroed workspace matches the oracle."""
    from kv_cache_compression_score_b200 import kvc
    lengths = [2000]
    bt = synth.packed_batch(4246, lengths, 32, 8, 128, 32, "bf16", 0.0, 3.0)
    q, k, v = (to_device(bt[x], "bf16") for x in ("q_win", "k", "v"))
    comp = Compressor("bf16", lengths, 32, 8, 128, 32, 7, 200)
    ctr = comp.buf.ws[256:256 + 32 * 8].view(torch.int32)
    ctr[0] = -1 << 20                                   # head 0's stats barrier can never fill
    comp.score(q, k)
    assert kvc.kvc_check_workspace(comp.buf.ws) == kvc.KVC_ERR_DEVICE_CHECK
    assert int(ctr.abs().sum().item()) == 0             # the last CTA of each head reset them
    comp.buf.ws.zero_()
    comp.score(q, k)
    assert kvc.kvc_check_workspace(comp.buf.ws) == kvc.KVC_OK
    raw_o = O.raw_scores(bt["q_win"], bt["k"], bt["cu_seqlens"], 32, 8, 32, "bf16")
    assert_scores_close(comp.buf.scores_raw.cpu().numpy(), raw_o, what="raw scores after recovery")


@pytest.mark.parametrize("lengths,budget", [([3000, 1500], 300), ([4097], 1000), ([700, 64], 700), ([700, 64], 32),
                                            ([1000, 300, 129, 32, 777], 200)])
def test_compress_window_fused_select_gather(lengths, budget):
    """kvc_compress_window: scores, indices and gathered rows against the
    oracle (one launch with selection inside where it applies; the identity,
    budget == window and tiny-sequence edges included)."""
    run_and_check_compress("bf16", lengths, 32, 8, 128, 32, 7, budget, seed=4250, fused_call=True, repeat=2)


def test_compress_window_ties_exact():
    """Many equal pooled scores (boost-free keys, pool 7 plateaus): the fused
    selection keeps the lowest positions among equal scores, checked against
    the oracle's exact rule; repeated calls reuse the workspace."""
    r = run_and_check_compress("bf16", [2500], 32, 8, 128, 32, 7, 600, seed=4251, fused_call=True, repeat=3,
                               boost_frac=0.01, boost=40.0)
    # on the GPU's own fp32 pooled scores the selection is exact: identical to
    # the oracle's rule applied to those same values
    pooled_g = r["comp"].buf.scores.cpu().numpy().astype(np.float64)
    idx_ref = O.select_topk(pooled_g, r["bt"]["cu_seqlens"], 32, 600)
    assert np.array_equal(r["idx_g"], idx_ref)


def test_compress_window_all_equal_scores_overflow_path():
    """K = 0: every pooled prefix score is equal, so the bucket of the k-th key
    holds the whole prefix (more candidates than the exchange takes) and the
    radix path decides; the lowest positions must be kept, exactly as the
    oracle's rule (and the tie-break pin) says."""
    lengths, budget = [5000, 3000], 1000
    bt = synth.packed_batch(4254, lengths, 32, 8, 128, 32, "bf16", 0.0, 3.0)
    q, v = to_device(bt["q_win"], "bf16"), to_device(bt["v"], "bf16")
    k = torch.zeros_like(v)
    comp = Compressor("bf16", lengths, 32, 8, 128, 32, 7, budget)
    for _ in range(2):
        comp.compress(q, k, v)
    torch.cuda.synchronize()
    assert comp.device_error_word() == 0
    cu = bt["cu_seqlens"]
    idx_o = O.select_topk(O.pool_prefix(O.raw_scores(bt["q_win"], np.zeros_like(bt["k"]), cu, 32, 8, 32, "bf16"),
                                        cu, 32, 7), cu, 32, budget)
    assert np.array_equal(comp.buf.idx.cpu().numpy(), idx_o)
    for b, L in enumerate(lengths):
        seg = comp.buf.idx.cpu().numpy()[:, b * budget:(b + 1) * budget]
        assert np.array_equal(seg, np.broadcast_to(np.r_[np.arange(budget - 32), np.arange(L - 32, L)], seg.shape))


def test_compress_window_split_fallback():
    """More work items than fit at once: kvc_compress_window runs the three calls."""
    lengths = synth.ragged_lengths(4252, 20, 40, 700).tolist()
    run_and_check_compress("bf16", lengths, 32, 8, 128, 32, 7, 96, seed=4253, fused_call=True)


def test_bf16_tensor_core_small_block_d64():
    """G*w = 16 rows padded to the 128-row tile; d_h 64 (one swizzle atom)."""
    run_and_check_compress("bf16", [513, 64, 200], 8, 4, 64, 8, 3, 40, seed=77)


def test_bf16_cuda_core_large_block():
    """G*w = 192 rows: bf16 on the CUDA-core kernels."""
    run_and_check_compress("bf16", [400, 130], 8, 1, 128, 24, 5, 60, seed=5)


def test_fp32_d128_odd_block_and_empty_prefix():
    """G*w = 30 rows (not a multiple of 16); a sequence with len == w (P = 0)."""
    run_and_check_compress("f32", [300, 45, 10], 6, 2, 128, 10, 7, 12, seed=9)


def test_pool1_budget_edges():
    """pool 1 (no smoothing); budget == w keeps only the window; budget >= len is the identity."""
    run_and_check_compress("bf16", [700, 64], 32, 8, 128, 32, 1, 32, seed=3)
    run_and_check_compress("bf16", [700, 64], 32, 8, 128, 32, 7, 700, seed=3)


def test_probability_mass_on_gpu():
    """Summed over all visible keys, the raw scores of a KV head total G * w."""
    r = run_and_check_compress("bf16", [3000, 515], 32, 8, 128, 32, 7, 300, seed=11)
    raw = r["comp"].buf.scores_raw.cpu().numpy().astype(np.float64)
    cu = r["bt"]["cu_seqlens"]
    for b in range(2):
        np.testing.assert_allclose(raw[:, cu[b]:cu[b + 1]].sum(1), 4 * 32, rtol=1e-5)


# ---------------------------------------------------------------- selection
@pytest.mark.parametrize("levels,lengths", [(0, [5000, 100, 33, 40000, 40]), (5, [5000, 100, 33, 40000, 40]),
                                            (5, [5000, 41100, 33]), (0, [70000, 64])])
def test_select_isolated_exact(levels, lengths):
    """Seeded fp32 scores (with many exact ties at levels=5) fed to both sides:
    the index lists must be identical.  Batches whose longest prefix exceeds
    the select kernel's shared-memory cache exercise the global-memory path."""
    w, budget, n_kv = 32, 1024, 3
    T = int(sum(lengths))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = synth.random_scores(17 + levels, (n_kv, T), n_levels=levels)
    for b, L in enumerate(lengths):
        s[:, cu[b] + L - w:cu[b + 1]] = np.inf
    comp = Compressor("f32", lengths, 4 * n_kv, n_kv, 64, w, 7, budget)
    comp.buf.scores.copy_(torch.from_numpy(s))
    comp.select()
    torch.cuda.synchronize()
    idx_o = O.select_topk(s.astype(np.float64), cu, w, budget)
    np.testing.assert_array_equal(comp.buf.idx.cpu().numpy(), idx_o)


# ------------------------------------------------------------------ gather
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_gather_isolated_bit_exact(dtype, d):
    lengths, n_kv, budget = [900, 17, 256], 8, 300
    bt = synth.packed_batch(21, lengths, 8, n_kv, d, 4, dtype)
    idx = synth.index_lists(22, lengths, n_kv, budget)
    comp = Compressor(dtype, lengths, 8, n_kv, d, 4, 7, budget)
    comp.buf.idx.copy_(torch.from_numpy(idx))
    k, v = to_device(bt["k"], dtype), to_device(bt["v"], dtype)
    comp.gather(k, v)
    torch.cuda.synchronize()
    kc_o, vc_o = O.gather_kv(bt["k"], bt["v"], idx.astype(np.int64), bt["cu_seqlens"], budget)
    assert np.array_equal(from_device(comp.buf.k_c), kc_o)
    assert np.array_equal(from_device(comp.buf.v_c), vc_o)


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("dtype,d,n_h,n_kv", [("f32", 64, 4, 2), ("bf16", 128, 32, 8), ("bf16", 64, 8, 8),
                                              ("f32", 128, 16, 2), ("bf16", 128, 16, 8), ("bf16", 128, 64, 8),
                                              ("bf16", 64, 16, 4)])
def test_decode_isolated(dtype, d, n_h, n_kv):
    """Synthetic compact caches with ragged lengths, one empty cache, a
    length-1 cache and two queries aliasing the same cache."""
    lens = [2048, 0, 1, 777, 2048, 130]
    offs = [0, 2048, 2048, 2049, 0, 2826]
    rows = 2826 + 130
    kc, vc = synth.keys_values(31, 0, rows, n_kv, d, dtype)
    q = synth.decode_queries(32, len(lens), n_h, d, dtype)
    got, ref, err = run_and_check_decode(dtype, q, kc, vc, offs, lens, n_kv)
    assert np.all(got[1] == 0)


def test_decode_twice_reuses_workspace():
    lens, offs = [5000, 3000], [0, 5000]
    kc, vc = synth.keys_values(41, 0, 8000, 8, 128, "bf16")
    q = synth.decode_queries(42, 2, 32, 128, "bf16")
    for _ in range(2):
        run_and_check_decode("bf16", q, kc, vc, offs, lens, 8)


def test_identity_budget_gives_full_attention():
    """B >= S: selection is the identity, the compact cache is the cache, and
    decode over it is full attention over the original cache."""
    L = 1500
    r = run_and_check_compress("bf16", [L], 32, 8, 128, 32, 7, L, seed=51)
    np.testing.assert_array_equal(r["idx_g"], np.broadcast_to(np.arange(L), (8, L)))
    kc = from_device(r["comp"].buf.k_c)
    assert np.array_equal(kc, r["bt"]["k"])
    q = synth.decode_queries(52, 1, 32, 128, "bf16")
    run_and_check_decode("bf16", q, r["bt"]["k"], r["bt"]["v"], [0], [L], 8)


# --------------------------------------------------------------------- TSP
def test_tsp_isolated_exact():
    """Dyadic raw scores (k/1024): their fp32 head sums are exact, so both
    sides see identical aggregated values and must pick identical sets."""
    S, w, n_rows, k_tsp, D = 5000, 32, 8, 997, 256
    raw = synth.random_scores(61, (n_rows, S), n_levels=1024)
    hidden = synth.hidden_states(62, S, D, "bf16")
    sel = TspSelector(S, w, 7, k_tsp, D, "bf16")
    idx, hout = sel.run(torch.from_numpy(raw).cuda(), to_device(hidden, "bf16"))
    torch.cuda.synchronize()
    idx_o = O.tsp_select(raw.astype(np.float64), S, w, 7, k_tsp)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_o)
    assert np.array_equal(from_device(hout), O.tsp_gather(hidden, idx_o))


def test_tsp_after_scoring_tie_band():
    """TSP on the raw scores of the scoring kernels (one sequence)."""
    S, w = 3000, 32
    r = run_and_check_compress("bf16", [S], 32, 8, 128, w, 7, 300, seed=71)
    k_tsp = O.rate_count(0.2, S)
    hidden = synth.hidden_states(72, S, 512, "bf16")
    sel = TspSelector(S, w, 7, k_tsp, 512, "bf16")
    idx, hout = sel.run(r["comp"].buf.scores_raw, to_device(hidden, "bf16"))
    torch.cuda.synchronize()
    idx_o = O.tsp_select(r["raw_o"], S, w, 7, k_tsp)
    pooled_o = O.tsp_pooled(r["raw_o"], S, w, 7)
    g = idx.cpu().numpy()
    assert np.all(np.diff(g) > 0) and np.array_equal(g[k_tsp:], np.arange(S - w, S))
    diff = set(g[:k_tsp].tolist()) ^ set(idx_o[:k_tsp].tolist())
    kth = np.sort(pooled_o)[::-1][k_tsp - 1]
    assert all(abs(pooled_o[j] - kth) <= 1e-5 * kth for j in diff)
    assert np.array_equal(from_device(hout), O.tsp_gather(hidden, g))
