"""Parity at the full workload sizes, in the launch configuration the bench
uses.  The fp64 oracle computes every output of these sizes, so the whole
output is compared (not a sample).

Workloads (seeded synthetic stand-ins for the pages' long-context models):
  Llama-3-8B-shaped layer: n_h 32, n_kv 8, d_h 128, bf16, S 32768, window 32,
      pool 7, budget 2048, 1% of keys boosted; decode batch 16;
  long context: S 131072, budget 4096 and budget S (identity);
  FastKV TSP layer: S 32768, k_tsp = floor(0.2 S), hidden [S, 4096] bf16,
      then the first propagated layer at S' = k_tsp + 32 with budget
      floor(0.1 S);
  ragged: 16 lengths uniform on [4096, 65536], budget 1024.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_score_b200 import synth
from kv_cache_compression_score_b200.runner import TspSelector, from_device, to_device
from oracle import kvc_oracle as O
from parity_helpers import log_parity, run_and_check_compress, run_and_check_decode

pytestmark = pytest.mark.gpu

N_H, N_KV, D, W, POOL = 32, 8, 128, 32, 7


@pytest.fixture(autouse=True, scope="module")
def _built():
    from kv_cache_compression_score_b200 import build
    build.build()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("fused", [False, True])
def test_llama8b_layer_s32k(fused):
    """fused: kvc_compress_window (one launch: score, select and gather)."""
    r = run_and_check_compress("bf16", [32768], N_H, N_KV, D, W, POOL, 2048, seed=1002, boost_frac=0.01,
                               fused_call=fused)
    # decode at batch 16 over 16 compact caches of 2048 rows (the step's own cache first)
    kc = [from_device(r["comp"].buf.k_c)]
    vc = [from_device(r["comp"].buf.v_c)]
    for b in range(1, 16):
        k, v = synth.keys_values(1009, b, 2048, N_KV, D, "bf16")
        kc.append(k)
        vc.append(v)
    q = synth.decode_queries(1010, 16, N_H, D, "bf16")
    run_and_check_decode("bf16", q, np.concatenate(kc), np.concatenate(vc), np.arange(16) * 2048, [2048] * 16, N_KV)


@pytest.mark.parametrize("budget,fused", [(4096, False), (131072, False), (4096, True), (131072, True)])
def test_long_context_s128k(budget, fused):
    S = 131072
    r = run_and_check_compress("bf16", [S], N_H, N_KV, D, W, POOL, budget, seed=1003, boost_frac=0.01,
                               fused_call=fused)
    if budget >= S:
        # identity: every position kept, compact cache == cache, decode == full attention
        np.testing.assert_array_equal(r["idx_g"], np.broadcast_to(np.arange(S), (N_KV, S)))
        assert np.array_equal(from_device(r["comp"].buf.k_c), r["bt"]["k"])
        q = synth.decode_queries(1011, 8, N_H, D, "bf16")
        run_and_check_decode("bf16", q, r["bt"]["k"], r["bt"]["v"], [0] * 8, [S] * 8, N_KV)
    else:
        q = synth.decode_queries(1012, 8, N_H, D, "bf16")
        run_and_check_decode("bf16", q, from_device(r["comp"].buf.k_c), from_device(r["comp"].buf.v_c), [0] * 8,
                             [budget] * 8, N_KV)


def test_fastkv_tsp_layer_and_next_layer():
    S = 32768
    k_tsp, kv_budget = O.rate_count(0.2, S), O.rate_count(0.1, S)
    r = run_and_check_compress("bf16", [S], N_H, N_KV, D, W, POOL, kv_budget, seed=1004 + 15, boost_frac=0.01)
    hidden = synth.hidden_states(1004, S, 4096, "bf16")
    sel = TspSelector(S, W, POOL, k_tsp, 4096, "bf16")
    idx, hout = sel.run(r["comp"].buf.scores_raw, to_device(hidden, "bf16"))
    torch.cuda.synchronize()
    idx_o = O.tsp_select(r["raw_o"], S, W, POOL, k_tsp)
    pooled_o = O.tsp_pooled(r["raw_o"], S, W, POOL)
    g = idx.cpu().numpy()
    assert len(g) == k_tsp + W and np.all(np.diff(g) > 0)
    np.testing.assert_array_equal(g[k_tsp:], np.arange(S - W, S))
    kth = np.sort(pooled_o)[::-1][k_tsp - 1]
    diff = set(g[:k_tsp].tolist()) ^ set(idx_o[:k_tsp].tolist())
    assert all(abs(pooled_o[j] - kth) <= 1e-5 * kth for j in diff)
    # hidden rows: a byte copy of the rows the GPU's own index list names, every row
    assert np.array_equal(from_device(hout), O.tsp_gather(hidden, g))
    log_parity(dict(what="tsp", S=S, k_tsp=k_tsp, tie_band_index_differences=len(diff), rows_compared=len(g)))
    # first layer after the TSP layer runs on S' = k_tsp + w tokens, same KV budget
    run_and_check_compress("bf16", [k_tsp + W], N_H, N_KV, D, W, POOL, kv_budget, seed=1004 + 16, boost_frac=0.01)


@pytest.mark.parametrize("schedule", ["uniform", "pyramid"])
def test_fastkv_32_layer_chain(schedule):
    """The whole FastKV workload: 32 layers of the Llama-3-8B shape, layers
    0-15 at S = 32768, token-selective propagation at layer 15 (k_tsp =
    floor(0.2 S) plus the window, hidden [S, 4096]), layers 16-31 at
    S' = k_tsp + 32.  Per-layer KV budgets: 10% of S on every layer, or the
    PyramidKV schedule around the same mean (first layer 2 * 3276 - 1024,
    last layer 1024).  Every layer's one-call compression is checked against
    the oracle."""
    from kv_cache_compression_score_b200 import kvc
    S, L = 32768, 32
    k_tsp, b_avg = O.rate_count(0.2, S), O.rate_count(0.1, S)
    budgets = (np.full(L, b_avg) if schedule == "uniform" else kvc.kvc_pyramid_budgets(L, b_avg, 1024))
    if schedule == "pyramid":
        np.testing.assert_array_equal(budgets, O.pyramid_budgets(L, b_avg, 1024))
    S_next = k_tsp + W
    n_diff = 0
    for layer in range(L):
        length = S if layer <= 15 else S_next
        r = run_and_check_compress("bf16", [length], N_H, N_KV, D, W, POOL, int(budgets[layer]),
                                   seed=4000 + layer, boost_frac=0.01, fused_call=True)
        n_diff += r["n_diff"]
        if layer == 15:
            hidden = synth.hidden_states(4100, S, 4096, "bf16")
            sel = TspSelector(S, W, POOL, k_tsp, 4096, "bf16")
            idx, hout = sel.run(r["comp"].buf.scores_raw, to_device(hidden, "bf16"))
            torch.cuda.synchronize()
            g = idx.cpu().numpy()
            idx_o = O.tsp_select(r["raw_o"], S, W, POOL, k_tsp)
            pooled_o = O.tsp_pooled(r["raw_o"], S, W, POOL)
            kth = np.sort(pooled_o)[::-1][k_tsp - 1]
            diff = set(g[:k_tsp].tolist()) ^ set(idx_o[:k_tsp].tolist())
            assert all(abs(pooled_o[j] - kth) <= 1e-5 * kth for j in diff)
            assert np.array_equal(from_device(hout), O.tsp_gather(hidden, g))
        del r
    log_parity(dict(what="fastkv_chain", schedule=schedule, layers=L, budgets=[int(b) for b in budgets],
                    tie_band_index_differences=n_diff))


@pytest.mark.parametrize("fused", [False, True])
def test_ragged_16_sequences(fused):
    lens = synth.ragged_lengths(1005, 16, 4096, 65536)
    r = run_and_check_compress("bf16", lens, N_H, N_KV, D, W, POOL, 1024, seed=1005, boost_frac=0.01,
                               fused_call=fused)
    cb = O.budget_offsets(lens, 1024)
    q = synth.decode_queries(1013, 16, N_H, D, "bf16")
    run_and_check_decode("bf16", q, from_device(r["comp"].buf.k_c), from_device(r["comp"].buf.v_c), cb[:-1],
                         np.diff(cb), N_KV)
