"""FreeKV decode steps on the GPU against the oracle (FreeKV, technical
summary 2.A: reuse the previous step's tokens; heads whose query drifted
below tau are scored, selected and gathered again before attention).

Per step: the flags agree with the oracle's except for heads whose smallest
cosine lies within 1e-5 of tau; with the GPU's flags, the index lists of the
re-selected heads match the oracle's selection within the tie band, the other
heads' lists are unchanged, every compact row is the byte copy its index
names, and decode matches the oracle over the GPU's compact cache."""
import numpy as np
import pytest
import torch

from kv_cache_compression_score_b200 import synth
from kv_cache_compression_score_b200.runner import FreeKvStep, from_device, to_device
from oracle import kvc_oracle as O
from parity_helpers import DECODE_ATOL, assert_selection_matches, log_parity

pytestmark = pytest.mark.gpu
TAU_BAND = 1e-5


@pytest.fixture(autouse=True, scope="module")
def _built():
    from kv_cache_compression_score_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _check_step(fk, bt, q_cur, q_prev, idx_before, tau, n_kv, w, pool_k, budget):
    lengths = bt["seqlens"]
    cu = bt["cu_seqlens"]
    flags_g = fk.reselected.cpu().numpy().astype(bool)
    flags_o, cos = O.freekv_flags(q_cur, q_prev, n_kv, tau, "bf16")
    G = q_cur.shape[1] // n_kv
    cmin = cos.reshape(cos.shape[0], n_kv, G).min(axis=2)
    differ = flags_g != flags_o
    assert np.all(np.abs(cmin[differ] - tau) <= TAU_BAND), "re-selection flags differ away from tau"
    idx_g = fk.idx.cpu().numpy()
    cb = O.budget_offsets(lengths, budget)
    # heads kept: index lists unchanged
    for b in range(len(lengths)):
        for h in range(n_kv):
            if not flags_g[b, h]:
                np.testing.assert_array_equal(idx_g[h, cb[b]:cb[b + 1]], idx_before[h, cb[b]:cb[b + 1]])
    # re-selected heads: the oracle's selection from the current query, within the tie band
    raw_o = O.decode_query_scores(q_cur, bt["k"], cu, n_kv, "bf16")
    pooled_o = O.pool_prefix(raw_o, cu, w, pool_k)
    fresh_o = O.select_topk(pooled_o, cu, w, budget)
    mixed = idx_before.astype(np.int64).copy()
    for b in range(len(lengths)):
        for h in range(n_kv):
            if flags_g[b, h]:
                mixed[h, cb[b]:cb[b + 1]] = fresh_o[h, cb[b]:cb[b + 1]]
    n_diff = assert_selection_matches(idx_g, mixed, pooled_o, lengths, w, budget)
    # compact rows: byte copies of the rows the GPU's index lists name
    kc_o, vc_o = O.gather_kv(bt["k"], bt["v"], idx_g.astype(np.int64), cu, budget)
    assert np.array_equal(from_device(fk.k_c), kc_o) and np.array_equal(from_device(fk.v_c), vc_o)
    out_o = O.gqa_decode(q_cur, kc_o, vc_o, cb[:-1], np.diff(cb), n_kv, "bf16")
    err = float(np.abs(fk.out.cpu().numpy() - out_o).max())
    log_parity(dict(what="freekv_step", n_seqs=len(lengths), tau=tau, reselected=int(flags_g.sum()),
                    heads=int(flags_g.size), flag_band_differences=int(differ.sum()),
                    tie_band_index_differences=n_diff, max_abs_err=err))
    assert err <= DECODE_ATOL["bf16"], err
    return flags_g, idx_g


def _run_steps(lengths, n_h, n_kv, d, w, pool_k, budget, seed, n_steps=3, tau=0.9):
    bt = synth.packed_batch(seed, lengths, n_h, n_kv, d, w, "bf16", 0.01)
    k, v = to_device(bt["k"], "bf16"), to_device(bt["v"], "bf16")
    fk = FreeKvStep(lengths, n_h, n_kv, d, w, pool_k, budget, tau)
    q_prev = synth.decode_queries(seed + 1, len(lengths), n_h, d, "bf16")
    # first step: every head selects (tau above any cosine)
    fk.step(to_device(q_prev, "bf16"), to_device(q_prev, "bf16"), k, v, tau=2.0)
    torch.cuda.synchronize()
    idx_before = np.zeros((n_kv, int(O.budget_offsets(lengths, budget)[-1])), dtype=np.int32)
    flags, idx = _check_step(fk, bt, q_prev, q_prev, idx_before, 2.0, n_kv, w, pool_k, budget)
    assert flags.all()
    counts = []
    for s in range(n_steps):
        q_cur = synth.drifted_queries(seed + 10 + s, q_prev, "bf16", group=n_h // n_kv)
        fk.step(to_device(q_cur, "bf16"), to_device(q_prev, "bf16"), k, v)
        torch.cuda.synchronize()
        flags, idx = _check_step(fk, bt, q_cur, q_prev, idx, tau, n_kv, w, pool_k, budget)
        counts.append(int(flags.sum()))
        q_prev = q_cur
    assert 0 < sum(counts) < n_steps * flags.size, counts   # some heads re-selected, some not
    # tau below every cosine: nothing re-selected, decode over the previous cache
    q_cur = synth.drifted_queries(seed + 99, q_prev, "bf16", group=n_h // n_kv)
    fk.step(to_device(q_cur, "bf16"), to_device(q_prev, "bf16"), k, v, tau=-2.0)
    torch.cuda.synchronize()
    flags, idx2 = _check_step(fk, bt, q_cur, q_prev, idx, -2.0, n_kv, w, pool_k, budget)
    assert not flags.any() and np.array_equal(idx2, idx)


@pytest.mark.parametrize("lengths,d,n_h,n_kv", [([3000, 1500, 777, 4096], 128, 32, 8), ([2100, 64], 64, 16, 2)])
def test_freekv_steps_small(lengths, d, n_h, n_kv):
    _run_steps(lengths, n_h, n_kv, d, 32, 7, 512, seed=5100 + d)


def test_freekv_steps_llama8b_batch16_s32k():
    """Decode batch 16 over full caches of S = 32768 (Llama-3-8B shape),
    budget 2048 per head."""
    _run_steps([32768] * 16, 32, 8, 128, 32, 7, 2048, seed=5200, n_steps=2)
