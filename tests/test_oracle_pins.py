"""Pins of the fp64 oracle to facts that do not come from the oracle itself:
the pages' worked example, closed forms, invariants, brute force on tiny
inputs, and library routines for the special cases that reduce to them."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import kvc_oracle as O
from kv_cache_compression_score_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(a):
    return np.asarray(a, dtype=np.float32)


# ---------------------------------------------------------------------------
# cache-size formula: the pages' worked example
# ---------------------------------------------------------------------------
def test_cache_bytes_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "cache_bytes.json")))
    for c in g["cases"]:
        n = c.get("n_seqs", 1)
        assert n * O.cache_bytes(c["L"], c["S"], c["n_kv"], c["d_h"], c["b"]) == c["bytes"], c["what"]
    wk = g["weak"]
    assert O.cache_bytes(wk["L"], wk["S"], wk["n_kv"], wk["d_h"], wk["b"]) == wk["gib"] * 2**30


# ---------------------------------------------------------------------------
# stored inputs: exact widening of bf16 bit patterns
# ---------------------------------------------------------------------------
# bf16 is the top half of an IEEE binary32: sign, 8 exponent bits, 7 mantissa
# bits.  Each pattern below is decoded by hand from that definition.
BF16_CASES = [
    (0x3F80, 1.0),                      # exponent 127, mantissa 0
    (0xC000, -2.0),                     # sign, exponent 128
    (0xC040, -3.0),                     # exponent 128, mantissa 0b1000000 -> 1.5 * 2
    (0x4049, 3.140625),                 # exponent 128, mantissa 0b1001001 -> (1 + 73/128) * 2
    (0x3E80, 0.25),                     # exponent 125
    (0x0001, 2.0 ** -133),              # smallest subnormal: 2^-126 * 2^-7
    (0x007F, 127 * 2.0 ** -133),        # largest subnormal
    (0x0080, 2.0 ** -126),              # smallest normal
    (0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127),   # largest finite
    (0x8000, -0.0),
    (0x0000, 0.0),
    (0x7F80, math.inf),
    (0xFF80, -math.inf),
]


def test_bf16_widening_hand_decoded_patterns():
    bits = np.array([b for b, _ in BF16_CASES], dtype=np.uint16)
    got = O.to_f64(bits, "bf16")
    for (b, want), g in zip(BF16_CASES, got):
        assert g == want and math.copysign(1.0, g) == math.copysign(1.0, want), f"0x{b:04X}: {g!r} != {want!r}"
    nan = O.to_f64(np.array([0x7FC0, 0xFFC1], dtype=np.uint16), "bf16")
    assert np.all(np.isnan(nan))


def test_bf16_widening_matches_torch_on_every_pattern():
    """All 65536 patterns against torch's own bf16 -> float64 conversion of
    the same bits (an implementation that shares nothing with the oracle)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = O.to_f64(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~fin)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))


def test_f32_widening_is_the_identity_on_values():
    x = np.array([1.0, -2.5, 2.0 ** -149, 3.4028234663852886e38, -0.0], dtype=np.float32)
    got = O.to_f64(x, "f32")
    assert np.array_equal(got, np.array([1.0, -2.5, 2.0 ** -149, 3.4028234663852886e38, -0.0]))
    assert math.copysign(1.0, got[4]) == -1.0


# ---------------------------------------------------------------------------
# scoring: closed forms
# ---------------------------------------------------------------------------
def _batch(lengths, n_h, n_kv, d, w, seed=7, dtype="f32"):
    return synth.packed_batch(seed, lengths, n_h, n_kv, d, w, dtype)


@pytest.mark.parametrize("lengths,n_h,n_kv,w", [([40], 4, 2, 5), ([33, 17, 9], 6, 3, 4), ([12], 2, 2, 12)])
def test_zero_keys_closed_form(lengths, n_h, n_kv, w):
    """K = 0: every visible logit is 0, so row i spreads 1/(P+i+1) over its
    P+i+1 visible keys; raw is G * sum_{i >= max(0, j-P)} 1/(P+i+1)."""
    d = 8
    bt = _batch(lengths, n_h, n_kv, d, w)
    k = np.zeros_like(bt["k"])
    raw = O.raw_scores(bt["q_win"], k, bt["cu_seqlens"], n_h, n_kv, w, "f32")
    G = n_h // n_kv
    for b, L in enumerate(lengths):
        t0 = bt["cu_seqlens"][b]
        P = L - w
        for j in range(L):
            first_row = max(0, j - P)
            expect = G * sum(1.0 / (P + i + 1) for i in range(first_row, w))
            np.testing.assert_allclose(raw[:, t0 + j], expect, rtol=1e-13)
    # Q = 0 gives the same closed form
    raw_q0 = O.raw_scores(np.zeros_like(bt["q_win"]), bt["k"], bt["cu_seqlens"], n_h, n_kv, w, "f32")
    np.testing.assert_allclose(raw_q0, raw, rtol=1e-13)


def test_row_stats_zero_keys():
    """K = 0: m = 0 and l = number of visible keys = P + i + 1."""
    L, w, n_h, n_kv = 30, 6, 4, 2
    bt = _batch([L], n_h, n_kv, 8, w)
    m, l = O.row_stats(bt["q_win"], np.zeros_like(bt["k"]), bt["cu_seqlens"], n_h, n_kv, w, "f32")
    assert np.all(m == 0.0)
    np.testing.assert_array_equal(l[0], np.broadcast_to(L - w + 1 + np.arange(w), (n_h, w)))


def test_scale_two_key_closed_form():
    """One row, two visible keys: z1 = scale*a, z2 = 0, so p1 = 1/(1+exp(-scale*a))."""
    d, a, scale = 4, 3.0, 0.37
    q = np.zeros((1, 1, d)); q[0, 0, 0] = a
    k = np.zeros((2, d)); k[0, 0] = 1.0
    pi, m, l = O.window_probs(q, k, 1, scale)
    np.testing.assert_allclose(pi[0, 0, 0], 1.0 / (1.0 + math.exp(-scale * a)), rtol=1e-15)
    np.testing.assert_allclose(m[0, 0], scale * a, rtol=1e-15)


def test_probability_mass_invariant():
    """Each window row is a probability distribution: summed over all visible
    keys (prefix and window) the raw scores of a KV head total G * w."""
    lengths, n_h, n_kv, w = [70, 41], 8, 2, 6
    bt = _batch(lengths, n_h, n_kv, 16, w, seed=3)
    raw = O.raw_scores(bt["q_win"], bt["k"], bt["cu_seqlens"], n_h, n_kv, w, "f32")
    cu = bt["cu_seqlens"]
    for b in range(len(lengths)):
        s = raw[:, cu[b]:cu[b + 1]].sum(axis=1)
        np.testing.assert_allclose(s, (n_h // n_kv) * w, rtol=1e-12)


def test_brute_force_loops_tiny():
    """Pure-Python loops (math.exp, explicit causal test) on a tiny ragged batch."""
    lengths, n_h, n_kv, w, d = [9, 6], 4, 2, 3, 5
    bt = _batch(lengths, n_h, n_kv, d, w, seed=11)
    scale = 0.41
    raw = O.raw_scores(bt["q_win"], bt["k"], bt["cu_seqlens"], n_h, n_kv, w, "f32", scale)
    q = bt["q_win"].astype(np.float64)
    k = bt["k"].astype(np.float64)
    G = n_h // n_kv
    for b, L in enumerate(lengths):
        t0 = int(bt["cu_seqlens"][b])
        for h in range(n_kv):
            acc = [0.0] * L
            for g in range(G):
                for i in range(w):
                    row_pos = L - w + i
                    zs = []
                    for j in range(L):
                        if j <= row_pos:
                            zs.append(scale * sum(q[b * w + i, h * G + g, e] * k[t0 + j, h, e] for e in range(d)))
                    mx = max(zs)
                    den = sum(math.exp(z - mx) for z in zs)
                    for j, z in enumerate(zs):
                        acc[j] += math.exp(z - mx) / den
            np.testing.assert_allclose(raw[h, t0:t0 + L], acc, rtol=1e-12)


def test_gqa_contiguous_mapping():
    """Query heads 0..G-1 use KV head 0 (contiguous groups).  Heads of group 0
    point at a spike key of KV head 0 only; group 1 at a spike of KV head 1."""
    L, w, d, n_h, n_kv = 40, 4, 8, 4, 2
    k = np.zeros((L, n_kv, d), dtype=np.float32)
    k[5, 0, 0] = 30.0            # spike of KV head 0 along e0
    k[20, 1, 1] = 30.0           # spike of KV head 1 along e1
    q = np.zeros((w, n_h, d), dtype=np.float32)
    q[:, 0:2, 0] = 1.0           # group 0 -> e0
    q[:, 2:4, 1] = 1.0           # group 1 -> e1
    raw = O.raw_scores(q, k, np.array([0, L]), n_h, n_kv, w, "f32", scale=1.0)
    assert raw[0, 5] > 0.99 * 2 * w and raw[1, 20] > 0.99 * 2 * w
    assert raw[0, 20] < 0.01 and raw[1, 5] < 0.01


# ---------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------
def test_pool_matches_torch_maxpool():
    x = synth.random_scores(5, (300,)).astype(np.float64)
    for pk in (1, 3, 7, 9):
        ref = torch.nn.functional.max_pool1d(torch.tensor(x)[None, None], pk, stride=1,
                                             padding=(pk - 1) // 2)[0, 0].numpy()
        np.testing.assert_array_equal(O.maxpool1d_same(x, pk), ref)


def test_spike_plateau_and_window_excluded():
    """A dominant prefix key j* gives a pooled plateau of width 7 (clipped to the
    prefix); a dominant window key does not leak into the pooled prefix."""
    L, w, d, n_h, n_kv, pk = 64, 8, 8, 2, 1, 7
    P = L - w
    for jstar in (0, 2, 30, P - 2, P - 1):
        k = np.zeros((L, n_kv, d), dtype=np.float32)
        k[jstar, 0, 0] = 40.0
        q = np.zeros((w, n_h, d), dtype=np.float32); q[:, :, 0] = 1.0
        cu = np.array([0, L])
        raw = O.raw_scores(q, k, cu, n_h, n_kv, w, "f32", scale=1.0)
        pooled = O.pool_prefix(raw, cu, w, pk)
        hot = np.where(pooled[0, :P] > 0.9 * n_h * w)[0]
        np.testing.assert_array_equal(hot, np.arange(max(0, jstar - 3), min(P, jstar + 4)))
        assert np.all(np.isinf(pooled[0, P:]))
    # spike on the first window key: visible to every window row, never pooled into the prefix
    k = np.zeros((L, n_kv, d), dtype=np.float32); k[P, 0, 0] = 40.0
    q = np.zeros((w, n_h, d), dtype=np.float32); q[:, :, 0] = 1.0
    raw = O.raw_scores(q, k, np.array([0, L]), n_h, n_kv, w, "f32", scale=1.0)
    pooled = O.pool_prefix(raw, np.array([0, L]), w, pk)
    assert raw[0, P] > 0.99 * n_h * w
    assert pooled[0, :P].max() < 1e-6


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------
def _brute_topk(scores, k_sel):
    """Among all k_sel-subsets: maximise the descending score vector, then take
    the lexicographically smallest index tuple (lowest-index tie rule)."""
    best_key, best = None, None
    for sub in itertools.combinations(range(len(scores)), k_sel):
        key = (tuple(sorted((scores[i] for i in sub), reverse=True)), tuple(-i for i in sub))
        if best_key is None or key > best_key:
            best_key, best = key, sub
    return np.array(best, dtype=np.int64)


def test_topk_brute_force_with_ties():
    for seed in range(12):
        n = 6 + seed % 7
        s = synth.random_scores(seed, (n,), n_levels=3).astype(np.float64)
        for k_sel in range(0, n + 1):
            np.testing.assert_array_equal(O.topk_prefix(s, k_sel), _brute_topk(s, k_sel))


def test_select_one_brute_force():
    for seed in range(8):
        L, w = 9 + seed % 5, 2 + seed % 2
        s = synth.random_scores(100 + seed, (L,), n_levels=4).astype(np.float64)
        pooled = O.maxpool1d_same(s[:L - w], 3)
        for budget in range(w, L + 2):
            got = O.select_one(pooled, L, w, budget)
            if budget >= L:
                np.testing.assert_array_equal(got, np.arange(L))
                continue
            expect = np.concatenate([_brute_topk(pooled, budget - w), np.arange(L - w, L)])
            np.testing.assert_array_equal(got, expect)


def test_select_invariants_and_edges():
    lengths, n_h, n_kv, w, B = [50, 33, 12], 4, 2, 6, 20
    bt = _batch(lengths, n_h, n_kv, 8, w, seed=21)
    cu = bt["cu_seqlens"]
    raw = O.raw_scores(bt["q_win"], bt["k"], cu, n_h, n_kv, w, "f32")
    pooled = O.pool_prefix(raw, cu, w, 7)
    idx = O.select_topk(pooled, cu, w, B)
    cb = O.budget_offsets(lengths, B)
    assert idx.shape == (n_kv, cb[-1])
    for b, L in enumerate(lengths):
        seg = idx[:, cb[b]:cb[b + 1]]
        for h in range(n_kv):
            assert np.all(np.diff(seg[h]) > 0)                      # ascending, distinct
            assert set(range(L - w, L)) <= set(seg[h].tolist())     # window always kept
            if B >= L:
                np.testing.assert_array_equal(seg[h], np.arange(L))
    # all scores equal (K = 0): the lowest prefix positions win
    raw0 = O.raw_scores(bt["q_win"], np.zeros_like(bt["k"]), cu, n_h, n_kv, w, "f32")
    idx0 = O.select_topk(O.pool_prefix(raw0, cu, w, 7), cu, w, B)
    np.testing.assert_array_equal(idx0[0, :B], np.concatenate([np.arange(B - w), np.arange(50 - w, 50)]))
    with pytest.raises(ValueError):
        O.select_one(np.zeros(10), 14, 4, 3)
    with pytest.raises(ValueError):
        O.maxpool1d_same(np.zeros(5), 4)


# ---------------------------------------------------------------------------
# gather + decode
# ---------------------------------------------------------------------------
def test_gather_bytes_and_identity():
    lengths, n_kv, w, B = [20, 7], 2, 3, 10
    bt = _batch(lengths, 4, n_kv, 8, w, seed=5, dtype="bf16")
    cu = bt["cu_seqlens"]
    idx = np.concatenate([np.stack([np.arange(10)[::-1] % 20] * n_kv), np.stack([np.arange(7)] * n_kv)], axis=1)
    kc, vc = O.gather_kv(bt["k"], bt["v"], idx, cu, B)
    assert kc.dtype == np.uint16
    for t in range(10):
        np.testing.assert_array_equal(kc[t], bt["k"][idx[0, t]])
    np.testing.assert_array_equal(kc[10:], bt["k"][20:27])
    np.testing.assert_array_equal(vc[10:], bt["v"][20:27])


def test_decode_closed_forms():
    n_h, n_kv, d, n = 4, 2, 8, 13
    q = synth.decode_queries(1, 1, n_h, d, "f32")
    rng_k, rng_v = synth.keys_values(2, 0, n, n_kv, d, "f32")
    off, ln = np.array([0]), np.array([n])
    # equal V rows -> that row
    v_eq = np.broadcast_to(rng_v[3:4], rng_v.shape).copy()
    out = O.gqa_decode(q, rng_k, v_eq, off, ln, n_kv, "f32")
    for qh in range(n_h):
        np.testing.assert_allclose(out[0, qh], rng_v[3, qh // 2].astype(np.float64), rtol=1e-14)
    # K = 0 -> mean of V
    out = O.gqa_decode(q, np.zeros_like(rng_k), rng_v, off, ln, n_kv, "f32")
    for qh in range(n_h):
        np.testing.assert_allclose(out[0, qh], rng_v[:, qh // 2].astype(np.float64).mean(0), rtol=1e-12)
    # permuting cache rows leaves the output unchanged
    perm = np.array(synth.boosted_positions(9, 0, 0, n, 1.0))[::-1]
    a = O.gqa_decode(q, rng_k, rng_v, off, ln, n_kv, "f32")
    b = O.gqa_decode(q, rng_k[perm], rng_v[perm], off, ln, n_kv, "f32")
    np.testing.assert_allclose(a, b, rtol=1e-12)
    # two rows, closed form with the scale
    k2 = np.zeros((2, 1, 2), dtype=np.float32); k2[0, 0, 0] = 1.0
    v2 = np.zeros((2, 1, 2), dtype=np.float32); v2[0, 0, 1] = 1.0; v2[1, 0, 0] = 1.0
    q2 = np.zeros((1, 1, 2), dtype=np.float32); q2[0, 0, 0] = 2.0
    o2 = O.gqa_decode(q2, k2, v2, [0], [2], 1, "f32", scale=0.5)
    p0 = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(o2[0, 0], [1 - p0, p0], rtol=1e-15)
    # empty cache -> 0
    assert np.all(O.gqa_decode(q, rng_k, rng_v, off, np.array([0]), n_kv, "f32") == 0)


def test_decode_matches_torch_sdpa_and_identity_budget():
    """B >= S: selection is the identity and decode over the compact cache
    equals full attention (torch fp64 scaled_dot_product_attention)."""
    L, n_h, n_kv, d, w = 37, 8, 2, 16, 4
    bt = _batch([L], n_h, n_kv, d, w, seed=31, dtype="bf16")
    cu = bt["cu_seqlens"]
    raw = O.raw_scores(bt["q_win"], bt["k"], cu, n_h, n_kv, w, "bf16")
    idx = O.select_topk(O.pool_prefix(raw, cu, w, 7), cu, w, L + 5)
    np.testing.assert_array_equal(idx, np.broadcast_to(np.arange(L), (n_kv, L)))
    kc, vc = O.gather_kv(bt["k"], bt["v"], idx, cu, L + 5)
    np.testing.assert_array_equal(kc, bt["k"])
    q = synth.decode_queries(4, 1, n_h, d, "bf16")
    out = O.gqa_decode(q, kc, vc, [0], [L], n_kv, "bf16")
    G = n_h // n_kv
    qt = torch.tensor(O.to_f64(q, "bf16"))[:, :, None, :]                       # [1, n_h, 1, d]
    kt = torch.tensor(O.to_f64(bt["k"], "bf16")).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    vt = torch.tensor(O.to_f64(bt["v"], "bf16")).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0].numpy()
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-14)


def test_window_probs_match_torch_softmax():
    """The causal window softmax is torch's fp64 softmax over the visible keys."""
    bt = _batch([25], 4, 2, 8, 5, seed=41)
    qf = O.to_f64(bt["q_win"], "f32"); kf = O.to_f64(bt["k"], "f32")
    pi, _, _ = O.window_probs(np.transpose(qf[:, 0:2], (1, 0, 2)), kf[:, 0], 5, 0.3)
    z = 0.3 * torch.einsum("igd,jd->gij", torch.tensor(qf[:, 0:2]), torch.tensor(kf[:, 0]))
    mask = torch.ones(5, 25, dtype=torch.bool).tril(diagonal=20)
    ref = torch.softmax(z.masked_fill(~mask, float("-inf")), dim=-1).numpy()
    np.testing.assert_allclose(pi, ref, rtol=1e-13, atol=1e-300)


# ---------------------------------------------------------------------------
# TSP
# ---------------------------------------------------------------------------
def test_tsp_rates_and_ties():
    assert O.rate_count(0.2, 32768) == 6553
    assert O.rate_count(0.1, 32768) == 3276
    S, w = 40, 4
    raw = np.ones((3, S))
    idx = O.tsp_select(raw, S, w, 7, 10)
    np.testing.assert_array_equal(idx, np.concatenate([np.arange(10), np.arange(36, 40)]))
    with pytest.raises(ValueError):
        O.tsp_select(raw, S, w, 7, S - w + 1)


def test_tsp_sums_heads_before_pooling():
    """Disjoint spikes in different heads both survive the head sum; a spike
    smaller than another head's plateau still wins where it is alone."""
    S, w = 60, 4
    raw = np.zeros((2, S))
    raw[0, 10] = 5.0
    raw[1, 40] = 3.0
    pooled = O.tsp_pooled(raw, S, w, 3)
    np.testing.assert_array_equal(np.where(pooled == 5.0)[0], [9, 10, 11])
    np.testing.assert_array_equal(np.where(pooled == 3.0)[0], [39, 40, 41])
    idx = O.tsp_select(raw, S, w, 3, 6)
    np.testing.assert_array_equal(idx, [9, 10, 11, 39, 40, 41, 56, 57, 58, 59])
    hidden = synth.hidden_states(3, S, 16, "bf16")
    np.testing.assert_array_equal(O.tsp_gather(hidden, idx), hidden[idx])
    # two heads agreeing on a moderate token outrank one head's larger spike
    raw = np.zeros((2, S))
    raw[0, 20] = raw[1, 20] = 3.0
    raw[0, 45] = 5.0
    np.testing.assert_array_equal(O.tsp_select(raw, S, w, 1, 1), [20, 56, 57, 58, 59])


# ---------------------------------------------------------------------------
# generator sanity (inputs, not the method)
# ---------------------------------------------------------------------------
def test_generators_deterministic_and_normal():
    a = synth.normal_tensor(1, synth.T_K, 0, (1000, 4), "f32")
    b = synth.normal_tensor(1, synth.T_K, 0, (1000, 4), "f32")
    np.testing.assert_array_equal(a, b)
    assert abs(a.mean()) < 0.05 and abs(a.std() - 1) < 0.05
    bits = synth.normal_tensor(1, synth.T_K, 0, (1000, 4), "bf16")
    back = synth.bf16_bits_to_f32(bits)
    assert np.max(np.abs(back - a) / np.maximum(np.abs(a), 1e-30)) <= 2.0 ** -8
    lens = synth.ragged_lengths(1005, 16, 4096, 65536)
    assert lens.min() >= 4096 and lens.max() <= 65536
    pos = synth.boosted_positions(1002, 0, 0, 32768, 0.01)
    assert len(pos) == 327 and len(np.unique(pos)) == 327


# ---------------------------------------------------------------------------
# quantised compact cache (int8 codes, one float32 scale per (row, head))
# ---------------------------------------------------------------------------
def test_quantize_exact_power_of_two_rows():
    """max|x| = 127 * 2^e and every element a multiple of 2^e: the scale is
    exactly 2^e, the codes are x / 2^e and dequantisation gives x back."""
    for e in (-7, 0, 3):
        codes = np.array([[127, -5, 0, 64, -127, 1], [-127, 2, 3, -4, 100, 7]], dtype=np.int64)
        x = (codes * 2.0 ** e).astype(np.float32)
        q, s = O.quantize_rows_int8(x)
        assert q.dtype == np.int8 and s.dtype == np.float32
        np.testing.assert_array_equal(s, [2.0 ** e, 2.0 ** e])
        np.testing.assert_array_equal(q, codes)
        np.testing.assert_array_equal(O.dequantize_rows(q, s), x.astype(np.float64))


def test_quantize_rounds_half_to_even_and_clips():
    """Scale 1 (max|x| = 127): x / scale = x, so the codes are x rounded half
    to even -- 2.5 -> 2, -2.5 -> -2, 3.5 -> 4, 0.5 -> 0, -0.5 -> -0."""
    x = np.array([[127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 126.49, -126.51]], dtype=np.float32)
    q, s = O.quantize_rows_int8(x)
    assert s[0] == 1.0
    np.testing.assert_array_equal(q[0], [127, 2, -2, 4, 0, 0, 126, -127])


def test_quantize_zero_row_and_error_bound():
    x = synth.normal_tensor(77, synth.T_K, 0, (64, 128), "f32")
    x[5] = 0.0
    q, s = O.quantize_rows_int8(x)
    assert s[5] == 0.0 and np.all(q[5] == 0)
    assert np.all(np.abs(q.astype(np.int64)) <= 127)
    for r in range(64):
        if r == 5:
            continue
        j = np.argmax(np.abs(x[r]))
        assert abs(int(q[r, j])) == 127                      # the largest element maps to +-127
        err = np.abs(x[r].astype(np.float64) - O.dequantize_rows(q[r:r + 1], s[r:r + 1])[0])
        assert err.max() <= 0.5 * float(s[r]) * (1 + 2.0 ** -20)   # half a quantisation step
    # scaling a row by a power of two scales the scale and keeps the codes
    q2, s2 = O.quantize_rows_int8((x * np.float32(8.0)).astype(np.float32))
    np.testing.assert_array_equal(q2, q)
    np.testing.assert_array_equal(s2, s * np.float32(8.0))


def test_gather_q8_is_gather_then_quantize_per_head_row():
    lengths, n_kv, d, w, B = [40, 9], 2, 16, 4, 12
    bt = synth.packed_batch(81, lengths, 4, n_kv, d, w, "bf16")
    idx = synth.index_lists(82, lengths, n_kv, B).astype(np.int64)
    kq, vq, ks, vs = O.gather_kv_q8(bt["k"], bt["v"], idx, bt["cu_seqlens"], B, "bf16")
    kc, vc = O.gather_kv(bt["k"], bt["v"], idx, bt["cu_seqlens"], B)
    assert kq.shape == kc.shape and ks.shape == (n_kv, kc.shape[0])
    for t in range(kc.shape[0]):
        for h in range(n_kv):
            row = O.to_f64(kc[t, h], "bf16").astype(np.float32)
            amax = np.max(np.abs(row))
            assert ks[h, t] == np.float32(amax) / np.float32(127)
            np.testing.assert_array_equal(kq[t, h], np.clip(np.rint(row / ks[h, t]), -127, 127))


def test_decode_q8_lossless_cache_equals_plain_decode():
    """A cache whose rows hold integers in [-127, 127] with +-127 present is
    quantised without loss (scale 1), so decode over it equals decode over
    the plain float32 cache; scaling the cache by 2^-4 scales only the
    scales."""
    n_h, n_kv, d, rows = 8, 2, 16, 50
    u = synth.uniform_u64(synth.stream_key(91, synth.T_K, 0), rows * n_kv * d)
    ints = ((u % np.uint64(255)).astype(np.int64) - 127).reshape(rows, n_kv, d)
    ints[:, :, 0] = 127
    kf = (ints * 2.0 ** -4).astype(np.float32)
    vf = (ints[::-1] * 2.0 ** -4).astype(np.float32)
    kq, ks = O.quantize_rows_int8(kf)
    vq, vs = O.quantize_rows_int8(vf)
    assert np.all(ks == 2.0 ** -4) and np.all(vs == 2.0 ** -4)
    q = synth.decode_queries(92, 3, n_h, d, "bf16")
    offs, lens = [0, 10, 0], [50, 40, 1]
    got = O.gqa_decode_q8(q, kq, vq, ks.T, vs.T, offs, lens, n_kv, "bf16")
    ref = O.gqa_decode(q, kf, vf, offs, lens, n_kv, "bf16", cache_dtype="f32")
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------------------
# PyramidKV per-layer budgets
# ---------------------------------------------------------------------------
def test_pyramid_budgets_shape_and_mean():
    b = O.pyramid_budgets(32, 3276, 1000)
    assert b[0] == 2 * 3276 - 1000 and b[-1] == 1000          # the two ends
    assert np.all(np.diff(b) <= 0)                            # never grows with depth
    steps = -np.diff(b)
    assert steps.max() - steps.min() <= 1                     # linear up to rounding
    assert 32 * 3276 <= b.sum() < 32 * 3276 + 32              # mean B_avg, rounded up by < 1 per layer
    np.testing.assert_array_equal(O.pyramid_budgets(8, 100, 100), np.full(8, 100))   # flat schedule
    np.testing.assert_array_equal(O.pyramid_budgets(1, 77, 10), [77])
    np.testing.assert_array_equal(O.pyramid_budgets(3, 10, 4), [16, 10, 4])           # by hand
    np.testing.assert_array_equal(O.pyramid_budgets(4, 10, 5), [15, 12, 9, 5])        # 15 - floor(10 l / 3)
    with pytest.raises(ValueError):
        O.pyramid_budgets(4, 10, 11)


# ---------------------------------------------------------------------------
# FreeKV decode-time retrieval
# ---------------------------------------------------------------------------
def test_freekv_cosine_cases_by_hand():
    """Hand-made query pairs: equal (cos 1), opposite (-1), orthogonal (0),
    45 degrees (1/sqrt 2), a zero vector (0 by convention)."""
    d = 4
    cur = np.array([[[1, 0, 0, 0], [0, 2, 0, 0], [1, 0, 0, 0], [3, 0, 0, 0], [0, 0, 0, 0], [1, 1, 0, 0]]],
                   dtype=np.float32)
    prev = np.array([[[2, 0, 0, 0], [0, -1, 0, 0], [0, 0, 5, 0], [1, 1, 0, 0], [1, 0, 0, 0], [1, 1, 0, 0]]],
                    dtype=np.float32)
    flags, cos = O.freekv_flags(cur, prev, 3, 0.5, "f32")        # G = 2: heads (0,1), (2,3), (4,5)
    np.testing.assert_allclose(cos[0], [1, -1, 0, 1 / math.sqrt(2), 0, 1], rtol=1e-15, atol=1e-15)
    np.testing.assert_array_equal(flags[0], [True, True, True])     # group minima -1, 0, 0
    flags, _ = O.freekv_flags(cur, prev, 6, 0.5, "f32")             # G = 1
    np.testing.assert_array_equal(flags[0], [False, True, True, False, True, False])
    assert d == cur.shape[-1]


def test_decode_query_scores_is_a_one_row_window():
    """A decode query after the cache scores keys exactly as an observation
    window of one row placed on the last cached position (which sees every
    key), and torch's fp64 softmax agrees."""
    lengths, n_h, n_kv, d = [30, 9], 4, 2, 8
    bt = _batch(lengths, n_h, n_kv, d, 1, seed=61, dtype="bf16")
    q = bt["q_win"].reshape(len(lengths), n_h, d)                  # one window row per sequence
    raw = O.decode_query_scores(q, bt["k"], bt["cu_seqlens"], n_kv, "bf16")
    raw_w = O.raw_scores(bt["q_win"], bt["k"], bt["cu_seqlens"], n_h, n_kv, 1, "bf16")
    np.testing.assert_allclose(raw, raw_w, rtol=1e-13, atol=1e-300)
    G = n_h // n_kv
    qt = torch.tensor(O.to_f64(q, "bf16"))
    kt = torch.tensor(O.to_f64(bt["k"], "bf16"))
    z = torch.einsum("gd,jd->gj", qt[0, 0:G], kt[0:30, 0]) / math.sqrt(d)
    np.testing.assert_allclose(raw[0, 0:30], torch.softmax(z, dim=1).sum(0).numpy(), rtol=1e-13)
    # K = 0: every key gets G / len
    raw0 = O.decode_query_scores(q, np.zeros_like(bt["k"]), bt["cu_seqlens"], n_kv, "bf16")
    np.testing.assert_allclose(raw0[:, :30], G / 30, rtol=1e-14)
    np.testing.assert_allclose(raw0[:, 30:], G / 9, rtol=1e-14)


def test_freekv_step_tau_extremes():
    """tau = -2: no head is corrected, the step is decode over the previous
    compact cache; tau = 2: every head is corrected, the step is a fresh
    score / select / gather with the current query followed by decode."""
    lengths, n_h, n_kv, d, w, B = [60, 45], 8, 2, 16, 4, 20
    bt = _batch(lengths, n_h, n_kv, d, w, seed=71, dtype="bf16")
    cu = bt["cu_seqlens"]
    q_prev = synth.decode_queries(72, 2, n_h, d, "bf16")
    q_cur = synth.decode_queries(73, 2, n_h, d, "bf16")
    idx_prev = O.select_topk(O.pool_prefix(O.decode_query_scores(q_prev, bt["k"], cu, n_kv, "bf16"), cu, w, 5),
                             cu, w, B)
    f, idx, kc, vc, out = O.freekv_step(q_cur, q_prev, bt["k"], bt["v"], cu, idx_prev, n_kv, w, 5, B, -2.0, "bf16")
    assert not f.any()
    np.testing.assert_array_equal(idx, idx_prev)
    kc_p, vc_p = O.gather_kv(bt["k"], bt["v"], idx_prev, cu, B)
    cb = O.budget_offsets(lengths, B)
    np.testing.assert_array_equal(out, O.gqa_decode(q_cur, kc_p, vc_p, cb[:-1], np.diff(cb), n_kv, "bf16"))
    f, idx, kc, vc, out = O.freekv_step(q_cur, q_prev, bt["k"], bt["v"], cu, idx_prev, n_kv, w, 5, B, 2.0, "bf16")
    assert f.all()
    fresh = O.select_topk(O.pool_prefix(O.decode_query_scores(q_cur, bt["k"], cu, n_kv, "bf16"), cu, w, 5), cu, w, B)
    np.testing.assert_array_equal(idx, fresh)
    # the same query twice: cos = 1, nothing below tau = 0.999
    f, idx, _, _, _ = O.freekv_step(q_cur, q_cur, bt["k"], bt["v"], cu, idx_prev, n_kv, w, 5, B, 0.999, "bf16")
    assert not f.any() and np.array_equal(idx, idx_prev)


# ---------------------------------------------------------------------------
# xKV cross-layer factorisation and selective reconstruction
# ---------------------------------------------------------------------------
def _low_rank_layers(seed, S, n_kv, d, W, rank, noise=0.0):
    """W layers whose keys share a rank-`rank` token basis (plus noise).  The
    factors are small integers, so without noise the stored float32 keys have
    exactly that rank."""
    U = np.round(2 * synth.normal_tensor(seed, synth.T_K, 0, (n_kv, S, rank), "f32").astype(np.float64))
    layers = []
    for l in range(W):
        M = np.round(2 * synth.normal_tensor(seed, synth.T_V, l + 1, (n_kv, rank, d), "f32").astype(np.float64))
        E = synth.normal_tensor(seed, synth.T_QDEC, l + 1, (n_kv, S, d), "f32").astype(np.float64)
        layers.append(np.transpose(U @ M + noise * E, (1, 0, 2)).astype(np.float32))   # [S, n_kv, d]
    return layers


def test_xkv_exact_for_low_rank_windows():
    """Keys of exact rank <= r are rebuilt exactly (Eckart-Young with no tail)."""
    S, n_kv, d, W, r = 60, 2, 8, 3, 5
    layers = _low_rank_layers(3, S, n_kv, d, W, 4)
    A, Vt = O.xkv_factorize(layers, r, "f32")
    idx = np.stack([np.arange(S)[::-1], np.arange(S)])
    for l in range(W):
        rec = O.xkv_reconstruct(A, Vt, l, d, idx)
        for h in range(n_kv):
            np.testing.assert_allclose(rec[:, h], layers[l][idx[h], h].astype(np.float64), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(np.einsum("hrk,hsk->hrs", Vt, Vt), np.broadcast_to(np.eye(r), (n_kv, r, r)),
                               atol=1e-12)


def test_xkv_error_is_the_singular_tail():
    """Noisy window: the reconstruction error of all rows equals the norm of
    the discarded singular values, and a single layer (W = 1) is the plain
    truncated SVD of that layer."""
    S, n_kv, d, W, r = 80, 2, 6, 4, 7
    layers = _low_rank_layers(5, S, n_kv, d, W, 5, noise=0.3)
    A, Vt = O.xkv_factorize(layers, r, "f32")
    idx = np.broadcast_to(np.arange(S), (n_kv, S))
    X = np.concatenate([l.astype(np.float64) for l in layers], axis=2)
    rec = np.concatenate([O.xkv_reconstruct(A, Vt, l, d, idx) for l in range(W)], axis=2)
    for h in range(n_kv):
        sv = np.linalg.svd(X[:, h], compute_uv=False)
        np.testing.assert_allclose(np.linalg.norm(X[:, h] - rec[:, h]), np.sqrt(np.sum(sv[r:] ** 2)), rtol=1e-9)
    r1 = 4
    A1, Vt1 = O.xkv_factorize(layers[:1], r1, "f32")
    for h in range(n_kv):
        u, sv, vt = np.linalg.svd(layers[0][:, h].astype(np.float64), full_matrices=False)
        np.testing.assert_allclose(A1[h] @ Vt1[h], (u[:, :r1] * sv[:r1]) @ vt[:r1], atol=1e-9)


def test_xkv_window_bytes():
    # per head S*r basis + r*W*d blocks; 8x smaller than the window's keys for S=32768, d=128, W=4, r=64 (fp32 basis
    # against bf16 keys: 4x)
    assert O.xkv_window_bytes(32768, 8, 128, 4, 64, 4, 4) == 8 * (32768 * 64 * 4 + 64 * 512 * 4)
    assert 4 * 32768 * 8 * 128 * 2 / O.xkv_window_bytes(32768, 8, 128, 4, 64, 2, 4) > 7.5
