"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and compare with the fp64 oracle on the same inputs."""
import numpy as np
import torch

from kv_cache_compression_score_b200 import synth
from kv_cache_compression_score_b200.runner import Compressor, Decoder, from_device, to_device
from oracle import kvc_oracle as O

SCORE_RTOL = 1e-5          # scores, relative (all terms are positive sums)
SCORE_FLOOR = 1e-30        # below this both sides may flush to zero (fp32 subnormals)
DECODE_ATOL = {"f32": 1e-5, "bf16": 2e-3}
TIE_BAND = 1e-5            # selected sets may differ only within this relative band of the k-th score


def log_parity(rec):
    """Append one parity record (JSON line) to $KVC_PARITY_LOG when it is set,
    so a GPU run can keep the tie-band counts and error maxima of every case."""
    import json
    import os
    path = os.environ.get("KVC_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def assert_scores_close(got, ref, rtol=SCORE_RTOL, what="scores"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: inf pattern differs"
    assert np.array_equal(got[~fin], ref[~fin]), f"{what}: infinities differ"
    err = np.abs(got[fin] - ref[fin])
    tol = rtol * np.abs(ref[fin]) + SCORE_FLOOR
    bad = err > tol
    if bad.any():
        i = np.argmax(err / tol)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside rtol {rtol}; worst rel "
                             f"{(err / np.maximum(np.abs(ref[fin]), 1e-300))[i]:.3e} "
                             f"(got {got[fin][i]!r}, ref {ref[fin][i]!r})")


def max_rel(got, ref):
    ref = np.asarray(ref, dtype=np.float64)
    fin = np.isfinite(ref) & (np.abs(ref) > SCORE_FLOOR)
    return float(np.max(np.abs(np.asarray(got, np.float64)[fin] - ref[fin]) / np.abs(ref[fin]))) if fin.any() else 0.0


def assert_selection_matches(idx_gpu, idx_ora, pooled_ora, lengths, w, budget, band=TIE_BAND):
    """Equal sizes and order rules; the two sets may differ only on prefix
    tokens whose oracle pooled score lies within `band` (relative) of the
    k-th largest oracle score.  Returns the number of differing tokens."""
    lengths = np.asarray(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    cb = O.budget_offsets(lengths, budget)
    assert idx_gpu.shape == idx_ora.shape
    n_diff = 0
    for b, L in enumerate(lengths):
        for h in range(idx_gpu.shape[0]):
            g = idx_gpu[h, cb[b]:cb[b + 1]].astype(np.int64)
            o = idx_ora[h, cb[b]:cb[b + 1]]
            assert len(g) == min(budget, L)
            assert np.all(np.diff(g) > 0), "indices must be ascending and distinct"
            assert g.min(initial=0) >= 0 and g.max(initial=0) < L
            if budget >= L:
                np.testing.assert_array_equal(g, np.arange(L))
                continue
            P, k_sel = L - w, budget - w
            np.testing.assert_array_equal(g[k_sel:], np.arange(P, L))       # window always kept
            diff = set(g[:k_sel].tolist()) ^ set(o[:k_sel].tolist())
            if diff:
                s = pooled_ora[h, cu[b]:cu[b] + P]
                kth = np.sort(s)[::-1][k_sel - 1]
                for j in diff:
                    assert abs(s[j] - kth) <= band * kth, \
                        f"seq {b} head {h}: token {j} (score {s[j]!r}) outside the tie band of {kth!r}"
                n_diff += len(diff)
    return n_diff


def assert_gather_exact(comp, bt, idx_g, budget):
    """K_c / V_c against the oracle's byte copy of the rows named by the GPU's
    index lists (gather is exact given the indices), on every row."""
    kc_o, vc_o = O.gather_kv(bt["k"], bt["v"], idx_g.astype(np.int64), bt["cu_seqlens"], budget)
    kc_g, vc_g = from_device(comp.buf.k_c), from_device(comp.buf.v_c)
    assert kc_g.shape == kc_o.shape and vc_g.shape == vc_o.shape
    for name, g, o in (("K", kc_g, kc_o), ("V", vc_g, vc_o)):
        if not np.array_equal(g.view(np.uint8), o.view(np.uint8)):
            bad = np.argwhere(np.any(g.reshape(g.shape[0], g.shape[1], -1) != o.reshape(o.shape[0], o.shape[1], -1),
                                     axis=2))
            raise AssertionError(f"gathered {name} differs on {len(bad)} (slot, head) rows, first {bad[:4].tolist()}")


def upload_batch(bt, dtype):
    return to_device(bt["q_win"], dtype), to_device(bt["k"], dtype), to_device(bt["v"], dtype)


def run_and_check_compress(dtype, lengths, n_h, n_kv, d, w, pool_k, budget, seed, boost_frac=0.0, boost=3.0,
                           check_gather=True, repeat=1, fused_call=False):
    """Whole score -> select -> gather path on one seeded batch, every output
    compared with the oracle (after `repeat` runs on the same buffers).
    Returns a dict of the pieces for further checks."""
    bt = synth.packed_batch(seed, lengths, n_h, n_kv, d, w, dtype, boost_frac, boost)
    q, k, v = upload_batch(bt, dtype)
    comp = Compressor(dtype, lengths, n_h, n_kv, d, w, pool_k, budget)
    for _ in range(repeat):
        if fused_call:
            comp.compress(q, k, v)
        else:
            comp.run(q, k, v)
    torch.cuda.synchronize()
    assert comp.device_error_word() == 0
    # the per-(sequence, head) arrival counters are left at zero for the next call
    ctr = comp.buf.ws[256:256 + 32 * len(lengths) * n_kv].view(torch.int32)
    assert int(ctr.abs().sum().item()) == 0
    cu = bt["cu_seqlens"]
    raw_o = O.raw_scores(bt["q_win"], bt["k"], cu, n_h, n_kv, w, dtype)
    pooled_o = O.pool_prefix(raw_o, cu, w, pool_k)
    raw_g = comp.buf.scores_raw.cpu().numpy()
    pooled_g = comp.buf.scores.cpu().numpy()
    assert_scores_close(raw_g, raw_o, what="raw scores")
    assert_scores_close(pooled_g, pooled_o, what="pooled scores")
    idx_o = O.select_topk(pooled_o, cu, w, budget)
    idx_g = comp.buf.idx.cpu().numpy()
    n_diff = assert_selection_matches(idx_g, idx_o, pooled_o, lengths, w, budget)
    if check_gather:
        # the compact caches are bit-exact copies of the rows the GPU's own index
        # lists name: every row of every head and sequence is compared
        assert_gather_exact(comp, bt, idx_g, budget)
    n_rows = int(np.sum(np.minimum(np.asarray(lengths), budget))) * n_kv
    log_parity(dict(what="compress", dtype=dtype, n_seqs=len(lengths), T=int(np.sum(lengths)), budget=budget,
                    fused_call=fused_call, tie_band_index_differences=n_diff, retained_rows=n_rows,
                    gathered_rows_compared=n_rows if check_gather else 0,
                    max_rel_raw=max_rel(raw_g, raw_o), max_rel_pooled=max_rel(pooled_g, pooled_o)))
    # the tie band admits a few swaps among equal-looking scores, never a large share
    assert n_diff <= max(8, n_rows // 100), f"{n_diff} index differences in {n_rows} rows"
    return dict(bt=bt, comp=comp, raw_o=raw_o, pooled_o=pooled_o, idx_o=idx_o, idx_g=idx_g, n_diff=n_diff,
                dev=(q, k, v))


def run_and_check_decode(dtype, q_np, kc_np, vc_np, offsets, lens, n_kv, max_len=None):
    q = to_device(q_np, dtype)
    kc = to_device(kc_np, dtype)
    vc = to_device(vc_np, dtype)
    off = torch.tensor(np.asarray(offsets, dtype=np.int64), device="cuda")
    ln = torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda")
    batch, n_h, d = q_np.shape
    dec = Decoder(batch, n_h, n_kv, d, int(max(lens)) if max_len is None else max_len)
    out = dec.run(q, kc, vc, off, ln)
    torch.cuda.synchronize()
    ref = O.gqa_decode(q_np, kc_np, vc_np, offsets, lens, n_kv, dtype)
    got = out.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref).max()
    log_parity(dict(what="decode", dtype=dtype, batch=int(batch), n_h=int(n_h), d_h=int(d),
                    rows=int(np.sum(lens)), max_abs_err=float(err), atol=DECODE_ATOL[dtype]))
    assert err <= DECODE_ATOL[dtype], f"decode max abs error {err:.3e} > {DECODE_ATOL[dtype]}"
    # the completion counters are left at zero for the next call
    tick = dec.ws[256:256 + 4 * batch * n_kv].view(torch.int32)
    assert int(tick.abs().sum().item()) == 0
    return got, ref, err
