"""xKV cross-layer factorisation and selective reconstruction on the GPU
against the oracle's truncated SVD (xKV technical summary, sections 2.2 and
2.3).

A and Vt are unique only up to a rotation of the r basis vectors, so the
tests compare what is unique: the projector Vt^T Vt onto the rank-r subspace
and the reconstructed rows A[idx] Vt[:, layer block].  The windows are
synthetic cross-layer keys with a spectral gap after r (checked on the
oracle's singular values), so that `iters` steps of subspace iteration reach
float32 resolution.

Tolerance of a reconstructed element (derived, per element j of row x):
  |got - ref| <= 2^-8 |ref|            bf16 output rounding (unit roundoff 2^-8)
               + eps_P ||x||_2          subspace: |x (P_gpu - P_ref) e_j| <= ||P_gpu - P_ref||_2 ||x||
               + 2^-16 ||x||_2          tensor-core products with float32 operands split into two
                                        bf16 terms (each term's residual <= 2^-17 of the value;
                                        Cauchy-Schwarz with ||Vt[:, j]|| <= 1, ||A_row|| <= ||x||)
               + 2^-8 ||x||_2           bf16 basis only: |dA . Vt[:, j]| <= ||dA|| <= 2^-8 ||A_row|| <= 2^-8 ||x||
               + 1e-6                   float32 accumulation floor
with eps_P = 1e-4, itself checked on the projector directly.  The basis is
checked against X Vt^T with the bound (2^-16 + F 2^-24) ||x|| (the split of V
and the float32 sum of F products), plus 2^-8 |A| for a bf16 basis.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_score_b200 import kvc, synth
from kv_cache_compression_score_b200.runner import Decoder, from_device, to_device
from oracle import kvc_oracle as O
from parity_helpers import DECODE_ATOL, log_parity

pytestmark = pytest.mark.gpu

EPS_P = 1e-4
U_BF16 = 2.0 ** -8


@pytest.fixture(autouse=True, scope="module")
def _built():
    from kv_cache_compression_score_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _factorize(keys_np, r, iters, basis_dtype, seed):
    W = len(keys_np)
    S, n_kv, d = keys_np[0].shape
    F = W * d
    k_dev = [to_device(k, "bf16") for k in keys_np]
    v0 = torch.from_numpy(synth.start_basis(seed, n_kv, F, r)).cuda()
    basis = torch.empty((n_kv, S, r), dtype=basis_dtype, device="cuda")
    blocks = torch.empty((n_kv, r, F), dtype=torch.float32, device="cuda")
    ws = torch.empty(kvc.kvc_xkv_workspace_size(S, n_kv, d, W, r), dtype=torch.uint8, device="cuda")
    kvc.kvc_xkv_factorize(k_dev, r, iters, v0, basis, blocks, ws)
    torch.cuda.synchronize()
    return k_dev, basis, blocks


def _check_case(S, n_kv, d, W, r, basis_dtype, seed, iters=8, n_sel=None, rank=None):
    keys = synth.cross_layer_keys(seed, S, n_kv, d, W, rank or r)
    X = np.concatenate([O.to_f64(k, "bf16") for k in keys], axis=2)          # [S, n_kv, F]
    # precondition: a spectral gap after r in every head
    for h in range(n_kv):
        sv = np.linalg.svd(X[:, h, :], compute_uv=False)
        if r < len(sv):
            assert sv[r - 1] / sv[r] > 3.0, f"head {h}: no spectral gap ({sv[r - 1]} vs {sv[r]})"
    A_ref, Vt_ref = O.xkv_factorize(keys, r, "bf16")
    k_dev, basis, blocks = _factorize(keys, r, iters, basis_dtype, seed + 1)
    Vt = blocks.cpu().numpy().astype(np.float64)
    A = basis.float().cpu().numpy().astype(np.float64)
    # orthonormal rows, and the projector against the oracle's
    p_err = 0.0
    for h in range(n_kv):
        assert np.abs(Vt[h] @ Vt[h].T - np.eye(r)).max() < 1e-5
        p_err = max(p_err, np.linalg.norm(Vt[h].T @ Vt[h] - Vt_ref[h].T @ Vt_ref[h], 2))
    assert p_err < EPS_P, f"projector distance {p_err:.3e}"
    # the basis is X Vt^T (property at any size)
    xn = np.linalg.norm(X, axis=2)                                            # [S, n_kv]
    a_want = np.einsum("shf,hrf->hsr", X, Vt)
    a_tol = (2.0 ** -16 + X.shape[2] * 2.0 ** -24) * xn.T[..., None] + 1e-6
    if basis_dtype == torch.bfloat16:
        a_tol = a_tol + U_BF16 * np.abs(a_want)
    assert np.all(np.abs(A - a_want) <= a_tol)
    # selective reconstruction of every layer
    n_sel = n_sel or min(S, 700)
    idx = synth.index_lists(seed + 2, [S], n_kv, n_sel)
    idx_dev = torch.from_numpy(idx).cuda()
    worst = 0.0
    for layer in range(W):
        out = torch.empty((n_sel, n_kv, d), dtype=torch.bfloat16, device="cuda")
        kvc.kvc_xkv_reconstruct(W, layer, basis, blocks, idx_dev, out)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy().astype(np.float64)
        ref = O.xkv_reconstruct(A_ref, Vt_ref, layer, d, idx)
        xrow = np.stack([xn[idx[h], h] for h in range(n_kv)], axis=1)[..., None]   # [n_sel, n_kv, 1]
        tol = U_BF16 * np.abs(ref) + (EPS_P + 2.0 ** -16 + (U_BF16 if basis_dtype == torch.bfloat16 else 0.0)) * xrow \
            + 1e-6
        err = np.abs(got - ref)
        worst = max(worst, float((err / tol).max()))
        assert np.all(err <= tol), f"layer {layer}: {int((err > tol).sum())} elements outside the bound"
    log_parity({"test": "xkv", "S": S, "n_kv": n_kv, "d": d, "W": W, "r": r,
                "basis": str(basis_dtype).split(".")[-1], "projector_dist": p_err, "worst_err_over_tol": worst})


@pytest.mark.parametrize("S,n_kv,d,W,r,bdt", [
    (2048, 4, 128, 4, 64, torch.float32),
    (2048, 4, 128, 4, 64, torch.bfloat16),
    (1000, 2, 64, 3, 32, torch.bfloat16),     # ragged against the 32-token steps and 64-token projection tiles
    (333, 3, 128, 1, 16, torch.float32),      # W = 1: a plain per-layer truncated SVD
    (1536, 2, 64, 8, 64, torch.bfloat16),     # F = 512, the largest window
])
def test_xkv_factorize_and_reconstruct(S, n_kv, d, W, r, bdt):
    _check_case(S, n_kv, d, W, r, bdt, seed=4100 + S + W)


def test_xkv_full_size():
    """The measured workload's shape: 32768 tokens, 8 KV heads, d_h 128, W = 4, r = 64."""
    _check_case(32768, 8, 128, 4, 64, torch.bfloat16, seed=4200, n_sel=2048)


def test_xkv_out_of_range_rows_are_zero():
    S, n_kv, d, W, r = 300, 2, 64, 2, 16
    keys = synth.cross_layer_keys(7, S, n_kv, d, W, r)
    _, basis, blocks = _factorize(keys, r, 6, torch.float32, 8)
    idx = torch.tensor([[0, -1, S, 5], [S + 100, 3, 2, -7]], dtype=torch.int32, device="cuda")
    out = torch.full((4, n_kv, d), 7.0, dtype=torch.bfloat16, device="cuda")
    kvc.kvc_xkv_reconstruct(W, 1, basis, blocks, idx, out)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    for h, t in [(0, 1), (0, 2), (1, 0), (1, 3)]:
        assert np.all(o[t, h] == 0.0)
    for h, t in [(0, 0), (0, 3), (1, 1), (1, 2)]:
        assert np.any(o[t, h] != 0.0)


def test_xkv_rebuilt_rows_feed_decode():
    """Rows rebuilt by kvc_xkv_reconstruct are a compact cache in the decode
    layout: decode over them matches the oracle's decode over the oracle's
    bf16-rounded rebuilt rows (the same rows up to the bound above)."""
    S, n_kv, d, W, r, n_sel, n_h = 4096, 8, 128, 4, 64, 512, 32
    keys = synth.cross_layer_keys(4300, S, n_kv, d, W, r)
    vals = synth.cross_layer_keys(4301, S, n_kv, d, W, r)
    _, kb, kt = _factorize(keys, r, 8, torch.bfloat16, 4302)
    _, vb, vt = _factorize(vals, r, 8, torch.bfloat16, 4303)
    idx = synth.index_lists(4304, [S], n_kv, n_sel)
    idx_dev = torch.from_numpy(idx).cuda()
    layer = 2
    kc = torch.empty((n_sel, n_kv, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)
    kvc.kvc_xkv_reconstruct(W, layer, kb, kt, idx_dev, kc)
    kvc.kvc_xkv_reconstruct(W, layer, vb, vt, idx_dev, vc)
    q = synth.decode_queries(4305, 1, n_h, d, "bf16")
    dec = Decoder(1, n_h, n_kv, d, n_sel)
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    ln = torch.full((1,), n_sel, dtype=torch.int32, device="cuda")
    dec.run(to_device(q, "bf16"), kc, vc, off, ln)
    torch.cuda.synchronize()
    got = dec.out.cpu().numpy().astype(np.float64)
    # decode over the GPU's rebuilt rows, in the oracle
    ref_gpu_rows = O.gqa_decode(q, from_device(kc), from_device(vc), [0], [n_sel], n_kv, "bf16")
    assert np.abs(got - ref_gpu_rows).max() <= DECODE_ATOL["bf16"]
    # and against decode over the oracle's own rebuilt rows (bf16): to first
    # order, perturbing V by dV and the logits by dz moves each output by at
    # most |dV|_inf + 2 |dz|_inf |V|_inf (the softmax weights move by at most
    # 2 p_t |dz|_inf and sum to 1); a factor 1.5 covers the second order
    A_k, Vt_k = O.xkv_factorize(keys, r, "bf16")
    A_v, Vt_v = O.xkv_factorize(vals, r, "bf16")
    rk = synth.round_to(O.xkv_reconstruct(A_k, Vt_k, layer, d, idx), "bf16")
    rv = synth.round_to(O.xkv_reconstruct(A_v, Vt_v, layer, d, idx), "bf16")
    ref = O.gqa_decode(q, rk, rv, [0], [n_sel], n_kv, "bf16")
    kg, vg = O.to_f64(from_device(kc), "bf16"), O.to_f64(from_device(vc), "bf16")
    ko, vo = O.to_f64(rk, "bf16"), O.to_f64(rv, "bf16")
    qf = O.to_f64(q, "bf16")[0].reshape(n_kv, n_h // n_kv, d)
    dz = np.abs(np.einsum("hgd,thd->thg", qf, kg - ko)).max() / np.sqrt(d)
    tol = 1.5 * (np.abs(vg - vo).max() + 2.0 * dz * np.abs(vo).max()) + DECODE_ATOL["bf16"]
    err = float(np.abs(got - ref).max())
    log_parity({"test": "xkv_decode", "S": S, "n_sel": n_sel, "max_abs_err": err, "tol": float(tol)})
    assert err <= tol, (err, tol)
