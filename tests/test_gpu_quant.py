"""Quantised compact cache on the GPU (int8 codes, one float32 scale per
(row, head)): gather-and-quantise is bit-exact against the oracle's
quantiser on the GPU's own indices, and decode over the int8 caches matches
the oracle's decode over the dequantised values."""
import numpy as np
import pytest
import torch

from kv_cache_compression_score_b200 import kvc, synth
from kv_cache_compression_score_b200.runner import Decoder, from_device, to_device
from oracle import kvc_oracle as O
from parity_helpers import DECODE_ATOL, log_parity, run_and_check_compress

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from kv_cache_compression_score_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _gather_q8(comp, k, v, budget, pitch_extra=0):
    b = comp.buf
    Tb, n_kv, d = b.k_c.shape
    kq = torch.empty((Tb, n_kv, d), dtype=torch.int8, device="cuda")
    vq = torch.empty_like(kq)
    pitch = (Tb + pitch_extra + 3) // 4 * 4
    ks = torch.full((n_kv, pitch), float("nan"), dtype=torch.float32, device="cuda")
    vs = torch.full_like(ks, float("nan"))
    kvc.kvc_gather_kv_q8(b.seqlens, b.cu_seqlens, b.cu_budget, budget, b.idx, k, v, kq, vq, ks, vs)
    return kq, vq, ks, vs


def _decode_q8(q_np, kq, vq, ks, vs, offs, lens, n_kv):
    batch, n_h, d = q_np.shape
    dec = Decoder(batch, n_h, n_kv, d, int(max(lens)))
    off = torch.tensor(np.asarray(offs, dtype=np.int64), device="cuda")
    ln = torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda")
    kvc.kvc_gqa_decode_attn_q8(to_device(q_np, "bf16"), kq, vq, ks, vs, off, ln, int(max(lens)), 0.0, dec.out, dec.ws)
    torch.cuda.synchronize()
    tick = dec.ws[256:256 + 4 * batch * n_kv].view(torch.int32)
    assert int(tick.abs().sum().item()) == 0
    return dec.out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("lengths,budget,d", [([3000, 700, 77], 512, 128), ([2500], 1000, 64)])
def test_gather_q8_bit_exact_and_decode(lengths, budget, d):
    n_h, n_kv, w = 32, 8, 32
    r = run_and_check_compress("bf16", lengths, n_h, n_kv, d, w, 7, budget, seed=3100 + d, boost_frac=0.01,
                               fused_call=True)
    q_dev, k_dev, v_dev = r["dev"]
    kq, vq, ks, vs = _gather_q8(r["comp"], k_dev, v_dev, budget, pitch_extra=5)
    torch.cuda.synchronize()
    cu = r["bt"]["cu_seqlens"]
    kq_o, vq_o, ks_o, vs_o = O.gather_kv_q8(r["bt"]["k"], r["bt"]["v"], r["idx_g"].astype(np.int64), cu, budget,
                                            "bf16")
    Tb = kq_o.shape[0]
    assert np.array_equal(kq.cpu().numpy(), kq_o) and np.array_equal(vq.cpu().numpy(), vq_o)
    assert np.array_equal(ks.cpu().numpy()[:, :Tb], ks_o) and np.array_equal(vs.cpu().numpy()[:, :Tb], vs_o)
    # decode over the int8 caches, one query per sequence
    cb = O.budget_offsets(lengths, budget)
    q = synth.decode_queries(3200 + d, len(lengths), n_h, d, "bf16")
    got = _decode_q8(q, kq, vq, ks, vs, cb[:-1], np.diff(cb), n_kv)
    ref = O.gqa_decode_q8(q, kq_o, vq_o, ks_o, vs_o, cb[:-1], np.diff(cb), n_kv, "bf16")
    err = float(np.abs(got - ref).max())
    log_parity(dict(what="decode_q8", d_h=d, rows=int(cb[-1]), max_abs_err=err))
    assert err <= DECODE_ATOL["bf16"], err


@pytest.mark.parametrize("n_h,n_kv,d", [(32, 8, 128), (8, 8, 64), (16, 2, 128)])
def test_decode_q8_ragged_empty_aliased(n_h, n_kv, d):
    """Seeded int8 caches: ragged lengths, an empty cache, a length-1 cache and
    two queries on the same cache; a zero row (scale 0) among them."""
    lens = [2048, 0, 1, 777, 2048, 130]
    offs = [0, 2048, 2048, 2049, 0, 2826]
    rows = 2826 + 130
    kf, vf = synth.keys_values(3300, 0, rows, n_kv, d, "f32")
    kf[5] = 0.0
    kq, ks = O.quantize_rows_int8(kf)
    vq, vs = O.quantize_rows_int8(vf)
    ks_t, vs_t = np.ascontiguousarray(ks.T), np.ascontiguousarray(vs.T)
    q = synth.decode_queries(3301, len(lens), n_h, d, "bf16")
    got = _decode_q8(q, torch.from_numpy(kq).cuda(), torch.from_numpy(vq).cuda(), torch.from_numpy(ks_t).cuda(),
                     torch.from_numpy(vs_t).cuda(), offs, lens, n_kv)
    ref = O.gqa_decode_q8(q, kq, vq, ks_t, vs_t, offs, lens, n_kv, "bf16")
    assert np.all(got[1] == 0)
    err = float(np.abs(got - ref).max())
    log_parity(dict(what="decode_q8", d_h=d, n_h=n_h, rows=int(sum(lens)), max_abs_err=err))
    assert err <= DECODE_ATOL["bf16"], err


def test_decode_q8_llama8b_batch16():
    """The Llama-3-8B-shaped decode (batch 16 x 2048 rows, n_h 32, n_kv 8,
    d_h 128) over int8 caches quantised by the GPU from seeded bf16 caches."""
    n_h, n_kv, d, B, nb = 32, 8, 128, 2048, 16
    k, v = synth.keys_values(3400, 0, nb * B, n_kv, d, "bf16")
    idx = np.broadcast_to(np.arange(nb * B, dtype=np.int32), (n_kv, nb * B)).copy()
    cu = torch.tensor([0, nb * B], dtype=torch.int32, device="cuda")
    kq = torch.empty((nb * B, n_kv, d), dtype=torch.int8, device="cuda")
    vq = torch.empty_like(kq)
    ks = torch.empty((n_kv, nb * B), dtype=torch.float32, device="cuda")
    vs = torch.empty_like(ks)
    kvc.kvc_gather_kv_q8([nb * B], cu, cu, nb * B, torch.from_numpy(idx).cuda(), to_device(k, "bf16"),
                         to_device(v, "bf16"), kq, vq, ks, vs)
    torch.cuda.synchronize()
    kq_o, vq_o, ks_o, vs_o = O.gather_kv_q8(k, v, idx.astype(np.int64), [0, nb * B], nb * B, "bf16")
    assert np.array_equal(kq.cpu().numpy(), kq_o) and np.array_equal(ks.cpu().numpy(), ks_o)
    q = synth.decode_queries(3401, nb, n_h, d, "bf16")
    offs, lens = np.arange(nb) * B, [B] * nb
    got = _decode_q8(q, kq, vq, ks, vs, offs, lens, n_kv)
    ref = O.gqa_decode_q8(q, kq_o, vq_o, ks_o, vs_o, offs, lens, n_kv, "bf16")
    err = float(np.abs(got - ref).max())
    log_parity(dict(what="decode_q8", d_h=d, batch=nb, rows=nb * B, max_abs_err=err))
    assert err <= DECODE_ATOL["bf16"], err


def test_gather_q8_exact_ties_and_tiny_scales():
    """Quotients that land exactly on half-integers (round half to even),
    scales below the smallest normal float, all-zero vectors and seeded rows:
    codes and scales bit-identical to the oracle's float32 quantiser."""
    n_kv, d = 2, 128
    rows = []
    halves = np.arange(d, dtype=np.float64) - 63.5                     # -63.5 .. 63.5: x / 1 = k + 0.5
    r0 = halves.copy(); r0[0] = 127.0                                   # amax 127: scale exactly 1
    r1 = halves / 2.0; r1[5] = -63.5                                    # amax 63.5: scale exactly 0.5
    r2 = np.zeros(d); r2[0] = 2.0 ** -127; r2[1:9] = 2.0 ** -128; r2[9] = -(2.0 ** -128)   # subnormal scale, ties
    r3 = np.zeros(d)                                                    # all zero: scale 0, codes 0
    kr, vr = synth.keys_values(3500, 0, 4, n_kv, d, "f32")
    for extra in (r0, r1, r2, r3):
        rows.append(extra)
    base = np.stack(rows)                                               # [4, d]
    k64 = np.concatenate([np.repeat(base[:, None, :], n_kv, axis=1), kr.astype(np.float64)], axis=0)
    v64 = np.concatenate([np.repeat(base[::-1, None, :], n_kv, axis=1), vr.astype(np.float64)], axis=0)
    k_bits, v_bits = synth.round_to(k64, "bf16"), synth.round_to(v64, "bf16")
    assert np.array_equal(synth.bf16_bits_to_f32(k_bits[:4]).astype(np.float64), k64[:4])   # exactly representable
    N = k64.shape[0]
    idx = np.broadcast_to(np.arange(N, dtype=np.int32), (n_kv, N)).copy()
    cu = torch.tensor([0, N], dtype=torch.int32, device="cuda")
    kq = torch.empty((N, n_kv, d), dtype=torch.int8, device="cuda")
    vq = torch.empty_like(kq)
    ks = torch.empty((n_kv, N), dtype=torch.float32, device="cuda")
    vs = torch.empty_like(ks)
    kvc.kvc_gather_kv_q8([N], cu, cu, N, torch.from_numpy(idx).cuda(), to_device(k_bits, "bf16"),
                         to_device(v_bits, "bf16"), kq, vq, ks, vs)
    torch.cuda.synchronize()
    kq_o, vq_o, ks_o, vs_o = O.gather_kv_q8(k_bits, v_bits, idx.astype(np.int64), [0, N], N, "bf16")
    assert np.array_equal(kq.cpu().numpy(), kq_o) and np.array_equal(vq.cpu().numpy(), vq_o)
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), ks_o.view(np.uint32))
    assert np.array_equal(vs.cpu().numpy().view(np.uint32), vs_o.view(np.uint32))
    # the tie rows really are ties: codes alternate by round-half-to-even
    assert list(kq_o[0, 0, 1:4]) == [-62, -62, -60] and list(kq_o[0, 0, 63:67]) == [0, 0, 2, 2]
    assert ks_o[0, 2] > 0 and ks_o[0, 2] < np.finfo(np.float32).tiny
    assert kq_o[2, 0, 1] == 64 and kq_o[2, 0, 9] == -64
