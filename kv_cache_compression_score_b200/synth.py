"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module draws numbers and lays them out; it holds none of the scoring,
selection, gather or attention arithmetic.  Every tensor is a pure function of
(seed, tensor id, sequence index, element index):

* uniform bits come from a counter-based splitmix64 stream (Steele, Lea and
  Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014): the
  stream key is splitmix64 of (seed, tensor id, sequence) and element n of the
  stream is splitmix64(key + (n + 1) * golden_gamma);
* normals come from the Box-Muller transform in float64 on pairs of uniforms;
* values are rounded to float32 (round to nearest even) and, for bf16, from
  float32 to bf16 (round to nearest even on the bit pattern).  bf16 tensors are
  returned as uint16 bit patterns so no library reinterprets them.

Shapes follow the NHD layout the kernels use: keys and values of a packed batch
are [T, n_kv, d_h], window queries are [n_seqs * w, n_h, d_h], decode queries
are [batch, n_h, d_h].  Salient-key boosting follows the reading "1% of key
positions per head are moved by +3 sigma along one random unit direction per
head".
"""
from __future__ import annotations

import numpy as np

MASK64 = np.uint64(0xFFFFFFFFFFFFFFFF)
GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)

# Tensor ids: one independent stream per (seed, id, sequence).
T_QWIN, T_K, T_V, T_QDEC, T_HIDDEN, T_BOOST_DIR, T_BOOST_POS, T_LENGTHS, T_SCORES, T_DRIFT, T_XKV = range(1, 12)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int, seq: int = 0) -> np.uint64:
    """64-bit key of one stream; distinct (seed, tensor, seq) give unrelated streams."""
    raw = ((int(seed) & 0xFFFFFFFF) << 32) ^ ((int(tensor_id) & 0xFFFF) << 16) ^ (int(seq) & 0xFFFF)
    with np.errstate(over="ignore"):
        return _mix64(np.array([raw], dtype=np.uint64) * GOLDEN_GAMMA + GOLDEN_GAMMA)[0]


def uniform_u64(key: np.uint64, n: int, start: int = 0) -> np.ndarray:
    """Elements start..start+n-1 of the splitmix64 stream `key` (uint64)."""
    ctr = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + ctr * GOLDEN_GAMMA)


def uniform01(key: np.uint64, n: int, start: int = 0) -> np.ndarray:
    """Uniforms in the open interval (0, 1) from the top 53 bits, float64."""
    u = uniform_u64(key, n, start) >> np.uint64(11)
    return (u.astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal_f64(key: np.uint64, n: int) -> np.ndarray:
    """n standard normals by Box-Muller; element 2k, 2k+1 use uniforms 2k, 2k+1."""
    m = (n + 1) // 2
    u = uniform01(key, 2 * m)
    u1, u2 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * m, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:n]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (for building test inputs)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x64: np.ndarray, dtype: str) -> np.ndarray:
    """float64 -> stored representation: float32 array, or uint16 bf16 bits."""
    f = x64.astype(np.float32)
    if dtype == "f32":
        return f
    if dtype == "bf16":
        return f32_to_bf16_bits(f)
    raise ValueError(f"unknown dtype {dtype!r}")


def normal_tensor(seed: int, tensor_id: int, seq: int, shape, dtype: str) -> np.ndarray:
    n = int(np.prod(shape))
    return round_to(normal_f64(stream_key(seed, tensor_id, seq), n).reshape(shape), dtype)


def ragged_lengths(seed: int, n_seqs: int, lo: int, hi: int) -> np.ndarray:
    """n_seqs integers uniform on [lo, hi] inclusive (int32)."""
    span = np.uint64(hi - lo + 1)
    u = uniform_u64(stream_key(seed, T_LENGTHS, 0), n_seqs)
    return (np.int64(lo) + (u % span).astype(np.int64)).astype(np.int32)


def boosted_positions(seed: int, seq: int, head: int, length: int, frac: float) -> np.ndarray:
    """floor(frac*length) distinct positions in [0, length), sorted (sampled without replacement)."""
    m = int(np.floor(frac * length))
    if m == 0:
        return np.zeros(0, dtype=np.int64)
    keys = uniform_u64(stream_key(seed, T_BOOST_POS, seq * 256 + head), length)
    return np.sort(np.argsort(keys, kind="stable")[:m])


def boost_direction(seed: int, seq: int, head: int, d_h: int) -> np.ndarray:
    v = normal_f64(stream_key(seed, T_BOOST_DIR, seq * 256 + head), d_h)
    return v / np.linalg.norm(v)


def keys_values(seed: int, seq: int, length: int, n_kv: int, d_h: int, dtype: str,
                boost_frac: float = 0.0, boost: float = 3.0):
    """K and V of one sequence, [length, n_kv, d_h], N(0,1), optionally boosted keys."""
    k = normal_f64(stream_key(seed, T_K, seq), length * n_kv * d_h).reshape(length, n_kv, d_h)
    if boost_frac > 0.0:
        for h in range(n_kv):
            pos = boosted_positions(seed, seq, h, length, boost_frac)
            k[pos, h, :] += boost * boost_direction(seed, seq, h, d_h)[None, :]
    v = normal_f64(stream_key(seed, T_V, seq), length * n_kv * d_h).reshape(length, n_kv, d_h)
    return round_to(k, dtype), round_to(v, dtype)


def window_queries(seed: int, seq: int, w: int, n_h: int, d_h: int, dtype: str) -> np.ndarray:
    return normal_tensor(seed, T_QWIN, seq, (w, n_h, d_h), dtype)


def decode_queries(seed: int, batch: int, n_h: int, d_h: int, dtype: str) -> np.ndarray:
    return normal_tensor(seed, T_QDEC, 0, (batch, n_h, d_h), dtype)


def hidden_states(seed: int, length: int, D: int, dtype: str) -> np.ndarray:
    return normal_tensor(seed, T_HIDDEN, 0, (length, D), dtype)


def random_scores(seed: int, shape, n_levels: int = 0) -> np.ndarray:
    """Non-negative float32 scores for selection tests.  With n_levels > 0 the
    values are drawn from n_levels distinct levels so that ties are frequent."""
    n = int(np.prod(shape))
    key = stream_key(seed, T_SCORES, 0)
    if n_levels > 0:
        lv = (uniform_u64(key, n) % np.uint64(n_levels)).astype(np.float64)
        return (lv / n_levels).astype(np.float32).reshape(shape)
    return uniform01(key, n).astype(np.float32).reshape(shape)


def packed_batch(seed: int, lengths, n_h: int, n_kv: int, d_h: int, w: int, dtype: str,
                 boost_frac: float = 0.0, boost: float = 3.0):
    """A packed ragged batch: dict with q_win, k, v, cu_seqlens (int32), seqlens."""
    lengths = np.asarray(lengths, dtype=np.int32)
    ks, vs, qs = [], [], []
    for b, L in enumerate(lengths):
        k, v = keys_values(seed, b, int(L), n_kv, d_h, dtype, boost_frac, boost)
        ks.append(k)
        vs.append(v)
        qs.append(window_queries(seed, b, w, n_h, d_h, dtype))
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths, dtype=np.int64).astype(np.int32)
    return {
        "q_win": np.concatenate(qs, axis=0),
        "k": np.concatenate(ks, axis=0),
        "v": np.concatenate(vs, axis=0),
        "cu_seqlens": cu,
        "seqlens": lengths,
    }


def index_lists(seed: int, lengths, n_kv: int, budget: int) -> np.ndarray:
    """Seeded stand-in index lists for gather tests: per (sequence, head) a
    sorted sample without replacement of min(budget, len) positions of
    [0, len), concatenated per head -> int32 [n_kv, sum_b min(budget, len_b)]."""
    rows = [[] for _ in range(n_kv)]
    for b, L in enumerate(lengths):
        kept = min(int(budget), int(L))
        for h in range(n_kv):
            keys = uniform_u64(stream_key(seed, T_SCORES, b * 256 + h + 1), int(L))
            rows[h].append(np.sort(np.argsort(keys, kind="stable")[:kept]))
    return np.stack([np.concatenate(r) if r else np.zeros(0, np.int64) for r in rows]).astype(np.int32)


def drifted_queries(seed: int, q_prev_bits: np.ndarray, dtype: str, lo: float = 0.0, hi: float = 0.9,
                    group: int = 1) -> np.ndarray:
    """Next-step decode queries: q_prev + sigma * noise with one sigma per
    (batch entry, group of `group` consecutive query heads) drawn uniformly
    from [lo, hi] -- from nearly equal queries to strongly drifted ones, so
    that some groups fall below a similarity threshold and others do not."""
    prev = bf16_bits_to_f32(q_prev_bits).astype(np.float64) if dtype == "bf16" else \
        np.asarray(q_prev_bits, dtype=np.float64)
    batch, n_h, d = prev.shape
    sig = lo + (hi - lo) * uniform01(stream_key(seed, T_DRIFT, 0), batch * (n_h // group))
    sig = np.repeat(sig.reshape(batch, n_h // group), group, axis=1).reshape(batch, n_h, 1)
    noise = normal_f64(stream_key(seed, T_DRIFT, 1), batch * n_h * d).reshape(batch, n_h, d)
    return round_to(prev + sig * noise, dtype)


def cross_layer_keys(seed: int, S: int, n_kv: int, d_h: int, W: int, rank: int, noise: float = 0.05,
                     dtype: str = "bf16") -> list:
    """Keys of W layers, [S, n_kv, d_h] each, whose per-head concatenation
    [K_1[:, h] | ... | K_W[:, h]] is a rank-`rank` matrix plus noise: a token
    factor Z_h ([S, rank], N(0,1), column c scaled by 2^(-2c/rank)) shared by
    the W layers, times per-layer loadings ([rank, d_h], N(0,1) / sqrt(rank)),
    plus noise * N(0,1) per element.  The shared token factor stands for the
    aligned dominant singular vectors across layers that the xKV page reports;
    the scaled columns give a decaying spectrum with a gap after `rank`."""
    F = W * d_h
    out = np.zeros((W, S, n_kv, d_h))
    col = 2.0 ** (-2.0 * np.arange(rank) / rank)
    for h in range(n_kv):
        Z = normal_f64(stream_key(seed, T_XKV, 3 * h), S * rank).reshape(S, rank) * col
        B = normal_f64(stream_key(seed, T_XKV, 3 * h + 1), rank * F).reshape(rank, F) / np.sqrt(rank)
        E = normal_f64(stream_key(seed, T_XKV, 3 * h + 2), S * F).reshape(S, F) * noise
        X = Z @ B + E
        for l in range(W):
            out[l, :, h, :] = X[:, l * d_h:(l + 1) * d_h]
    return [round_to(out[l], dtype) for l in range(W)]


def start_basis(seed: int, n_kv: int, F: int, r: int) -> np.ndarray:
    """Gaussian start basis [n_kv, F, r] (float32) for subspace iteration."""
    key = stream_key(seed, T_XKV, 0xFFFF)
    return normal_f64(key, n_kv * F * r).reshape(n_kv, F, r).astype(np.float32)
