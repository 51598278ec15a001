"""Buffer plans around the C ABI: allocate the device outputs and workspaces
for one batch shape with torch, then run the entry points in order.

No arithmetic of the method happens here; every step runs in libkvc.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import kvc

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def to_device(a: np.ndarray, dtype: str, device="cuda", pin: bool = False) -> torch.Tensor:
    """Stored host array (fp32 values or uint16 bf16 bits) -> device tensor of the matching dtype."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if pin:
        t = t.pin_memory()
    return t.to(device, non_blocking=pin)


def from_device(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host array in the stored representation (bf16 as uint16 bits)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def zeroed_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


@dataclass
class CompressBuffers:
    seqlens: np.ndarray
    cu_seqlens: torch.Tensor
    cu_budget_host: np.ndarray
    cu_budget: torch.Tensor
    scores: torch.Tensor
    scores_raw: torch.Tensor
    idx: torch.Tensor
    k_c: torch.Tensor
    v_c: torch.Tensor
    ws: torch.Tensor


class Compressor:
    """Score, select and gather for one packed batch shape (kvc_score_window,
    kvc_select_topk, kvc_gather_kv)."""

    def __init__(self, dtype: str, seqlens, n_h: int, n_kv: int, d_h: int, w: int, pool_k: int, budget: int,
                 scale: float = 0.0, device="cuda", keep_raw: bool = True):
        self.dtype, self.n_h, self.n_kv, self.d_h, self.w = dtype, n_h, n_kv, d_h, w
        self.pool_k, self.budget, self.scale = pool_k, budget, scale
        sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
        T = int(sl.sum())
        cu = np.zeros(len(sl) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(sl)
        cb = kvc.kvc_budget_offsets(sl, budget)
        code = kvc.KVC_F32 if dtype == "f32" else kvc.KVC_BF16
        ws_bytes = kvc.kvc_score_window_workspace_size(code, sl, n_h, n_kv, d_h, w)
        if ws_bytes == 0:
            raise kvc.KvcError(1, kvc.lib().kvc_last_error().decode())
        td = TORCH_DTYPE[dtype]
        Tb = int(cb[-1])
        self.buf = CompressBuffers(
            seqlens=sl,
            cu_seqlens=torch.from_numpy(cu).to(device),
            cu_budget_host=cb,
            cu_budget=torch.from_numpy(cb).to(device),
            scores=torch.empty((n_kv, T), dtype=torch.float32, device=device),
            scores_raw=torch.empty((n_kv, T), dtype=torch.float32, device=device) if keep_raw else None,
            idx=torch.empty((n_kv, Tb), dtype=torch.int32, device=device),
            k_c=torch.empty((Tb, n_kv, d_h), dtype=td, device=device),
            v_c=torch.empty((Tb, n_kv, d_h), dtype=td, device=device),
            ws=zeroed_workspace(ws_bytes, device),
        )

    def score(self, q_win, k, stream=None):
        b = self.buf
        kvc.kvc_score_window(q_win, k, b.seqlens, b.cu_seqlens, self.n_h, self.n_kv, self.w, self.pool_k, self.scale,
                             b.scores, b.scores_raw, b.ws, stream)

    def select(self, stream=None):
        b = self.buf
        kvc.kvc_select_topk(b.seqlens, b.cu_seqlens, b.cu_budget, self.n_kv, self.w, self.budget, b.scores, b.idx,
                            stream)

    def gather(self, k, v, stream=None):
        b = self.buf
        kvc.kvc_gather_kv(b.seqlens, b.cu_seqlens, b.cu_budget, self.budget, b.idx, k, v, b.k_c, b.v_c, stream)

    def compress(self, q_win, k, v, stream=None):
        """kvc_compress_window: the same three steps in one call."""
        b = self.buf
        kvc.kvc_compress_window(q_win, k, v, b.seqlens, b.cu_seqlens, b.cu_budget, self.n_h, self.n_kv, self.w,
                                self.pool_k, self.budget, self.scale, b.scores, b.scores_raw, b.idx, b.k_c, b.v_c,
                                b.ws, stream)
        return b.idx, b.k_c, b.v_c

    def run(self, q_win, k, v, stream=None):
        self.score(q_win, k, stream)
        self.select(stream)
        self.gather(k, v, stream)
        return self.buf.idx, self.buf.k_c, self.buf.v_c

    def device_error_word(self) -> int:
        return int(self.buf.ws[:4].view(torch.int32).item())


class Decoder:
    """GQA decode attention over compact caches (kvc_gqa_decode_attn)."""

    def __init__(self, batch: int, n_h: int, n_kv: int, d_h: int, max_kv_len: int, scale: float = 0.0,
                 device="cuda"):
        self.max_kv_len, self.scale = max_kv_len, scale
        self.out = torch.empty((batch, n_h, d_h), dtype=torch.float32, device=device)
        self.ws = zeroed_workspace(kvc.kvc_gqa_decode_workspace_size(batch, n_h, n_kv, d_h, max_kv_len), device)

    def run(self, q, k_c, v_c, kv_row_offset, kv_len, stream=None):
        kvc.kvc_gqa_decode_attn(q, k_c, v_c, kv_row_offset, kv_len, self.max_kv_len, self.scale, self.out, self.ws,
                                stream)
        return self.out


class TspSelector:
    """FastKV token-selective propagation for one sequence (kvc_tsp_select_gather)."""

    def __init__(self, S: int, w: int, pool_k: int, k_tsp: int, D: int, dtype: str, device="cuda"):
        self.S, self.w, self.pool_k, self.k_tsp = S, w, pool_k, k_tsp
        self.idx = torch.empty(k_tsp + w, dtype=torch.int32, device=device)
        self.hidden_out = torch.empty((k_tsp + w, D), dtype=TORCH_DTYPE[dtype], device=device)
        self.ws = zeroed_workspace(kvc.kvc_tsp_workspace_size(S, w), device)

    def run(self, scores_raw, hidden, stream=None):
        kvc.kvc_tsp_select_gather(scores_raw, self.w, self.pool_k, self.k_tsp, hidden, self.idx, self.hidden_out,
                                  self.ws, stream)
        return self.idx, self.hidden_out


class FreeKvStep:
    """FreeKV decode steps over full caches of one packed batch (kvc_freekv_step):
    holds the index lists, compact caches, flags and output between steps."""

    def __init__(self, seqlens, n_h: int, n_kv: int, d_h: int, w: int, pool_k: int, budget: int, tau: float,
                 scale: float = 0.0, device="cuda"):
        self.n_h, self.w, self.pool_k, self.budget, self.tau, self.scale = n_h, w, pool_k, budget, tau, scale
        sl = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
        cu = np.zeros(len(sl) + 1, dtype=np.int32)
        cu[1:] = np.cumsum(sl)
        cb = kvc.kvc_budget_offsets(sl, budget)
        Tb = int(cb[-1])
        self.seqlens = sl
        self.cu_seqlens = torch.from_numpy(cu).to(device)
        self.cu_budget_host = cb
        self.cu_budget = torch.from_numpy(cb).to(device)
        self.idx = torch.zeros((n_kv, Tb), dtype=torch.int32, device=device)
        self.k_c = torch.zeros((Tb, n_kv, d_h), dtype=torch.bfloat16, device=device)
        self.v_c = torch.zeros_like(self.k_c)
        self.reselected = torch.zeros((len(sl), n_kv), dtype=torch.int32, device=device)
        self.out = torch.empty((len(sl), n_h, d_h), dtype=torch.float32, device=device)
        self.ws = zeroed_workspace(kvc.kvc_freekv_workspace_size(sl, n_h, n_kv, d_h, w, budget), device)

    def step(self, q_cur, q_prev, k, v, tau=None, stream=None):
        kvc.kvc_freekv_step(self.seqlens, self.cu_seqlens, self.cu_budget, self.n_h, self.w, self.pool_k, self.budget,
                            self.tau if tau is None else tau, self.scale, q_cur, q_prev, k, v, self.idx, self.k_c,
                            self.v_c, self.reselected, self.out, self.ws, stream)
        return self.out
