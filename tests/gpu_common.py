"""Shared helpers of the GPU parity tests: workload tensors, oracle glue, set comparison.

Inputs come from ``lsa_synth`` only; expected values come from ``oracle`` only.  The oracle is
always run on exactly the bytes the GPU received (bf16 / e4m3 codes decoded exactly to fp64).
"""

from __future__ import annotations

import math

import numpy as np
import torch

import lsa_synth as S
from oracle import lsa_oracle as O

TIE_REL = 1e-5      # selection parity: positions within 1e-5 relative of the K-th score are ties
ATTN_REL = 1e-2     # attention parity: per (b, h) row, max |err| / max |ref| <= 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a bf16 / fp32 / e4m3-code tensor (codes are returned as-is)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return O.bf16_to_f64(t.view(torch.int16).numpy())
    if t.dtype == torch.float32:
        return t.numpy().astype(np.float64)
    raise TypeError(t.dtype)


def dequant_rows(codes: torch.Tensor, scale: torch.Tensor) -> np.ndarray:
    """Oracle-side e4m3 decode: code value (format definition) times the row scale, in fp64."""
    v = O.e4m3_to_f64(codes.detach().cpu().view(torch.uint8).numpy())
    return v * scale.detach().cpu().numpy().astype(np.float64)[..., None]


def check_index_sets(idx_row: np.ndarray, cnt: int, oracle_set: np.ndarray, scores_row: np.ndarray,
                     kth: float, kmax: int, fixed: set | None = None) -> int:
    """Bit-exact set check except ties; returns the number of tie positions that differ.

    idx_row: GPU row (int32, length >= kmax).  The first cnt entries must be strictly ascending,
    the rest -1 up to kmax.  A position in the symmetric difference must be a dynamic one whose
    oracle score is within TIE_REL relative of the oracle's K-th score.
    """
    got = idx_row[:cnt]
    assert cnt == oracle_set.size, f"count {cnt} != oracle {oracle_set.size}"
    assert np.all(np.diff(got) > 0), "GPU set not strictly ascending"
    assert np.all(idx_row[cnt:kmax] == -1), "padding must be -1"
    diff = np.setxor1d(got, oracle_set)
    if diff.size == 0:
        return 0
    tol = TIE_REL * abs(kth) if kth != 0 else 1e-30
    for s in diff.tolist():
        assert fixed is None or s not in fixed, f"fixed position {s} differs"
        assert abs(scores_row[s] - kth) <= tol, f"position {s}: score {scores_row[s]!r} vs K-th {kth!r} is not a tie"
    return int(diff.size)


def attn_rel_err(out_gpu: torch.Tensor, ref: np.ndarray) -> float:
    """max over (h) of max|o_gpu - o_ref| / max|o_ref| for one query (out [H, d_v])."""
    og = f64(out_gpu)
    num = np.abs(og - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    return float((num / den).max())


class Decode:
    """Device + host tensors of a token-mode workload, generated from lsa_synth."""

    def __init__(self, wl: S.Workload, device="cuda", fp8: bool = False, B: int | None = None,
                 q_pos: torch.Tensor | None = None):
        self.wl = wl
        self.B = B if B is not None else wl.B
        self.device = device
        q_I, w = S.index_queries(wl, "cpu")
        self.q_I_cpu = q_I[: self.B].contiguous()
        self.w_cpu = w[: self.B].contiguous()
        self.k_I = S.index_keys(wl, q_I, device)  # [L, d_I] bf16 on the device
        self.q_pos = (q_pos if q_pos is not None else wl.q_pos()[: self.B]).to(device)
        self.q_I = self.q_I_cpu.to(device)
        self.w = self.w_cpu.to(device)
        self.fp8 = fp8
        if fp8:
            self.q8, self.q_scale = S.quantize_e4m3_rows(self.q_I)
            self.k8, self.k_scale = S.quantize_e4m3_rows(self.k_I)

    def oracle_scores(self, rows=None) -> np.ndarray:
        """fp64 oracle scores for query rows ``rows`` (default all) on the GPU's exact inputs."""
        rows = list(range(self.B)) if rows is None else list(rows)
        if self.fp8:
            q = dequant_rows(self.q8[rows], self.q_scale[rows])
            k = dequant_rows(self.k8, self.k_scale)
        else:
            q = f64(self.q_I_cpu[rows])
            k = f64(self.k_I)
        return O.index_score(q, f64(self.w_cpu[rows]), k, self.q_pos[rows].cpu().numpy())

    def oracle_scores_bf16(self, rows=None) -> np.ndarray:
        rows = list(range(self.B)) if rows is None else list(rows)
        return O.index_score(f64(self.q_I_cpu[rows]), f64(self.w_cpu[rows]), f64(self.k_I),
                             self.q_pos[rows].cpu().numpy())


def run_oracle_attention(q_b: torch.Tensor, kv: torch.Tensor, sel: np.ndarray, scale: float, d_v: int = 512):
    """Oracle attention of one query on the given selected positions (rows fetched from kv exactly)."""
    if sel.size:
        rows = kv[torch.as_tensor(sel, dtype=torch.int64, device=kv.device)]
    else:
        rows = kv[:0]
    return O.sparse_mla_attn(f64(q_b), f64(rows), scale, d_v)


def cuda_ok() -> bool:
    return torch.cuda.is_available()


def default_scale(d_qk=576):
    return 1.0 / math.sqrt(d_qk)
