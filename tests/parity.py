"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerance: a score may differ from the oracle's fp64 value by at most
    4e-3 * scale * sum_h |q_h| |k| + 1e-6
(fp32 accumulation of bf16 products), and the mask must match exactly: an
entry is -inf on the GPU iff it is -inf in the oracle.  A tighter bound
derived from fp32 rounding is checked as well:
    |d| <= 2^-16 * scale * sum_h sum_c |q_hc| |k_c| + 1e-6
(128 products accumulated in fp32, 2^-24 per rounding, with headroom for the
tensor core's accumulation order), so a lost term or head cannot hide under
the loose bound.
"""
from __future__ import annotations

import numpy as np
import torch

TIGHT = 2.0 ** -16


def _f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to(torch.float64).cpu().numpy()


def decode_bounds(q: torch.Tensor, k_cache: torch.Tensor, page_table: torch.Tensor, W: int, scale: float):
    """(loose, tight) tolerance arrays [B, Q, W] for decode scores; keys are
    gathered through the page table (a missing page counts as a zero key)."""
    qd = _f64(q)                                   # [B, Q, 4, 128]
    kc = _f64(k_cache)[:, :, 0, :]
    P, ps = kc.shape[0], kc.shape[1]
    table = page_table.cpu().numpy()
    B, Q = qd.shape[0], qd.shape[1]
    n = np.arange(W)
    logical = n // ps
    qn = np.linalg.norm(qd, axis=-1).sum(-1)       # [B, Q]
    qa = np.abs(qd).sum(2)                         # [B, Q, 128]
    loose = np.empty((B, Q, W))
    tight = np.empty((B, Q, W))
    for b in range(B):
        pages = np.full(W, -1)
        inb = logical < table.shape[1]
        pages[inb] = table[b, logical[inb]]
        ok = (pages >= 0) & (pages < P)
        keys = np.zeros((W, 128))
        keys[ok] = kc[pages[ok], n[ok] % ps]
        loose[b] = 4e-3 * scale * qn[b][:, None] * np.linalg.norm(keys, axis=-1)[None, :] + 1e-6
        tight[b] = TIGHT * scale * (qa[b] @ np.abs(keys).T) + 1e-6
    return loose, tight


def prefill_bounds(q: torch.Tensor, k: torch.Tensor, ks: np.ndarray, W: int, scale: float, rows=None):
    """(loose, tight) tolerance arrays [rows, W] for prefill scores (column j is key ks + j)."""
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    qd = _f64(q[torch.as_tensor(rows)])            # [R, 4, 128]
    ks_r = np.asarray(ks)[rows].astype(np.int64)
    if len(rows) and np.all(ks_r == ks_r[0]):
        # rows that share ks see the same key window: only its W keys matter
        k0, Nk = int(ks_r[0]), k.shape[0]
        lo, hi = max(k0, 0), min(k0 + W, Nk)
        loose = np.full((len(rows), W), 1e-6)
        tight = np.full((len(rows), W), 1e-6)
        if hi > lo:
            kd = _f64(k[lo:hi])
            qn = np.linalg.norm(qd, axis=-1).sum(-1)
            loose[:, lo - k0:hi - k0] += 4e-3 * scale * qn[:, None] * np.linalg.norm(kd, axis=-1)[None, :]
            tight[:, lo - k0:hi - k0] += TIGHT * scale * (np.abs(qd).sum(1) @ np.abs(kd).T)
        return loose, tight
    kd = _f64(k)
    Nk = kd.shape[0]
    cols = ks[rows][:, None].astype(np.int64) + np.arange(W)[None, :]
    inb = (cols >= 0) & (cols < Nk)
    cc = np.clip(cols, 0, max(Nk - 1, 0))
    kn = np.linalg.norm(kd, axis=-1) if Nk else np.zeros(1)
    qn = np.linalg.norm(qd, axis=-1).sum(-1)       # [R]
    loose = 4e-3 * scale * qn[:, None] * np.where(inb, kn[cc], 0.0) + 1e-6
    dots = np.abs(qd).sum(1) @ np.abs(kd).T if Nk else np.zeros((len(rows), 1))   # [R, Nk]
    tight = TIGHT * scale * np.where(inb, np.take_along_axis(dots, cc, axis=1), 0.0) + 1e-6
    return loose, tight


def compare_scores(gpu: np.ndarray, ref: np.ndarray, loose: np.ndarray, tight: np.ndarray) -> dict:
    """Assert parity of a block of scores; return error statistics."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref_inf, gpu_inf = np.isneginf(ref), np.isneginf(gpu)
    bad_mask = np.argwhere(ref_inf != gpu_inf)
    assert bad_mask.size == 0, f"mask differs at {bad_mask[:5].tolist()} ({len(bad_mask)} entries)"
    live = ~ref_inf
    assert np.all(np.isfinite(gpu[live])), "non-finite score where the oracle has a value"
    d = np.abs(gpu[live] - ref[live])
    worst_loose = float(np.max(d / loose[live])) if d.size else 0.0
    worst_tight = float(np.max(d / tight[live])) if d.size else 0.0
    assert worst_loose <= 1.0, f"score error {worst_loose:.3g}x the stated tolerance"
    assert worst_tight <= 1.0, f"score error {worst_tight:.3g}x the fp32 rounding bound"
    return {"max_abs": float(d.max()) if d.size else 0.0, "frac_of_tol": worst_loose,
            "frac_of_tight": worst_tight, "entries": int(live.sum())}


def topk_sets_agree(gpu_idx: np.ndarray, ora_idx: np.ndarray, ora_scores: np.ndarray, tol: np.ndarray, k: int):
    """Index sets equal except for swaps among entries whose oracle score lies
    within the tolerance of the k-th selected value.  Padding must agree."""
    g = gpu_idx[gpu_idx >= 0]
    o = ora_idx[ora_idx >= 0]
    assert len(g) == len(o), f"selected {len(g)} blocks, oracle {len(o)}"
    assert len(set(g.tolist())) == len(g), "duplicate index"
    assert np.all(np.diff(g) > 0), "indices not ascending"
    assert np.all(gpu_idx[len(g):] == -1), "padding not -1"
    sg, so = set(g.tolist()), set(o.tolist())
    if sg == so:
        return 0
    kth_idx = o[np.argmin(ora_scores[o])]
    kth = ora_scores[kth_idx]
    for j in sg ^ so:
        assert np.isfinite(ora_scores[j]), f"selected masked block {j}"
        # both scores may be off by their own tolerance
        assert abs(ora_scores[j] - kth) <= tol[j] + tol[kth_idx], \
            f"block {j} swapped but not tied with the k-th value"
    return len(sg ^ so) // 2
