"""ctypes front end of the fp64 CPU oracle for the QSA MQA indexer score.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline use it; the product package never imports it.  All arrays are numpy
(bf16 data travels as uint16 bit patterns) and everything runs on the host.
What each function computes, and the passages it follows, is stated in
``qsa_oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_i64, _int, _f64, _vp = C.c_int64, C.c_int, C.c_double, C.c_void_p

SCALE = 1.0 / np.sqrt(128.0)


def _bind(L: C.CDLL) -> C.CDLL:
    L.qsa_oracle_default_threads.restype = _int
    L.qsa_oracle_logical_position.restype = _i64
    L.qsa_oracle_logical_position.argtypes = [_i64, _i64, _i64]
    L.qsa_oracle_visible_blocks.restype = _i64
    L.qsa_oracle_visible_blocks.argtypes = [_i64, _i64]
    L.qsa_oracle_decode_visible.argtypes = [_vp, _i64, _i64, _vp]
    L.qsa_oracle_prefill_intervals.argtypes = [_vp, _vp, _vp, _i64, _vp, _vp]
    L.qsa_oracle_decode.argtypes = [_vp, _i64, _i64, _i64, _vp, _i64, _i64, _i64, _i64,
                                    _vp, _i64, _i64, _vp, _i64, _i64, _f64, _vp, _i64, _int, _int]
    L.qsa_oracle_prefill.argtypes = [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _i64, _f64,
                                     _vp, _i64, _int, _int]
    L.qsa_oracle_prefill_entries.argtypes = [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _f64,
                                             _vp, _vp, _i64, _vp, _int, _int]
    L.qsa_oracle_f16_to_double.argtypes = [C.c_uint16]
    L.qsa_oracle_f16_to_double.restype = C.c_double
    L.qsa_oracle_topk.argtypes = [_vp, _i64, _vp, _i64, _i64, _vp, _i64, _int]
    L.qsa_oracle_e4m3_to_double.argtypes = [C.c_uint8]
    L.qsa_oracle_e4m3_to_double.restype = C.c_double
    L.qsa_oracle_expand_indices.argtypes = [_vp, _i64, _vp, _vp, _i64, _i64, _vp, _i64]
    L.qsa_oracle_sparse_attention.argtypes = [_vp, _i64, _i64, _i64, _vp, _vp, _i64, _i64, _i64, _i64, _i64,
                                              _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                              _vp, _f64, _vp, _vp, _int]
    L.qsa_oracle_decode_fp8.argtypes = [_vp, _i64, _i64, _i64, _vp, _f64, _i64, _i64, _i64, _i64,
                                        _vp, _i64, _i64, _vp, _i64, _i64, _f64, _vp, _i64, _int]
    return L


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _bits16(x) -> tuple[np.ndarray, tuple[int, ...], int]:
    """bf16 / fp16 tensor, or a uint16 array of bf16 bits -> (uint16 bit
    array, element strides, 1 if fp16 else 0)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) in ("torch.bfloat16", "torch.float16"):
        import torch
        f16 = int(x.dtype == torch.float16)
        x = x.detach().cpu()
        bits = x.view(torch.int16).numpy().view(np.uint16)
        return bits, tuple(x.stride()), f16
    a = np.asarray(x)
    if a.dtype != np.uint16:
        raise TypeError("16-bit data must be a torch.bfloat16 / torch.float16 tensor or a uint16 bf16 bit array")
    return a, tuple(s // 2 for s in a.strides), 0


def _bf16_bits(x) -> tuple[np.ndarray, tuple[int, ...]]:
    """bf16 tensor/array -> (uint16 bit array, element strides)."""
    bits, strides, f16 = _bits16(x)
    if f16:
        raise TypeError("expected bf16 data")
    return bits, strides


def _i32(x) -> np.ndarray:
    a = x.cpu().numpy() if hasattr(x, "cpu") else np.asarray(x)
    return np.ascontiguousarray(a, dtype=np.int32)


class Oracle:
    """One loaded build of the oracle library."""

    def __init__(self, path: str | None = None):
        self.L = _bind(C.CDLL(path or _build.build()))

    def default_threads(self) -> int:
        return int(self.L.qsa_oracle_default_threads())

    def visible_blocks(self, pos: int, seq_len: int) -> int:
        return int(self.L.qsa_oracle_visible_blocks(pos, seq_len))

    def logical_position(self, seq_len: int, query_len: int, i: int) -> int:
        return int(self.L.qsa_oracle_logical_position(seq_len, query_len, i))

    def decode_visible(self, seq_lens, Q: int) -> np.ndarray:
        """visible[b, i] of every decode row."""
        sl = _i32(seq_lens)
        out = np.zeros((sl.shape[0], Q), dtype=np.int32)
        self.L.qsa_oracle_decode_visible(_ptr(sl), sl.shape[0], Q, _ptr(out))
        return out

    def prefill_intervals(self, cu_seqlens_q, seq_lens, key_offsets):
        """(ks, ke) int32 [T] of a packed prefill batch."""
        cu, sl, ko = _i32(cu_seqlens_q), _i32(seq_lens), _i32(key_offsets)
        T = int(cu[-1])
        ks = np.zeros(T, dtype=np.int32)
        ke = np.zeros(T, dtype=np.int32)
        self.L.qsa_oracle_prefill_intervals(_ptr(cu), _ptr(sl), _ptr(ko), sl.shape[0],
                                            _ptr(ks), _ptr(ke))
        return ks, ke

    @staticmethod
    def _decode_common(q, k_cache, page_table, seq_lens):
        qb, qs, f16 = _bits16(q)
        kb, kst, kf16 = _bits16(k_cache)
        if f16 != kf16:
            raise TypeError("q and k_cache must have the same dtype (bf16 or fp16)")
        if len(qs) != 4 or qs[3] != 1:
            raise ValueError("q must be [B, Q, 4, 128] with unit feature stride")
        if len(kst) != 4 or kst[3] != 1:
            raise ValueError("k_cache must be [pages, page_size, 1, 128] with unit feature stride")
        return qb, qs, kb, kst, _i32(page_table), _i32(seq_lens), f16

    def decode(self, q, k_cache, page_table, seq_lens, W: int, scale: float = SCALE,
               threads: int = 0) -> np.ndarray:
        """fp64 scores [B, Q, W] of the paged decode / spec-decode path (q and
        k_cache both bf16 or both fp16)."""
        qb, qs, kb, kst, pt, sl, f16 = self._decode_common(q, k_cache, page_table, seq_lens)
        B, Q = qb.shape[0], qb.shape[1]
        out = np.empty((B, Q, W), dtype=np.float64)
        self.L.qsa_oracle_decode(_ptr(qb), qs[0], qs[1], qs[2], _ptr(kb), kb.shape[0],
                                 kb.shape[1], kst[0], kst[1], _ptr(pt), pt.shape[1],
                                 pt.shape[1], _ptr(sl), B, Q, float(scale), _ptr(out), W,
                                 threads, f16)
        return out

    def f16_to_double(self, bits: int) -> float:
        """Value of one fp16 bit pattern."""
        return float(self.L.qsa_oracle_f16_to_double(int(bits) & 0xFFFF))

    def e4m3_to_double(self, code: int) -> float:
        """Value of one fp8 E4M3 code."""
        return float(self.L.qsa_oracle_e4m3_to_double(int(code) & 0xFF))

    def decode_fp8(self, q, k8, k_scale: float, page_table, seq_lens, W: int, scale: float = SCALE,
                   threads: int = 0) -> np.ndarray:
        """fp64 scores [B, Q, W] over an fp8 E4M3 key cache k8 (uint8 codes
        [pages, page_size, 1, 128]) with dequantisation scale k_scale."""
        qb, qs = _bf16_bits(q)
        if len(qs) != 4 or qs[3] != 1:
            raise ValueError("q must be [B, Q, 4, 128] with unit feature stride")
        if hasattr(k8, "cpu"):
            import torch
            k8 = k8.detach().cpu()
            if k8.dtype != torch.uint8:
                k8 = k8.view(torch.uint8)
            kst = tuple(k8.stride())
            kb = k8.numpy()
        else:
            kb = np.asarray(k8, dtype=np.uint8)
            kst = tuple(kb.strides)
        if len(kst) != 4 or kst[3] != 1:
            raise ValueError("k8 must be [pages, page_size, 1, 128] with unit feature stride")
        pt, sl = _i32(page_table), _i32(seq_lens)
        B, Q = qb.shape[0], qb.shape[1]
        out = np.empty((B, Q, W), dtype=np.float64)
        self.L.qsa_oracle_decode_fp8(_ptr(qb), qs[0], qs[1], qs[2], _ptr(kb), float(k_scale), kb.shape[0],
                                     kb.shape[1], kst[0], kst[1], _ptr(pt), pt.shape[1], pt.shape[1],
                                     _ptr(sl), B, Q, float(scale), _ptr(out), W, threads)
        return out

    @staticmethod
    def _prefill_common(q, k, ks, ke):
        qb, qs, f16 = _bits16(q)
        kb, kst, kf16 = _bits16(k)
        if f16 != kf16:
            raise TypeError("q and k must have the same dtype (bf16 or fp16)")
        if len(qs) != 3 or qs[2] != 1:
            raise ValueError("q must be [T, 4, 128] with unit feature stride")
        if len(kst) != 2 or kst[1] != 1:
            raise ValueError("k must be [Nk, 128] with unit feature stride")
        return qb, qs, kb, kst, _i32(ks), _i32(ke), f16

    def prefill(self, q, k, ks, ke, W: int, scale: float = SCALE, threads: int = 0) -> np.ndarray:
        """fp64 scores [T, W] of the packed prefill path (column j holds key ks[t] + j;
        q and k both bf16 or both fp16)."""
        qb, qs, kb, kst, a, b, f16 = self._prefill_common(q, k, ks, ke)
        T = qb.shape[0]
        out = np.empty((T, W), dtype=np.float64)
        self.L.qsa_oracle_prefill(_ptr(qb), qs[0], qs[1], _ptr(kb), kst[0], kb.shape[0],
                                  _ptr(a), _ptr(b), T, float(scale), _ptr(out), W, threads, f16)
        return out

    def prefill_entries(self, q, k, ks, ke, t, j, scale: float = SCALE,
                        threads: int = 0) -> np.ndarray:
        """fp64 scores of the listed prefill entries (row t[e], column j[e])."""
        qb, qs, kb, kst, a, b, f16 = self._prefill_common(q, k, ks, ke)
        tt = np.ascontiguousarray(t, dtype=np.int64)
        jj = np.ascontiguousarray(j, dtype=np.int64)
        out = np.empty(tt.shape[0], dtype=np.float64)
        self.L.qsa_oracle_prefill_entries(_ptr(qb), qs[0], qs[1], _ptr(kb), kst[0],
                                          kb.shape[0], _ptr(a), _ptr(b), float(scale),
                                          _ptr(tt), _ptr(jj), tt.shape[0], _ptr(out), threads, f16)
        return out

    def expand_indices(self, blocks, pos, seq_len_of_row) -> np.ndarray:
        """Token indices [rows, 4k + 3] of selected blocks [rows, k]: four
        tokens per block, then the row's open-group tokens, then -1."""
        blk = _i32(blocks)
        ps, sl = _i32(pos), _i32(seq_len_of_row)
        rows, k = blk.shape
        tok = np.empty((rows, 4 * k + 3), dtype=np.int32)
        self.L.qsa_oracle_expand_indices(_ptr(blk), k, _ptr(ps), _ptr(sl), rows, k, _ptr(tok), 4 * k + 3)
        return tok

    def sparse_attention(self, q, k_cache, v_cache, page_table, row_req, row_pos, seq_lens, tok,
                         scale: float, gate=None, threads: int = 0):
        """Sparse core attention in fp64: q bf16 [T, Hq, 256], paged K/V bf16
        [pages, page_size, Hkv, 256], token lists tok int32 [T, width]
        (request-local, -1 pads) -> (out [T, Hq, 256], lse [T, Hq])."""
        qb, qs = _bf16_bits(q)
        kb, kst = _bf16_bits(k_cache)
        vb, vst = _bf16_bits(v_cache)
        if len(qs) != 3 or qs[2] != 1 or qb.shape[2] != 256:
            raise ValueError("q must be [T, Hq, 256] with unit feature stride")
        if kst != vst or len(kst) != 4 or kst[3] != 1 or kb.shape != vb.shape or kb.shape[3] != 256:
            raise ValueError("K and V must be [pages, page_size, Hkv, 256] with the same strides")
        T, Hq = qb.shape[0], qb.shape[1]
        Hkv = kb.shape[2]
        if Hq % Hkv:
            raise ValueError("Hq must be a multiple of Hkv")
        pt, rq, rp, sl, tk = _i32(page_table), _i32(row_req), _i32(row_pos), _i32(seq_lens), _i32(tok)
        g = None if gate is None else np.ascontiguousarray(np.asarray(gate, dtype=np.float64).reshape(T, Hq))
        out = np.empty((T, Hq, 256), dtype=np.float64)
        lse = np.empty((T, Hq), dtype=np.float64)
        self.L.qsa_oracle_sparse_attention(_ptr(qb), qs[0], qs[1], Hq, _ptr(kb), _ptr(vb), kb.shape[0], kb.shape[1],
                                           kst[0], kst[1], kst[2], Hkv, _ptr(pt), pt.shape[1], pt.shape[1],
                                           _ptr(rq), _ptr(rp), _ptr(sl), _ptr(tk), tk.shape[1], tk.shape[1], T,
                                           None if g is None else _ptr(g), float(scale), _ptr(out), _ptr(lse),
                                           threads)
        return out, lse

    def topk(self, scores, lengths, k: int, threads: int = 0) -> np.ndarray:
        """Column indices [rows, k] of the k largest scores among each row's first
        lengths[r] columns, ascending, ties to the lower column, -1 padded."""
        s = np.ascontiguousarray(scores, dtype=np.float64)
        ln = _i32(lengths)
        rows = s.shape[0]
        if ln.shape[0] != rows or (rows and ln.max(initial=0) > s.shape[1]):
            raise ValueError("lengths must have one entry per row and not exceed the row width")
        idx = np.empty((rows, k), dtype=np.int32)
        self.L.qsa_oracle_topk(_ptr(s), s.shape[1], _ptr(ln), rows, k, _ptr(idx), k, threads)
        return idx


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from ``qsa_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def __getattr__(name):
    # module-level shortcuts: oracle.decode(...), oracle.topk(...), ...
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(get(), name)
