"""ctypes binding of ``libqsa.so`` (the C ABI declared in include/qsa.h).

Argument marshalling only: torch tensors supply device pointers, strides and
the current stream; every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if the library or a GPU is missing the
calls raise.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsa.so")
SCALE = 1.0 / math.sqrt(128.0)

_i64, _i32, _f32, _vp, _sz = C.c_int64, C.c_int32, C.c_float, C.c_void_p, C.c_size_t

SIGNATURES = {
    "qsa_status_string": (C.c_char_p, [C.c_int]),
    "qsa_last_error_detail": (C.c_char_p, []),
    "qsa_device_error": (C.c_int, [C.POINTER(C.c_uint32)]),
    "qsa_selftest_bounded_wait": (C.c_int, [C.c_uint64, _i32, _vp]),
    "qsa_mqa_decode": (C.c_int, [_vp, _i64, _i64, _i64, _vp, _i64, _i32, _i64, _i64, _vp, _i64, _i32,
                                 _vp, _i32, _i32, _f32, _vp, _i64, _i64, _i32, _vp]),
    "qsa_mqa_decode_f16": (C.c_int, [_vp, _i64, _i64, _i64, _vp, _i64, _i32, _i64, _i64, _vp, _i64, _i32,
                                     _vp, _i32, _i32, _f32, _vp, _i64, _i64, _i32, _vp]),
    "qsa_mqa_prefill_f16": (C.c_int, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _i64, _f32, _vp, _i64,
                                      _i32, _vp]),
    "qsa_mqa_decode_fp8": (C.c_int, [_vp, _i64, _i64, _i64, _vp, _f32, _i64, _i32, _i64, _i64, _vp, _i64,
                                     _i32, _vp, _i32, _i32, _f32, _vp, _i64, _i64, _i32, _vp]),
    "qsa_mqa_prefill": (C.c_int, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _i64, _f32, _vp, _i64,
                                  _i32, _vp]),
    "qsa_prefill_intervals": (C.c_int, [_vp, _vp, _vp, _i32, _i64, _vp, _vp, _vp]),
    "qsa_topk": (C.c_int, [_vp, _i64, _vp, _i64, _i32, _i32, _vp, _i64, _vp]),
    "qsa_topk_ws": (C.c_int, [_vp, _i64, _vp, _i64, _i32, _i32, _vp, _i64, _vp, C.c_size_t, _vp]),
    "qsa_topk_workspace_size": (C.c_size_t, [_i64, _i32, _i32]),
    "qsa_mqa_prefill_topk": (C.c_int, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _i64, _f32, _i32,
                                       _i32, _vp, _i64, _vp, _sz, _vp]),
    "qsa_prefill_topk_workspace_size": (_sz, [_i64, _i32]),
    "qsa_mqa_prefill_topk_noalloc": (C.c_int, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _vp, _i64, _f32, _i32,
                                               _i32, _vp, _i64, _vp]),
    "qsa_expand_block_indices": (C.c_int, [_vp, _i64, _i32, _vp, _vp, _i32, _i64, _vp, _i64, _vp]),
    "qsa_sparse_attention": (C.c_int, [_vp, _i64, _i64, _i32, _vp, _vp, _i64, _i32, _i64, _i64, _i64, _i32,
                                       _vp, _i64, _i32, _vp, _vp, _i32, _vp, _i64, _i32, _i64, _vp, _f32,
                                       _vp, _i64, _vp, _vp, _sz, _vp]),
    "qsa_sparse_attention_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "qsa_mqa_paged_batch": (C.c_int, [_vp, _i64, _i64, _vp, _i64, _i32, _i64, _i64, _vp, _i64, _i32, _vp, _vp,
                                      _i32, _i32, _i32, _i64, _f32, _vp, _i64, _i32, _vp, _sz, _vp]),
    "qsa_mqa_paged_batch_workspace_size": (_sz, [_i32, _i32, _i32, _i64, _i32]),
}

STATUS = {0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_ALIGNMENT", 3: "QSA_ERR_UNSUPPORTED",
          4: "QSA_ERR_WORKSPACE", 5: "QSA_ERR_CUDA"}


class QSAError(RuntimeError):
    def __init__(self, call: str, status: int, detail: str):
        self.call, self.status, self.detail = call, status, detail
        super().__init__(f"{call}: {STATUS.get(status, status)}: {detail}")


_lib = None


def lib() -> C.CDLL:
    """Load the in-tree library (built by ``python -m sparse_attention_block_qsa_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m sparse_attention_block_qsa_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(call: str, status: int) -> None:
    if status != 0:
        raise QSAError(call, status, lib().qsa_last_error_detail().decode())


def _ptr(t: torch.Tensor | None):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, dim: int) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, got {t.dim()}")


def device_error() -> int:
    """Read and clear the library's device error word (synchronises)."""
    v = C.c_uint32(0)
    _check("qsa_device_error", lib().qsa_device_error(C.byref(v)))
    return v.value


def selftest_bounded_wait(timeout_ns: int, arrive: bool, stream=None) -> None:
    """Launch the bounded-wait diagnostic (a wait on a barrier phase that
    nothing completes unless `arrive`); see qsa_selftest_bounded_wait."""
    _check("qsa_selftest_bounded_wait", lib().qsa_selftest_bounded_wait(timeout_ns, 1 if arrive else 0,
                                                                       _stream(stream)))


def _decode_checks(q, k_cache, page_table, seq_lens, W, out, q_dtype=torch.bfloat16):
    _need(q, "q", q_dtype, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Q = q.shape[0], q.shape[1]
    if out is None:
        out = torch.empty((B, Q, W), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, 3)
    if q.shape[2:] != (4, 128) or q.stride(3) != 1:
        raise ValueError("q must be [B, Q, 4, 128] with unit feature stride")
    if k_cache.shape[2:] != (1, 128) or k_cache.stride(3) != 1:
        raise ValueError("k_cache must be [pages, page_size, 1, 128] with unit feature stride")
    if page_table.stride(1) != 1 or seq_lens.stride(0) != 1 or out.stride(2) != 1:
        raise ValueError("page_table, seq_lens and out need a unit innermost stride")
    if out.shape[:2] != (B, Q) or page_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("batch shapes of q, page_table, seq_lens and out disagree")
    return B, Q, out


def mqa_decode(q: torch.Tensor, k_cache: torch.Tensor, page_table: torch.Tensor, seq_lens: torch.Tensor,
               W: int, scale: float = SCALE, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode / spec-decode scores: q [B, Q, 4, 128] and k_cache [pages,
    page_size, 1, 128] both bf16 or both fp16, page_table int32 [B,
    max_pages], seq_lens int32 [B] (tokens) -> out fp32 [B, Q, W]."""
    dt = q.dtype if isinstance(q, torch.Tensor) and q.dtype == torch.float16 else torch.bfloat16
    _need(k_cache, "k_cache", dt, 4)
    B, Q, out = _decode_checks(q, k_cache, page_table, seq_lens, W, out, dt)
    name = "qsa_mqa_decode_f16" if dt == torch.float16 else "qsa_mqa_decode"
    _check(name, getattr(lib(), name)(
        _ptr(q), q.stride(0), q.stride(1), q.stride(2),
        _ptr(k_cache), k_cache.shape[0], k_cache.shape[1], k_cache.stride(0), k_cache.stride(1),
        _ptr(page_table), page_table.stride(0), page_table.shape[1], _ptr(seq_lens), B, Q, scale,
        _ptr(out), out.stride(0), out.stride(1), out.shape[2], _stream(stream)))
    return out


def mqa_decode_fp8(q: torch.Tensor, k_cache: torch.Tensor, k_scale: float, page_table: torch.Tensor,
                   seq_lens: torch.Tensor, W: int, scale: float = SCALE, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """mqa_decode over an fp8 E4M3 key cache: k_cache float8_e4m3fn (or uint8
    codes) [pages, page_size, 1, 128] holding e4m3(bf16(k) / k_scale); keys
    are read as E4M3 value * k_scale (k_scale > 0)."""
    if isinstance(k_cache, torch.Tensor) and k_cache.dtype == torch.float8_e4m3fn:
        k_cache = k_cache.view(torch.uint8)
    _need(k_cache, "k_cache", torch.uint8, 4)
    B, Q, out = _decode_checks(q, k_cache, page_table, seq_lens, W, out)
    _check("qsa_mqa_decode_fp8", lib().qsa_mqa_decode_fp8(
        _ptr(q), q.stride(0), q.stride(1), q.stride(2),
        _ptr(k_cache), float(k_scale), k_cache.shape[0], k_cache.shape[1], k_cache.stride(0), k_cache.stride(1),
        _ptr(page_table), page_table.stride(0), page_table.shape[1], _ptr(seq_lens), B, Q, scale,
        _ptr(out), out.stride(0), out.stride(1), out.shape[2], _stream(stream)))
    return out


def _prefill_checks(q, k, ks, ke, dt=torch.bfloat16):
    _need(q, "q", dt, 3)
    _need(k, "k", dt, 2)
    _need(ks, "ks", torch.int32, 1)
    _need(ke, "ke", torch.int32, 1)
    if q.shape[1:] != (4, 128) or q.stride(2) != 1:
        raise ValueError("q must be [T, 4, 128] with unit feature stride")
    if k.shape[1] != 128 or k.stride(1) != 1:
        raise ValueError("k must be [Nk, 128] with unit feature stride")
    if ks.shape[0] != q.shape[0] or ke.shape[0] != q.shape[0] or ks.stride(0) != 1 or ke.stride(0) != 1:
        raise ValueError("ks and ke must be contiguous int32 [T]")


def mqa_prefill(q: torch.Tensor, k: torch.Tensor, ks: torch.Tensor, ke: torch.Tensor, W: int,
                scale: float = SCALE, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Prefill scores: q [T, 4, 128] and k [Nk, 128] both bf16 or both fp16,
    ks/ke int32 [T] -> out fp32 [T, W] with out[t, j] the score of key ks[t] + j."""
    dt = q.dtype if isinstance(q, torch.Tensor) and q.dtype == torch.float16 else torch.bfloat16
    _prefill_checks(q, k, ks, ke, dt)
    T = q.shape[0]
    if out is None:
        out = torch.empty((T, W), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, 2)
    if out.shape[0] != T or out.stride(1) != 1:
        raise ValueError("out must be [T, W] with unit column stride")
    name = "qsa_mqa_prefill_f16" if dt == torch.float16 else "qsa_mqa_prefill"
    _check(name, getattr(lib(), name)(
        _ptr(q), q.stride(0), q.stride(1), _ptr(k), k.stride(0), k.shape[0], _ptr(ks), _ptr(ke), T, scale,
        _ptr(out), out.stride(0), out.shape[1], _stream(stream)))
    return out


def prefill_intervals(cu_seqlens_q: torch.Tensor, seq_lens: torch.Tensor, key_offsets: torch.Tensor, T: int,
                      ks: torch.Tensor | None = None, ke: torch.Tensor | None = None, stream=None):
    """Per-row key intervals (ks, ke) int32 [T] of a packed prefill batch."""
    for t, n in ((cu_seqlens_q, "cu_seqlens_q"), (seq_lens, "seq_lens"), (key_offsets, "key_offsets")):
        _need(t, n, torch.int32, 1)
        if t.stride(0) != 1:
            raise ValueError(f"{n} must be contiguous")
    S = seq_lens.shape[0]
    if cu_seqlens_q.shape[0] != S + 1 or key_offsets.shape[0] != S:
        raise ValueError("cu_seqlens_q must have S + 1 entries and key_offsets S")
    dev = seq_lens.device
    ks = torch.empty(T, dtype=torch.int32, device=dev) if ks is None else ks
    ke = torch.empty(T, dtype=torch.int32, device=dev) if ke is None else ke
    _check("qsa_prefill_intervals", lib().qsa_prefill_intervals(
        _ptr(cu_seqlens_q), _ptr(seq_lens), _ptr(key_offsets), S, T, _ptr(ks), _ptr(ke), _stream(stream)))
    return ks, ke


def topk_workspace_size(rows: int, W: int, k: int) -> int:
    return int(lib().qsa_topk_workspace_size(rows, W, k))


def topk(scores: torch.Tensor, k: int, lengths: torch.Tensor | None = None, idx: torch.Tensor | None = None,
         stream=None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Top-k column indices int32 [rows, k] (ascending, -1 padded) of score rows fp32 [rows, W];
    with a workspace (a device tensor of at least topk_workspace_size bytes) through qsa_topk_ws."""
    _need(scores, "scores", torch.float32, 2)
    if scores.stride(1) != 1:
        raise ValueError("scores need a unit column stride")
    rows, W = scores.shape
    if lengths is not None:
        _need(lengths, "lengths", torch.int32, 1)
        if lengths.shape[0] != rows or lengths.stride(0) != 1:
            raise ValueError("lengths must be contiguous int32 [rows]")
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    _need(idx, "idx", torch.int32, 2)
    if idx.shape != (rows, k) or idx.stride(1) != 1:
        raise ValueError("idx must be [rows, k] with unit column stride")
    if workspace is not None:
        if not workspace.is_contiguous():
            raise ValueError("workspace must be contiguous")
        nbytes = workspace.numel() * workspace.element_size()
        _check("qsa_topk_ws", lib().qsa_topk_ws(_ptr(scores), scores.stride(0), _ptr(lengths), rows, W, k, _ptr(idx),
                                                idx.stride(0), _ptr(workspace), nbytes, _stream(stream)))
        return idx
    _check("qsa_topk", lib().qsa_topk(_ptr(scores), scores.stride(0), _ptr(lengths), rows, W, k, _ptr(idx),
                                      idx.stride(0), _stream(stream)))
    return idx


def prefill_topk_workspace_size(T: int, W: int) -> int:
    return int(lib().qsa_prefill_topk_workspace_size(T, W))


def mqa_prefill_topk(q: torch.Tensor, k: torch.Tensor, ks: torch.Tensor, ke: torch.Tensor, W: int,
                     topk_k: int, workspace: torch.Tensor, scale: float = SCALE,
                     idx: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Prefill scores followed by per-row top-k, chunked through ``workspace``
    (a CUDA tensor, any dtype, 16-byte aligned) -> idx int32 [T, topk_k]."""
    _prefill_checks(q, k, ks, ke)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    T = q.shape[0]
    if idx is None:
        idx = torch.empty((T, topk_k), dtype=torch.int32, device=q.device)
    _need(idx, "idx", torch.int32, 2)
    if idx.shape != (T, topk_k) or idx.stride(1) != 1:
        raise ValueError("idx must be [T, topk_k] with unit column stride")
    _check("qsa_mqa_prefill_topk", lib().qsa_mqa_prefill_topk(
        _ptr(q), q.stride(0), q.stride(1), _ptr(k), k.stride(0), k.shape[0], _ptr(ks), _ptr(ke), T, scale, W,
        topk_k, _ptr(idx), idx.stride(0), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))
    return idx


def mqa_prefill_topk_noalloc(q: torch.Tensor, k: torch.Tensor, ks: torch.Tensor, ke: torch.Tensor, W: int,
                             topk_k: int, scale: float = SCALE, idx: torch.Tensor | None = None,
                             stream=None) -> torch.Tensor:
    """Prefill scores followed by per-row top-k through the library's static
    scratch (no device allocation by the library) -> idx int32 [T, topk_k].
    Calls that overlap on the GPU share that scratch and must be serialised."""
    _prefill_checks(q, k, ks, ke)
    T = q.shape[0]
    if idx is None:
        idx = torch.empty((T, topk_k), dtype=torch.int32, device=q.device)
    _need(idx, "idx", torch.int32, 2)
    if idx.shape != (T, topk_k) or idx.stride(1) != 1:
        raise ValueError("idx must be [T, topk_k] with unit column stride")
    _check("qsa_mqa_prefill_topk_noalloc", lib().qsa_mqa_prefill_topk_noalloc(
        _ptr(q), q.stride(0), q.stride(1), _ptr(k), k.stride(0), k.shape[0], _ptr(ks), _ptr(ke), T, scale, W,
        topk_k, _ptr(idx), idx.stride(0), _stream(stream)))
    return idx


def _index_checks(cu_seqlens_q, seq_lens):
    for t, n in ((cu_seqlens_q, "cu_seqlens_q"), (seq_lens, "seq_lens")):
        _need(t, n, torch.int32, 1)
        if t.stride(0) != 1:
            raise ValueError(f"{n} must be contiguous")
    if cu_seqlens_q.shape[0] != seq_lens.shape[0] + 1:
        raise ValueError("cu_seqlens_q must have one more entry than seq_lens")


def expand_block_indices(blocks: torch.Tensor, cu_seqlens_q: torch.Tensor, seq_lens: torch.Tensor,
                         token_idx: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Selected blocks int32 [T, k] -> token indices int32 [T, 4k + 3] (four
    tokens per block, then the row's open group, then -1)."""
    _need(blocks, "blocks", torch.int32, 2)
    _index_checks(cu_seqlens_q, seq_lens)
    if blocks.stride(1) != 1:
        raise ValueError("blocks need a unit column stride")
    T, k = blocks.shape
    if token_idx is None:
        token_idx = torch.empty((T, 4 * k + 3), dtype=torch.int32, device=blocks.device)
    _need(token_idx, "token_idx", torch.int32, 2)
    if token_idx.shape != (T, 4 * k + 3) or token_idx.stride(1) != 1:
        raise ValueError("token_idx must be [T, 4k + 3] with unit column stride")
    _check("qsa_expand_block_indices", lib().qsa_expand_block_indices(
        _ptr(blocks), blocks.stride(0), k, _ptr(cu_seqlens_q), _ptr(seq_lens), seq_lens.shape[0], T,
        _ptr(token_idx), token_idx.stride(0), _stream(stream)))
    return token_idx


def sparse_attention_workspace_size(T: int, Hq: int, Hkv: int, width: int) -> int:
    return int(lib().qsa_sparse_attention_workspace_size(T, Hq, Hkv, width))


def sparse_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                     cu_seqlens_q: torch.Tensor, seq_lens: torch.Tensor, token_idx: torch.Tensor, scale: float,
                     gate: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """Sparse core attention: q bf16 [T, Hq, 256], K/V bf16 [pages, page_size,
    Hkv, 256], token_idx int32 [T, width] -> (out bf16 [T, Hq, 256], lse fp32
    [T, Hq]).  The workspace (any CUDA tensor, 16-byte aligned) is allocated
    here by torch when not given."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _need(token_idx, "token_idx", torch.int32, 2)
    _index_checks(cu_seqlens_q, seq_lens)
    T, Hq, Dq = q.shape
    if Dq != 256 or q.stride(2) != 1:
        raise ValueError("q must be [T, Hq, 256] with unit feature stride")
    if k_cache.shape != v_cache.shape or k_cache.stride() != v_cache.stride() or k_cache.shape[3] != 256 \
            or k_cache.stride(3) != 1:
        raise ValueError("k_cache and v_cache must be [pages, page_size, Hkv, 256] with the same strides")
    if token_idx.shape[0] != T or token_idx.stride(1) != 1 or page_table.stride(1) != 1:
        raise ValueError("token_idx must be [T, width] and page_table [R, max_pages], unit column strides")
    if page_table.shape[0] != seq_lens.shape[0]:
        raise ValueError("page_table needs one row per request")
    Hkv = k_cache.shape[2]
    width = token_idx.shape[1]
    if gate is not None:
        _need(gate, "gate", torch.float32, 2)
        if gate.shape != (T, Hq) or not gate.is_contiguous():
            raise ValueError("gate must be contiguous fp32 [T, Hq]")
    if out is None:
        out = torch.empty((T, Hq, 256), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, 3)
    if out.shape != (T, Hq, 256) or out.stride(2) != 1 or out.stride(1) != 256:
        raise ValueError("out must be [T, Hq, 256] with contiguous heads")
    if lse is None:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    _need(lse, "lse", torch.float32, 2)
    if lse.shape != (T, Hq) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32 [T, Hq]")
    need = sparse_attention_workspace_size(T, Hq, Hkv, max(width, 1))
    if workspace is None:
        workspace = torch.empty(max(need, 16) // 4 + 4, dtype=torch.float32, device=q.device)
    _check("qsa_sparse_attention", lib().qsa_sparse_attention(
        _ptr(q), q.stride(0), q.stride(1), Hq, _ptr(k_cache), _ptr(v_cache), k_cache.shape[0], k_cache.shape[1],
        k_cache.stride(0), k_cache.stride(1), k_cache.stride(2), Hkv, _ptr(page_table), page_table.stride(0),
        page_table.shape[1], _ptr(cu_seqlens_q), _ptr(seq_lens), seq_lens.shape[0], _ptr(token_idx),
        token_idx.stride(0), width, T, _ptr(gate), float(scale), _ptr(out), out.stride(0), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, lse


def paged_batch_workspace_size(R: int, num_decodes: int, decode_query_len: int, T: int, W: int) -> int:
    return int(lib().qsa_mqa_paged_batch_workspace_size(R, num_decodes, decode_query_len, T, W))


def mqa_paged_batch(q: torch.Tensor, k_cache: torch.Tensor, page_table: torch.Tensor, cu_seqlens_q: torch.Tensor,
                    seq_lens: torch.Tensor, num_decodes: int, decode_query_len: int, W: int, scale: float = SCALE,
                    out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """Scores of a mixed batch from the paged cache: q bf16 [T, 4, 128] (the
    num_decodes x decode_query_len decode rows first), k_cache bf16 [pages,
    page_size, 1, 128], page_table int32 [R, max_pages], cu_seqlens_q int32
    [R + 1], seq_lens int32 [R] -> out fp32 [T, W] (request-local key
    columns).  The workspace is allocated here by torch when not given."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _index_checks(cu_seqlens_q, seq_lens)
    if q.shape[1:] != (4, 128) or q.stride(2) != 1:
        raise ValueError("q must be [T, 4, 128] with unit feature stride")
    if k_cache.shape[2:] != (1, 128) or k_cache.stride(3) != 1 or page_table.stride(1) != 1:
        raise ValueError("k_cache must be [pages, page_size, 1, 128]; page_table needs a unit column stride")
    T = q.shape[0]
    R = seq_lens.shape[0]
    if out is None:
        out = torch.empty((T, W), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, 2)
    if out.shape != (T, W) or out.stride(1) != 1:
        raise ValueError("out must be [T, W] with unit column stride")
    if workspace is None:
        need = paged_batch_workspace_size(R, num_decodes, decode_query_len, T, W)
        workspace = torch.empty(max(need, 16) // 4 + 4, dtype=torch.float32, device=q.device)
    _check("qsa_mqa_paged_batch", lib().qsa_mqa_paged_batch(
        _ptr(q), q.stride(0), q.stride(1), _ptr(k_cache), k_cache.shape[0], k_cache.shape[1], k_cache.stride(0),
        k_cache.stride(1), _ptr(page_table), page_table.stride(0), page_table.shape[1], _ptr(cu_seqlens_q),
        _ptr(seq_lens), R, num_decodes, decode_query_len, T, scale, _ptr(out), out.stride(0), W,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out
