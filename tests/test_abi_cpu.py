"""The C-ABI library on a host without a GPU: it loads, exports every entry
point include/qsa.h declares, and rejects bad arguments on the host before
any CUDA call (no compute runs here)."""
import ctypes as C
import os
import re
import subprocess

import pytest
import torch

import sparse_attention_block_qsa_b200 as qsa
from sparse_attention_block_qsa_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qsa.h")

OK, INVALID, ALIGN, UNSUP, WS = 0, 1, 2, 3, 4
# fake device addresses: validation never dereferences them
A = 0x7f0000000000
S = 1 << 28        # distance between fake buffers


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 9
    L = qsa.lib()
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (qsa_\w+)", out))
    assert set(names) <= exported
    assert set(names) == set(_abi.SIGNATURES), "binding and header disagree"


def test_status_strings():
    L = qsa.lib()
    for code in range(6):
        assert L.qsa_status_string(code).decode().startswith(_abi.STATUS[code])


def decode(**kw):
    a = dict(q=A, sb=2048, st=512, sh=128, k=A + S, pages=100, ps=64, kps=64 * 128, krs=128, pt=A + 2 * S,
             pts=10, maxp=10, sl=A + 3 * S, B=4, Q=4, scale=0.088, out=A + 4 * S, osb=4 * 1000, ost=1000, W=1000)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_mqa_decode(a["q"], a["sb"], a["st"], a["sh"], a["k"], a["pages"], a["ps"], a["kps"], a["krs"],
                          a["pt"], a["pts"], a["maxp"], a["sl"], a["B"], a["Q"], a["scale"], a["out"], a["osb"],
                          a["ost"], a["W"], None)
    return st, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(Q=5), UNSUP), (dict(Q=0), UNSUP), (dict(ps=7), UNSUP), (dict(ps=1025), UNSUP),
    (dict(B=-1), INVALID), (dict(W=-1), INVALID), (dict(pages=0), INVALID), (dict(maxp=-1), INVALID),
    (dict(scale=float("nan")), INVALID), (dict(q=0), INVALID), (dict(out=0), INVALID),
    (dict(q=A + 2), ALIGN), (dict(k=A + S + 8), ALIGN), (dict(out=A + 4 * S + 2), ALIGN),
    (dict(sh=100), ALIGN), (dict(st=-8), ALIGN), (dict(krs=120), ALIGN), (dict(kps=7), ALIGN),
    (dict(pts=5), INVALID), (dict(ost=10), INVALID), (dict(osb=100), INVALID),
    (dict(out=A + 100), INVALID),                      # out overlaps q
])
def test_decode_rejects(kw, code):
    st, detail = decode(**kw)
    assert st == code, detail
    assert detail


def test_decode_empty_batch_is_a_no_op():
    assert decode(B=0)[0] == OK
    assert decode(W=0)[0] == OK


def decode_fp8(**kw):
    a = dict(q=A, sb=2048, st=512, sh=128, k=A + S, kscale=0.01, pages=100, ps=64, kps=64 * 128, krs=128,
             pt=A + 2 * S, pts=10, maxp=10, sl=A + 3 * S, B=4, Q=4, scale=0.088, out=A + 4 * S, osb=4 * 1000,
             ost=1000, W=1000)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_mqa_decode_fp8(a["q"], a["sb"], a["st"], a["sh"], a["k"], a["kscale"], a["pages"], a["ps"],
                              a["kps"], a["krs"], a["pt"], a["pts"], a["maxp"], a["sl"], a["B"], a["Q"], a["scale"],
                              a["out"], a["osb"], a["ost"], a["W"], None)
    return st, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(kscale=0.0), INVALID), (dict(kscale=-0.5), INVALID), (dict(kscale=float("nan")), INVALID),
    (dict(kscale=float("inf")), INVALID), (dict(kscale=1e30, scale=1e30), INVALID),
    (dict(krs=136), ALIGN),            # 8-byte multiple: fine for bf16 elements, not for 1-byte codes
    (dict(kps=64 * 128 + 8), ALIGN), (dict(krs=112), ALIGN), (dict(k=A + S + 8), ALIGN),
    (dict(Q=5), UNSUP), (dict(ps=4), UNSUP), (dict(sh=100), ALIGN),
    (dict(out=A + S + 64), INVALID),   # out overlaps the 1-byte cache
])
def test_decode_fp8_rejects(kw, code):
    st, detail = decode_fp8(**kw)
    assert st == code, detail
    assert detail


def test_decode_fp8_empty_batch_is_a_no_op():
    assert decode_fp8(B=0)[0] == OK
    assert decode_fp8(W=0)[0] == OK


def test_decode_fp8_cache_span_uses_one_byte_elements():
    # the bf16 span of this cache (100 pages x 16 KB) would reach out; the fp8 one (100 x 8 KB) does not
    end8 = A + S + 100 * 64 * 128
    st, detail = decode_fp8(out=end8 + 4096)     # passes validation (then needs a GPU)
    assert st != INVALID and "overlap" not in detail, detail
    st, detail = decode_fp8(out=end8 - 4096)
    assert st == INVALID and "overlap" in detail, detail


def prefill(**kw):
    a = dict(q=A, st=512, sh=128, k=A + S, ks_=128, Nk=1000, ks=A + 2 * S, ke=A + 3 * S, T=100, scale=0.088,
             out=A + 4 * S, os=2000, W=1000)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_mqa_prefill(a["q"], a["st"], a["sh"], a["k"], a["ks_"], a["Nk"], a["ks"], a["ke"], a["T"],
                           a["scale"], a["out"], a["os"], a["W"], None)
    return st, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(T=-1), INVALID), (dict(Nk=-3), INVALID), (dict(W=-1), INVALID), (dict(T=1 << 31), UNSUP),
    (dict(q=A + 8), ALIGN), (dict(k=A + S + 4), ALIGN), (dict(sh=0), ALIGN), (dict(st=0), ALIGN),
    (dict(st=100), ALIGN), (dict(ks_=64), ALIGN), (dict(os=999), INVALID), (dict(ks=0), INVALID),
    (dict(out=A + 2 * S), INVALID),                    # out overlaps ks
    (dict(scale=float("inf")), INVALID),
])
def test_prefill_rejects(kw, code):
    st, detail = prefill(**kw)
    assert st == code, detail


def test_prefill_empty_is_a_no_op():
    assert prefill(T=0)[0] == OK
    assert prefill(W=0)[0] == OK


def topk(**kw):
    a = dict(s=A, ss=5000, ln=0, rows=10, W=5000, k=512, idx=A + S, iss=512)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_topk(a["s"], a["ss"], a["ln"] or None, a["rows"], a["W"], a["k"], a["idx"], a["iss"], None)
    return st, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), UNSUP), (dict(k=2049), UNSUP), (dict(W=0), UNSUP), (dict(W=70000), UNSUP),
    (dict(rows=-1), INVALID), (dict(ss=10), INVALID), (dict(iss=100), INVALID), (dict(s=A + 2), ALIGN),
    (dict(idx=A + 4), INVALID),                         # idx overlaps scores
])
def test_topk_rejects(kw, code):
    st, detail = topk(**kw)
    assert st == code, detail


def topk_ws(ws=None, nbytes=None, **kw):
    a = dict(s=A, ss=5000, ln=0, rows=10, W=5000, k=512, idx=A + S, iss=512)
    a.update(kw)
    L = qsa.lib()
    need = L.qsa_topk_workspace_size(a["rows"], a["W"], a["k"])
    ws = A + 2 * S if ws is None else ws
    nbytes = need if nbytes is None else nbytes
    st = L.qsa_topk_ws(a["s"], a["ss"], a["ln"] or None, a["rows"], a["W"], a["k"], a["idx"], a["iss"], ws, nbytes,
                       None)
    return st, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), UNSUP), (dict(rows=-1), INVALID), (dict(s=A + 2), ALIGN),
    (dict(ws=0), INVALID), (dict(ws=A + 2 * S + 128), ALIGN), (dict(nbytes=1000), WS),
    (dict(ws=A), INVALID),                              # the workspace overlaps scores
    (dict(ws=A + S - 256), INVALID),                    # ... and idx
])
def test_topk_ws_rejects(kw, code):
    st, detail = topk_ws(**kw)
    assert st == code, detail


def test_topk_workspace_size():
    L = qsa.lib()
    size = L.qsa_topk_workspace_size
    # per row: a 64-byte header, a 256-bin histogram, 4096 keys and 4096 columns
    assert size(16384, 26624, 512) >= 16384 * (64 + 1024 + 4096 * 6)
    assert size(1, 26624, 512) < size(2, 26624, 512) and size(0, 100, 5) == 0
    assert size(1000, 100, 5) % 256 == 0


def test_fused_rejects_small_workspace():
    L = qsa.lib()
    st = L.qsa_mqa_prefill_topk(A, 512, 128, A + S, 128, 1000, A + 2 * S, A + 3 * S, 1000, 0.088, 1000, 512,
                                A + 4 * S, 512, A + 5 * S, 63 * 1000 * 4, None)
    assert st == WS, L.qsa_last_error_detail().decode()
    # one chunk of all rows in either layout: at least the score-row layout's
    # T rows of W floats plus 4096 bytes, growing with T, zero when empty
    size = L.qsa_prefill_topk_workspace_size
    assert size(16384, 26624) >= 16384 * 26624 * 4 + 4096
    assert size(64, 26624) < size(65, 26624) < size(16384, 26624)
    assert size(0, 26624) == 0 and size(16, 0) == 0


def test_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        qsa.mqa_decode(q, torch.zeros(1, 16, 1, 128, dtype=torch.bfloat16), torch.zeros(1, 1, dtype=torch.int32),
                       torch.zeros(1, dtype=torch.int32), 4)


def test_fp8_binding_refuses_cpu_tensors_and_wrong_dtypes():
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    pt, sl = torch.zeros(1, 1, dtype=torch.int32), torch.zeros(1, dtype=torch.int32)
    for kc in (torch.zeros(1, 16, 1, 128, dtype=torch.uint8),
               torch.zeros(1, 16, 1, 128, dtype=torch.float8_e4m3fn),
               torch.zeros(1, 16, 1, 128, dtype=torch.bfloat16)):
        with pytest.raises(TypeError):
            qsa.mqa_decode_fp8(q, kc, 0.5, pt, sl, 4)


def test_oracle_fp8_accepts_float8_and_uint8_views():
    import numpy as np
    import oracle
    import workloads as wl
    d = wl.make_decode("views", [300, 77], Q=2, page_size=8, seed=3)
    codes, ks = wl.e4m3_cache(d.k_cache)
    a = oracle.decode_fp8(d.q, codes, ks, d.page_table, d.seq_lens, d.W, threads=1)
    b = oracle.decode_fp8(d.q, codes.view(torch.float8_e4m3fn), ks, d.page_table, d.seq_lens, d.W, threads=1)
    assert np.array_equal(a, b)
    assert np.isfinite(a).any()


def test_selftest_rejects_long_limit():
    L = qsa.lib()
    assert L.qsa_selftest_bounded_wait(20_000_000_000, 0, None) == INVALID, L.qsa_last_error_detail().decode()


def attention(**kw):
    a = dict(q=A, qst=24 * 256, qsh=256, Hq=24, k=A + S, v=A + 2 * S, pages=100, ps=64, kps=64 * 512, krs=512,
             khs=256, Hkv=2, pt=A + 3 * S, pts=10, maxp=10, cu=A + 4 * S, sl=A + 4 * S + 4096, R=4, tok=A + 5 * S,
             toks=2051, width=2051, T=16, gate=None, scale=0.0625, out=A + 6 * S, ost=24 * 256, lse=None,
             ws=A + 7 * S, wsb=1 << 30)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_sparse_attention(a["q"], a["qst"], a["qsh"], a["Hq"], a["k"], a["v"], a["pages"], a["ps"], a["kps"],
                                a["krs"], a["khs"], a["Hkv"], a["pt"], a["pts"], a["maxp"], a["cu"], a["sl"], a["R"],
                                a["tok"], a["toks"], a["width"], a["T"], a["gate"], a["scale"], a["out"], a["ost"],
                                a["lse"], a["ws"], a["wsb"], None)
    return st, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=25), UNSUP), (dict(Hq=34, Hkv=2), UNSUP), (dict(Hkv=0), UNSUP), (dict(T=-1), INVALID),
    (dict(ps=0), INVALID), (dict(pages=0), INVALID), (dict(scale=float("inf")), INVALID), (dict(R=0), INVALID),
    (dict(q=0), INVALID), (dict(out=0), INVALID), (dict(tok=0), INVALID),
    (dict(q=A + 8), ALIGN), (dict(k=A + S + 2), ALIGN), (dict(out=A + 6 * S + 4), ALIGN),
    (dict(qsh=100), ALIGN), (dict(krs=500), ALIGN), (dict(qsh=128), INVALID), (dict(khs=128), INVALID),
    (dict(krs=256), INVALID), (dict(ost=256), INVALID), (dict(toks=100), INVALID), (dict(pts=5), INVALID),
    (dict(out=A + 112), INVALID),                      # out overlaps q
    (dict(wsb=1024), WS), (dict(ws=0), WS),
])
def test_attention_rejects(kw, code):
    st, detail = attention(**kw)
    assert st == code, detail
    assert detail


def test_attention_workspace_size():
    n = qsa.sparse_attention_workspace_size(64, 24, 2, 2051)
    # 64 rows x 2 KV heads = 128 pairs -> floor(1332 / 128) = 10 splits of ceil(65 / 10) = 7
    # of the 65 chunks of 32 entries (ceil(65 / 7) = 10 runs); 12 heads x (256 + 2) floats per split
    assert n == 64 * 2 * 10 * 12 * 258 * 4
    assert qsa.sparse_attention_workspace_size(0, 24, 2, 2051) == 0
    assert qsa.sparse_attention_workspace_size(4, 24, 5, 2051) == 0


@pytest.mark.parametrize("kw,code", [(dict(k=0), UNSUP), (dict(k=513), UNSUP), (dict(T=-1), INVALID),
                                     (dict(R=0), INVALID), (dict(blk=0), INVALID), (dict(tok=A + 2), ALIGN),
                                     (dict(tks=10), INVALID), (dict(tok=A + 4), INVALID)])
def test_expand_rejects(kw, code):
    a = dict(blk=A, bs=512, k=512, cu=A + S, sl=A + S + 4096, R=4, T=16, tok=A + 2 * S, tks=2051)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_expand_block_indices(a["blk"], a["bs"], a["k"], a["cu"], a["sl"], a["R"], a["T"], a["tok"], a["tks"],
                                    None)
    assert st == code, L.qsa_last_error_detail().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(D=5), INVALID), (dict(R=-1), INVALID), (dict(Qd=5), UNSUP), (dict(Qd=0), UNSUP),
    (dict(T=3), INVALID), (dict(D=4, T=20), INVALID), (dict(ps=7), UNSUP), (dict(W=1 << 30), UNSUP),
    (dict(q=0), INVALID), (dict(ost=10), INVALID), (dict(wsb=100), WS), (dict(ws=A + 7 * S + 8), ALIGN),
])
def test_paged_batch_rejects(kw, code):
    a = dict(q=A, qst=512, qsh=128, k=A + S, pages=100, ps=64, kps=64 * 128, krs=128, pt=A + 2 * S, pts=10, maxp=10,
             cu=A + 3 * S, sl=A + 3 * S + 4096, R=4, D=2, Qd=4, T=40, scale=0.088, out=A + 4 * S, ost=1000, W=1000,
             ws=A + 7 * S, wsb=1 << 30)
    a.update(kw)
    L = qsa.lib()
    st = L.qsa_mqa_paged_batch(a["q"], a["qst"], a["qsh"], a["k"], a["pages"], a["ps"], a["kps"], a["krs"], a["pt"],
                               a["pts"], a["maxp"], a["cu"], a["sl"], a["R"], a["D"], a["Qd"], a["T"], a["scale"],
                               a["out"], a["ost"], a["W"], a["ws"], a["wsb"], None)
    assert st == code, L.qsa_last_error_detail().decode()


def test_paged_batch_workspace_size():
    # 2 prefill requests x W = 1000 keys x 256 bytes, then ks and ke of the 32 prefill rows
    assert qsa.paged_batch_workspace_size(4, 2, 4, 40, 1000) == 2 * 1000 * 256 + 2 * 128
    assert qsa.paged_batch_workspace_size(4, 4, 4, 16, 1000) == 0       # decodes only


@pytest.mark.skipif(torch.cuda.is_available(), reason="passes validation and would launch on fake addresses")
def test_fused_workspace_is_checked_per_chunk_not_per_batch():
    """A small workspace followed in memory by idx (within T x W floats of the
    workspace start) is valid: the workspace only ever holds one chunk of rows.
    Validation passes and the call fails later, at the first CUDA call (no GPU
    here)."""
    L = qsa.lib()
    T, W, kk = 4096, 26624, 512
    ws_bytes = 64 << 20
    ws = A + 5 * S
    idx = ws + ws_bytes + 4096                       # right after the workspace
    st = L.qsa_mqa_prefill_topk(A, 512, 128, A + S, 128, 106496, A + 2 * S, A + 3 * S, T, 0.088, W, kk, idx, kk,
                                ws, ws_bytes, None)
    assert st == 5, L.qsa_last_error_detail().decode()   # QSA_ERR_CUDA: validation passed
