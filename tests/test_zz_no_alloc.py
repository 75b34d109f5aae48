"""The no-allocation fused prefill + top-k entry point (B200 only).

Some callers cannot allocate device memory when they call the indexer: a
host program whose device memory a framework plans up front, or a thread
where cudaMalloc is not allowed because it may synchronise the device.
qsa_mqa_prefill_topk_noalloc serves them from a static scratch array inside
the library.  Through the C ABI, two calls in a row must give the same block
indices as qsa_mqa_prefill_topk with a caller workspace (index results are
compared exactly).  The file sorts last so that a stop-at-first-failure run
has run every other test first; it also passes alone in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
from sparse_attention_block_qsa_b200 import _abi  # noqa: E402

DEV = torch.device("cuda")


def _p(t):
    return C.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_twice():
    # two packed sequences, long enough for several scratch chunks (W = 6506 ->
    # 16 MiB holds 640 rows of scores; 1800 rows need three chunks)
    p = wl.make_prefill("noalloc", [1000, 800], [25000, 4000], seed=21)
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    q, k = p.q.to(DEV), p.k.to(DEV)
    ks_d, ke_d = torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV)
    kk = 128
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    L = _abi.lib()

    ws = torch.empty(_abi.prefill_topk_workspace_size(p.T, p.W) // 4 + 1, dtype=torch.float32, device=DEV)
    want = torch.empty((p.T, kk), dtype=torch.int32, device=DEV)
    st = L.qsa_mqa_prefill_topk(_p(q), q.stride(0), q.stride(1), _p(k), k.stride(0), p.Nk, _p(ks_d), _p(ke_d), p.T,
                                _abi.SCALE, p.W, kk, _p(want), kk, _p(ws), ws.numel() * 4, stream)
    assert st == 0, L.qsa_last_error_detail().decode()

    for call in range(2):
        got = torch.full((p.T, kk), -7, dtype=torch.int32, device=DEV)
        st = L.qsa_mqa_prefill_topk_noalloc(_p(q), q.stride(0), q.stride(1), _p(k), k.stride(0), p.Nk, _p(ks_d),
                                            _p(ke_d), p.T, _abi.SCALE, p.W, kk, _p(got), kk, stream)
        assert st == 0, L.qsa_last_error_detail().decode()
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"call {call}: indices differ from the workspace entry point"
    assert qsa.device_error() == 0


def test_noalloc_rejects_rows_beyond_the_scratch():
    q = torch.zeros(64, 4, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(64, 128, dtype=torch.bfloat16, device=DEV)
    ks = torch.zeros(64, dtype=torch.int32, device=DEV)
    idx = torch.empty((64, 16), dtype=torch.int32, device=DEV)
    with pytest.raises(qsa.QSAError) as e:
        qsa.mqa_prefill_topk_noalloc(q, k, ks, ks, 65536, 16, idx=idx)
    assert e.value.status == 4


def test_noalloc_widest_rows_fill_the_scratch_exactly():
    # W = 65520: one chunk of 64 rows of scores plus the 4 KB of selection
    # state fills the 16 MiB scratch exactly; the result must equal the
    # workspace entry point's.  W = 65521 no longer fits and is refused.
    T, W, kk = 64, 65520, 16
    g = torch.Generator().manual_seed(5)
    q = torch.randn(T, 4, 128, generator=g).to(torch.bfloat16).to(DEV)
    k = torch.randn(W, 128, generator=g).to(torch.bfloat16).to(DEV)
    ks = torch.zeros(T, dtype=torch.int32, device=DEV)
    ke = torch.arange(T, dtype=torch.int32, device=DEV) * 3 + 40     # 40 .. 229 visible keys per row
    ke[-1] = W                                                       # one row sees every key
    ws = torch.empty(_abi.prefill_topk_workspace_size(T, W) // 4, dtype=torch.float32, device=DEV)
    want = qsa.mqa_prefill_topk(q, k, ks, ke, W, kk, ws)
    for _ in range(2):
        got = qsa.mqa_prefill_topk_noalloc(q, k, ks, ke, W, kk)
        torch.cuda.synchronize()
        assert torch.equal(got, want)
    assert qsa.device_error() == 0
    with pytest.raises(qsa.QSAError) as e:
        qsa.mqa_prefill_topk_noalloc(q, k, ks, ke, W + 1, kk)
    assert e.value.status == 4
