"""fp16 inputs and page sizes that are not powers of two (B200 only): the
CUDA path through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import compare_scores, decode_bounds, prefill_bounds

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
SCALE = 1.0 / np.sqrt(128.0)
DEV = torch.device("cuda", 0)


def _decode(d, q, kc, W=None):
    W = d.W if W is None else W
    res = qsa.mqa_decode(q.to(DEV), kc.to(DEV), d.page_table.to(DEV), d.seq_lens.to(DEV), W, scale=SCALE)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    ref = oracle.decode(q, kc, d.page_table, d.seq_lens, W, scale=SCALE)
    loose, tight = decode_bounds(q, kc, d.page_table, W, SCALE)
    return compare_scores(res.cpu().numpy(), ref, loose, tight)


@pytest.mark.parametrize("ps", [8, 12, 64, 100, 196])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("Q", [1, 4])
def test_decode_dtypes_and_page_sizes(ps, dtype, Q):
    lens = [0, 1, 5, 130, 513, 2049, 4 * 196 * 3 + 6, 5000]
    d = wl.make_decode("ps", lens, Q=Q, page_size=ps, seed=ps + Q, W=max(lens) // 4 + 11)
    _decode(d, d.q.to(dtype), d.k_cache.to(dtype))


def test_decode_page_196_invalid_pages_full_config():
    d = wl.make_decode("ps196", wl.lognormal_contexts(16, 3508, 102400, 819200, seed=0), Q=4, page_size=196,
                       seed=3, table_pad=1)
    t = d.page_table.clone()
    t[0, 2] = -1
    t[1, 5] = d.k_cache.shape[0] + 3
    d.page_table = t
    _decode(d, d.q, d.k_cache)


@pytest.mark.parametrize("ps", [196, 12])
def test_decode_fp8_page_sizes(ps):
    d = wl.make_decode("fp8ps", [3000, 777, 64, 1500], Q=3, page_size=ps, seed=ps)
    codes, ks = wl.e4m3_cache(d.k_cache)
    res = qsa.mqa_decode_fp8(d.q.to(DEV), codes.to(DEV), ks, d.page_table.to(DEV), d.seq_lens.to(DEV), d.W)
    torch.cuda.synchronize()
    ref = oracle.decode_fp8(d.q, codes, ks, d.page_table, d.seq_lens, d.W)
    kdq = codes.view(torch.float8_e4m3fn).to(torch.float64) * ks
    loose, tight = decode_bounds(d.q, kdq, d.page_table, d.W, SCALE)
    compare_scores(res.cpu().numpy(), ref, loose, tight)


@pytest.mark.parametrize("layout", [([64], [128]), ([37, 91, 5], [0, 517, 260]), ([300], [0])])
def test_prefill_f16(layout):
    new, pre = layout
    p = wl.make_prefill("f16", new, pre, seed=sum(new))
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    q, k = p.q.to(torch.float16), p.k.to(torch.float16)
    W = p.W + 5
    res = qsa.mqa_prefill(q.to(DEV), k.to(DEV), torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), W)
    torch.cuda.synchronize()
    ref = oracle.prefill(q, k, ks, ke, W)
    loose, tight = prefill_bounds(q, k, ks, W, SCALE)
    compare_scores(res.cpu().numpy(), ref, loose, tight)
