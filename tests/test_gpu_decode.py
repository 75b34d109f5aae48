"""Decode / spec-decode parity: the CUDA path through the C ABI against the
fp64 oracle, element by element (B200 only)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import compare_scores, decode_bounds

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
SCALE = 1.0 / np.sqrt(128.0)
DEV = torch.device("cuda")


def run_case(d: wl.DecodeInputs, q=None, k_cache=None, out=None, W=None):
    W = d.W if W is None else W
    q = d.q if q is None else q
    k_cache = d.k_cache if k_cache is None else k_cache
    dev = torch.device("cuda")
    res = qsa.mqa_decode(q.to(dev) if q.device.type == "cpu" else q, k_cache.to(dev) if k_cache.device.type == "cpu" else k_cache,
                         d.page_table.to(dev), d.seq_lens.to(dev), W, scale=SCALE, out=out)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    gpu = res.cpu().numpy()
    ref = oracle.decode(q.cpu(), k_cache.cpu(), d.page_table, d.seq_lens, W, scale=SCALE)
    loose, tight = decode_bounds(q.cpu(), k_cache.cpu(), d.page_table, W, SCALE)
    return compare_scores(gpu, ref, loose, tight)


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_decode_full_config(cfg):
    """The three decode workloads at full size, every output element."""
    st = run_case(wl.make_config(cfg))
    assert st["entries"] > 0


@pytest.mark.parametrize("ps", [8, 16, 32, 64])
@pytest.mark.parametrize("Q", [1, 2, 3, 4])
def test_decode_ragged(ps, Q):
    """Ragged lengths: empty, shorter than Q, not multiples of 4, spanning
    several units and a partial last unit; W larger than every row needs."""
    lens = [0, 1, 3, 4, 5, 7, 130, 511, 512, 513, 2049, 4 * 128 * 3 + 6]
    d = wl.make_decode("ragged", lens, Q=Q, page_size=ps, seed=ps * 10 + Q, W=max(lens) // 4 + 37)
    run_case(d)


def test_decode_invalid_pages_and_short_table():
    lens = [900, 1400, 333, 2000]
    d = wl.make_decode("bad_pages", lens, Q=4, page_size=16, seed=7, table_pad=2)
    t = d.page_table.clone()
    P = d.k_cache.shape[0]
    t[0, 1] = -1
    t[1, 3] = P + 4            # past the pool
    t[2, 0] = -7
    t[3, 5:] = -1              # table ends early
    d.page_table = t
    run_case(d)
    # a table with fewer columns than the visible keys need
    d2 = wl.make_decode("short_table", [3000], Q=1, page_size=64, seed=8)
    d2.page_table = d2.page_table[:, :5].contiguous()
    run_case(d2)


def test_decode_w_smaller_than_visible():
    d = wl.make_decode("narrow", [5000, 60, 1200], Q=2, page_size=32, seed=9)
    run_case(d, W=300)


def test_decode_strided_views():
    """Non-contiguous q / k_cache / out views that still meet the layout rules."""
    d = wl.make_decode("strided", [777, 1500, 64], Q=3, page_size=32, seed=11)
    dev = torch.device("cuda")
    B, Q = d.B, d.Q
    qbig = torch.zeros(B, Q + 1, 5, 136, dtype=torch.bfloat16)
    qbig[:, :Q, :4, :128] = d.q
    q = qbig.to(dev)[:, :Q, :4, :128]
    P, ps = d.k_cache.shape[:2]
    kbig = torch.zeros(P, ps + 3, 1, 144, dtype=torch.bfloat16)
    kbig[:, :ps, :, :128] = d.k_cache
    kc = kbig.to(dev)[:, :ps, :, :128]
    out = torch.full((B, Q, d.W + 9), 7.0, device=dev)[:, :, :d.W]
    run_case(d, q=q, k_cache=kc, out=out)


@pytest.mark.parametrize("axis", ["b", "t", "h"])
def test_decode_broadcast_query(axis):
    """Stride-0 query axes (decode accepts broadcast queries)."""
    d = wl.make_decode("bcast", [600, 1234, 99], Q=3, page_size=16, seed=12)
    dev = torch.device("cuda")
    base = d.q.to(dev)
    if axis == "b":
        q = base[:1].expand(d.B, -1, -1, -1)
    elif axis == "t":
        q = base[:, :1].expand(-1, d.Q, -1, -1)
    else:
        q = base[:, :, :1].expand(-1, -1, 4, -1)
    run_case(d, q=q)


def test_decode_repeat_is_bitwise_stable():
    d = wl.make_config(2)
    dev = torch.device("cuda")
    args = (d.q.to(dev), d.k_cache.to(dev), d.page_table.to(dev), d.seq_lens.to(dev), d.W)
    a = qsa.mqa_decode(*args).cpu()
    b = qsa.mqa_decode(*args).cpu()
    assert torch.equal(a, b)


def test_decode_zero_queries_give_zero():
    d = wl.make_decode("zero", [800, 333], Q=4, page_size=64, seed=13)
    d.q = torch.zeros_like(d.q)
    run_case(d)


# ---------------------------------------------------------------- fp8 E4M3 key cache

def run_case_fp8(d: wl.DecodeInputs, codes=None, k_scale=None, q=None, W=None, kc_dev=None, out=None):
    """The fp8 entry against the oracle's fp8 entry; the tolerance is the bf16
    one on the dequantised keys (torch's E4M3 decoding times k_scale)."""
    W = d.W if W is None else W
    q = d.q if q is None else q
    if codes is None:
        codes, k_scale = wl.e4m3_cache(d.k_cache, k_scale)
    dev = torch.device("cuda", 0)
    res = qsa.mqa_decode_fp8(q.to(dev) if q.device.type == "cpu" else q,
                             codes.to(dev) if kc_dev is None else kc_dev, k_scale,
                             d.page_table.to(dev), d.seq_lens.to(dev), W, scale=SCALE, out=out)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    gpu = res.cpu().numpy()
    ref = oracle.decode_fp8(q.cpu(), codes, k_scale, d.page_table, d.seq_lens, W, scale=SCALE)
    kdq = codes.view(torch.float8_e4m3fn).to(torch.float64) * k_scale
    loose, tight = decode_bounds(q.cpu(), kdq, d.page_table, W, SCALE)
    return compare_scores(gpu, ref, loose, tight)


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_decode_fp8_full_config(cfg):
    """The three decode workloads at full size with the fp8 cache, every element."""
    st = run_case_fp8(wl.make_config(cfg))
    assert st["entries"] > 0


@pytest.mark.parametrize("ps", [8, 16, 32, 64])
@pytest.mark.parametrize("Q", [1, 2, 3, 4])
def test_decode_fp8_ragged(ps, Q):
    lens = [0, 1, 3, 4, 5, 7, 130, 511, 512, 513, 2049, 4 * 128 * 3 + 6]
    d = wl.make_decode("ragged", lens, Q=Q, page_size=ps, seed=ps * 10 + Q + 500, W=max(lens) // 4 + 37)
    run_case_fp8(d)


def test_decode_fp8_invalid_pages_and_narrow_w():
    d = wl.make_decode("bad_pages", [900, 1400, 333, 2000], Q=4, page_size=16, seed=17, table_pad=2)
    t = d.page_table.clone()
    P = d.k_cache.shape[0]
    t[0, 1] = -1
    t[1, 3] = P + 4
    t[2, 0] = -7
    t[3, 5:] = -1
    d.page_table = t
    run_case_fp8(d)
    run_case_fp8(d, W=100)


@pytest.mark.parametrize("k_scale", [2.0 ** -7, 0.0173, 1.0, 3.5])
def test_decode_fp8_every_code(k_scale):
    """Uniformly random finite codes: subnormals, both zeros and +-448 all occur."""
    d = wl.make_decode("codes", [3000, 777, 64, 1500], Q=3, page_size=32, seed=19)
    g = torch.Generator().manual_seed(20)
    codes = torch.randint(0, 256, d.k_cache.shape, generator=g, dtype=torch.int32)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0x7E
    codes = codes.to(torch.uint8)
    run_case_fp8(d, codes=codes, k_scale=k_scale)


def test_decode_fp8_query_dynamic_range():
    """Query rows far outside fp16's range, tiny rows, zero rows and rows that
    mix magnitudes 2^20 apart (the kernel scales each row by a power of two)."""
    d = wl.make_decode("qrange", [2000, 1000, 600, 3000], Q=4, page_size=64, seed=21)
    q = d.q.float()
    q[0, :, 0] *= 2.0 ** 40
    q[0, :, 1] *= 2.0 ** -40
    q[1, 0] = 0.0
    q[1, 1, 2] = 0.0
    q[2, :, 0, :64] *= 2.0 ** 10
    q[2, :, 0, 64:] *= 2.0 ** -10
    q[3, :, :, 5] = 60000.0
    q[3, 2] *= 2.0 ** -100
    run_case_fp8(d, q=q.to(torch.bfloat16))


def test_decode_fp8_strided_views():
    """A cache view with 144-byte rows and padded pages, and a padded out."""
    d = wl.make_decode("strided", [777, 1500, 64], Q=3, page_size=32, seed=23)
    codes, ks = wl.e4m3_cache(d.k_cache)
    P, ps = codes.shape[:2]
    big = torch.zeros(P, ps + 2, 1, 144, dtype=torch.uint8)
    big[:, :ps, :, :128] = codes
    dev = torch.device("cuda", 0)
    kc = big.to(dev)[:, :ps, :, :128]
    out = torch.full((d.B, d.Q, d.W + 9), 7.0, device=dev)[:, :, :d.W]
    run_case_fp8(d, codes=codes, k_scale=ks, kc_dev=kc, out=out)


def test_decode_fp8_agrees_with_bf16_kernel_on_exact_keys():
    """With a power-of-two k_scale the dequantised keys are exact in bf16; the
    fp8 kernel's scores then match the bf16 kernel's within fp32 rounding."""
    d = wl.make_config(2)
    codes, _ = wl.e4m3_cache(d.k_cache)
    ks = 2.0 ** -6
    kbf = (codes.view(torch.float8_e4m3fn).to(torch.float32) * ks).to(torch.bfloat16)
    dev = torch.device("cuda", 0)
    a = qsa.mqa_decode_fp8(d.q.to(dev), codes.to(dev), ks, d.page_table.to(dev), d.seq_lens.to(dev), d.W)
    b = qsa.mqa_decode(d.q.to(dev), kbf.to(dev), d.page_table.to(dev), d.seq_lens.to(dev), d.W)
    a, b = a.cpu().numpy(), b.cpu().numpy()
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    live = np.isfinite(b)
    assert np.allclose(a[live], b[live], rtol=1e-5, atol=1e-5)


# ---------------------------------------------------------------- many requests

def _many(B, Q, ps, seed, max_len=400):
    g = np.random.default_rng(seed)
    lens = g.integers(0, max_len + 1, size=B).tolist()
    lens[0] = max_len                       # the widest row sets W
    return wl.make_decode(f"many{B}", lens, Q=Q, page_size=ps, seed=seed)


@pytest.mark.parametrize("B,Q,ps", [
    (100, 2, 16),     # block-wide prefix scan, one chunk per warp over several 32-request groups
    (1184, 1, 8),     # the largest batch with two warps per request
    (1500, 3, 32),    # block-wide scan, warps take contiguous tile ranges across requests
    (8200, 2, 8),     # more requests than one launch takes (two launches)
])
def test_decode_many_requests(B, Q, ps):
    run_case(_many(B, Q, ps, seed=B + Q))


def test_decode_fp8_many_requests():
    run_case_fp8(_many(1500, 4, 16, seed=99))


def test_decode_many_short_requests():
    """2000 requests of at most 60 tokens: every warp gets at most one
    half-batch, so the bf16 launch takes the two-half-batch loop, and warps
    cross from one request to the next (more than half as many requests as
    warps)."""
    run_case(_many(2000, 2, 8, seed=2002, max_len=60))


# ---------------------------------------------------------------- large pages, dense and padded rows

@pytest.mark.parametrize("ps", [32, 64, 128, 1024])
@pytest.mark.parametrize("Q", [1, 4])
def test_decode_large_pages_and_masks(ps, Q):
    lens = [1, 4, 129, 8 * ps + 5, 3000, 20000, 4 * ps * 3]
    d = wl.make_decode("bulk", lens, Q=Q, page_size=ps, seed=ps + Q, table_pad=1, W=max(lens) // 4 - 100)
    t = d.page_table.clone()
    t[4, 1] = -1                                   # a missing page
    t[5, 2] = d.k_cache.shape[0] + 9               # a page outside the pool
    d.page_table = t
    run_case(d)


@pytest.mark.parametrize("B", [1, 17, 32])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_decode_dense_and_padded_rows_agree(B, dtype):
    """The same keys in dense rows and in rows padded to 136 elements give
    bitwise the same scores (the row stride only moves the loads)."""
    lens = torch.randint(1, 12000, (B,), generator=torch.Generator().manual_seed(B)).tolist()
    d = wl.make_decode("dense_vs_padded", lens, Q=3, page_size=64, seed=B)
    q, kc = d.q.to(dtype).to(DEV), d.k_cache.to(dtype).to(DEV)
    padded = torch.zeros(kc.shape[0], kc.shape[1], 1, 136, dtype=dtype, device=DEV)
    padded[..., :128] = kc
    pt, sl = d.page_table.to(DEV), d.seq_lens.to(DEV)
    dense = qsa.mqa_decode(q, kc, pt, sl, d.W)
    regs = qsa.mqa_decode(q, padded[..., :128], pt, sl, d.W)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    assert torch.equal(torch.isneginf(dense), torch.isneginf(regs))
    assert torch.equal(dense, regs)
