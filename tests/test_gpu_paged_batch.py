"""Mixed decode + prefill batches from the paged cache in one call (B200
only), against the fp64 oracle.

Every row of request r is scored as the oracle's paged decode of that
request with all of its query rows (the decode oracle takes any number of
rows per request; its pins include runs longer than 4), so decode rows and
prefill rows are checked by the same definition: request-local key columns,
the causal visible count of each row, -inf for keys in missing pages."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import compare_scores, decode_bounds

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
DEV = torch.device("cuda")
SCALE = 1.0 / np.sqrt(128.0)


def run_and_check(b: wl.PagedBatchInputs, page_table=None, out=None, twice=False):
    pt = b.page_table if page_table is None else page_table
    args = (b.q.to(DEV), b.k_cache.to(DEV), pt.to(DEV), b.cu_seqlens_q.to(DEV), b.seq_lens.to(DEV),
            b.num_decodes, b.decode_query_len, b.W)
    got = qsa.mqa_paged_batch(*args, scale=SCALE, out=out)
    if twice:
        first = got.clone()
        got = qsa.mqa_paged_batch(*args, scale=SCALE, out=got)
        assert torch.equal(first, got)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    got = got.cpu().numpy()
    cu = b.cu_seqlens_q.numpy()
    for r in range(len(b.seq_lens)):
        rows = slice(int(cu[r]), int(cu[r + 1]))
        n = int(cu[r + 1] - cu[r])
        if n == 0:
            continue
        q = b.q[rows].reshape(1, n, 4, 128)
        ref = oracle.decode(q, b.k_cache, pt[r:r + 1], b.seq_lens[r:r + 1], b.W, scale=SCALE)
        loose, tight = decode_bounds(q, b.k_cache, pt[r:r + 1], b.W, SCALE)
        compare_scores(got[rows].reshape(1, n, b.W), ref, loose, tight)


@pytest.mark.parametrize("ps", [16, 64, 196])
def test_mixed_batch(ps):
    b = wl.make_paged_batch("mixed", [517, 2048, 61, 9000, 3], 2, [100, 7, 300], [3000, 0, 1290], ps, seed=ps)
    run_and_check(b, twice=True)


def test_mixed_batch_missing_pages_and_narrow_width():
    b = wl.make_paged_batch("mixed_bad", [700, 5000], 4, [260, 1000], [800, 6000], 16, seed=4, W=1500)
    pt = b.page_table.clone()
    pt[0, 3] = -1                                  # a decode request's page
    pt[2, 1] = -1                                  # prefill request pages: missing and out of the pool
    pt[3, 10] = b.k_cache.shape[0] + 2
    pt[3, 0] = -1
    pt[3, 40] = -1                                 # pages past the first 32 (another lane group)
    pt[3, 93] = -1                                 # the last, partly used page of the 1,500 keys
    run_and_check(b, page_table=pt)


def test_decode_only_and_prefill_only():
    b = wl.make_paged_batch("dec_only", [100, 4096, 33], 3, [], [], 64, seed=1)
    run_and_check(b)
    b = wl.make_paged_batch("pre_only", [], 1, [128, 1, 513], [64, 5000, 0], 64, seed=2)
    run_and_check(b)


def test_strided_output_rows():
    b = wl.make_paged_batch("strided", [300, 301], 1, [90], [400], 32, seed=3)
    big = torch.full((b.T, b.W + 24), 7.0, device=DEV)
    run_and_check(b, out=big[:, :b.W])
    assert bool((big[:, b.W:] == 7.0).all())       # nothing written past W
