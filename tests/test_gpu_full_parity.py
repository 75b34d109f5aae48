"""Every element of the two full-size prefill workloads against the fp64
oracle (B200 only), in the launch configuration the benchmark times.

The 8,192-row workload (50,144-token prefix, 14,584 keys) and the 4 x 4,096-
row workload (102,400-token prefixes, 4 x 26,624 keys, top-512) are scored by
qsa_mqa_prefill once; the oracle then scores the same rows chunk by chunk on
the host cores and every score is compared (mask exact, value within the
stated tolerance and the fp32 rounding bound).  For the top-512 workload the
GPU selection over the GPU scores must agree with the oracle's selection over
its fp64 scores on every row, up to swaps tied within tolerance of the k-th
value.  Also here: a batch of more rows than one prefill launch covers, which
takes the multi-launch path (query rows addressed from a non-zero first row).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import compare_scores, prefill_bounds, topk_sets_agree

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
SCALE = 1.0 / np.sqrt(128.0)
DEV = torch.device("cuda")
CHUNK = 1024


@pytest.mark.parametrize("cfg", [4, 5])
def test_prefill_full_config_every_element(cfg):
    p = wl.make_config(cfg)
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    ks_d, ke_d = torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV)
    out = qsa.mqa_prefill(p.q.to(DEV), p.k.to(DEV), ks_d, ke_d, p.W, scale=SCALE)
    idx = qsa.topk(out, wl.TOPK_K).cpu().numpy() if cfg == 5 else None
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    worst = 0.0
    swaps = 0
    for r0 in range(0, p.T, CHUNK):
        rows = np.arange(r0, min(r0 + CHUNK, p.T))
        ref = oracle.prefill(p.q[r0:r0 + len(rows)], p.k, ks[rows], ke[rows], p.W, scale=SCALE)
        loose, tight = prefill_bounds(p.q, p.k, ks, p.W, SCALE, rows=rows)
        stats = compare_scores(out[r0:r0 + len(rows)].cpu().numpy(), ref, loose, tight)
        worst = max(worst, stats["frac_of_tol"])
        if idx is not None:
            ora_idx = oracle.topk(ref, np.full(len(rows), p.W, dtype=np.int32), wl.TOPK_K)
            for i, r in enumerate(rows):
                swaps += topk_sets_agree(idx[r], ora_idx[i], ref[i], loose[i], wl.TOPK_K)
    assert worst <= 1.0
    if idx is not None:
        # ties within tolerance are rare with N(0, 1) data
        assert swaps <= p.T // 100, swaps


def test_prefill_more_rows_than_one_launch():
    """132,100 rows (two launches of at most 131,072 rows; the second reads
    its queries from row 131,072 on) against 200 keys with arbitrary
    intervals, W = 48: every element against the oracle."""
    T, Nk, W = 131072 + 1028, 200, 48
    g = torch.Generator().manual_seed(17)
    q = wl.randn_bf16((T, 4, 128), g)
    k = wl.randn_bf16((Nk, 128), g)
    rng = np.random.default_rng(17)
    ks = rng.integers(-20, Nk, size=T).astype(np.int32)
    ke = (ks + rng.integers(-5, 60, size=T)).astype(np.int32)
    ks[131071:131075] = [0, 3, -7, Nk - 2]
    ke[131071:131075] = [Nk, 50, 30, Nk + 9]
    out = qsa.mqa_prefill(q.to(DEV), k.to(DEV), torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), W,
                          scale=SCALE)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    ref = oracle.prefill(q, k, ks, ke, W, scale=SCALE)
    loose, tight = prefill_bounds(q, k, ks, W, SCALE)
    compare_scores(out.cpu().numpy(), ref, loose, tight)
