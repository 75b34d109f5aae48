"""Top-k parity (B200 only): on identical fp32 score rows the GPU selection
must equal the oracle's exactly (index work is bit-exact); after the fused
prefill the index sets may differ only by swaps tied within the score
tolerance of the k-th value."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import prefill_bounds, topk_sets_agree

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
SCALE = 1.0 / np.sqrt(128.0)
DEV = torch.device("cuda")


def gpu_topk(scores: np.ndarray, k: int, lengths=None, ws: bool = False):
    """qsa_topk, or with ws the workspace path (filter pass, list selection,
    exact pass) over the same rows."""
    s = torch.from_numpy(scores.astype(np.float32)).to(DEV)
    ln = None if lengths is None else torch.from_numpy(lengths.astype(np.int32)).to(DEV)
    workspace = None
    if ws:
        n = qsa.topk_workspace_size(s.shape[0], s.shape[1], k)
        workspace = torch.full((n,), 0x5A, dtype=torch.uint8, device=DEV)   # stale contents must not matter
    idx = qsa.topk(s, k, lengths=ln, workspace=workspace)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    return idx.cpu().numpy()


def ora_topk(scores: np.ndarray, k: int, lengths=None):
    s32 = scores.astype(np.float32).astype(np.float64)
    ln = np.full(s32.shape[0], s32.shape[1], dtype=np.int32) if lengths is None else lengths
    return oracle.topk(s32, np.minimum(np.maximum(ln, 0), s32.shape[1]), k)


@pytest.mark.parametrize("ws", [False, True])
@pytest.mark.parametrize("k", [1, 7, 512, 2048])
@pytest.mark.parametrize("W", [100, 5000, 26624])
def test_topk_random_rows(k, W, ws):
    rng = np.random.default_rng(k * 7 + W)
    rows = 64
    s = np.abs(rng.normal(size=(rows, W))) * 3
    s[rng.random(size=s.shape) < 0.03] = -np.inf
    lengths = rng.integers(-5, W + 10, size=rows).astype(np.int32)
    assert np.array_equal(gpu_topk(s, k, lengths, ws), ora_topk(s, k, lengths))
    assert np.array_equal(gpu_topk(s, k, ws=ws), ora_topk(s, k))


@pytest.mark.parametrize("ws", [False, True])
@pytest.mark.parametrize("W,k,rows", [(2048, 256, 9000), (26624, 512, 2400)])
def test_topk_predictions_across_rows(W, k, rows, ws):
    """Enough rows that each selecting warp takes several in turn, so the
    threshold predicted from one row meets the next: rows whose scale drops
    (the prediction admits fewer than k), jumps (the candidate list
    overflows), rows of heavy ties, rows whose boundary lies among zero
    scores, constant rows and rows shorter than k.  The selection must not
    depend on the prediction: it equals the oracle's exactly."""
    rng = np.random.default_rng(W + k)
    s = np.abs(rng.normal(size=(rows, W))).astype(np.float32) * 3
    r = np.arange(rows)
    s[r % 7 == 3] *= np.float32(0.3)
    s[r % 11 == 5] *= np.float32(5.0)
    tie_rows = r % 13 == 0
    s[tie_rows] = np.round(s[tie_rows] * 2) / 2
    few = r % 17 == 1
    s[few] = np.where(rng.random(size=(int(few.sum()), W)) < 0.95, 0.0, s[few])
    s[r % 19 == 2] = 2.5
    s[rng.random(size=s.shape) < 0.01] = -np.inf
    lengths = np.full(rows, W, dtype=np.int32)
    short = r % 23 == 4
    lengths[short] = rng.integers(0, k + 5, size=int(short.sum()))
    assert np.array_equal(gpu_topk(s, k, lengths, ws), ora_topk(s, k, lengths))


@pytest.mark.parametrize("ws", [False, True])
def test_topk_ties_signed_zero_negative_and_nan(ws):
    rng = np.random.default_rng(1)
    W, k = 3000, 300
    s = np.round(rng.normal(size=(40, W)), 1)          # heavy ties
    s[0] = 1.0                                          # all equal
    s[1] = 0.0
    s[1, ::2] = -0.0                                    # signed zeros tie
    s[2] = -np.abs(s[2])                                # negative values
    s[3, :] = -np.inf
    s[3, 17] = 5.0                                      # a single candidate
    s[4, rng.random(W) < 0.5] = np.nan                  # NaN never selected
    s[5, :] = np.float32(3.4e38)
    want = ora_topk(np.where(np.isnan(s), -np.inf, s), k)
    assert np.array_equal(gpu_topk(s, k, ws=ws), want)


def test_topk_uncached_wide_rows_and_odd_stride():
    rng = np.random.default_rng(2)
    s = rng.normal(size=(6, 60000))                     # wider than the shared-memory row cache
    assert np.array_equal(gpu_topk(s, 512), ora_topk(s, 512))
    s = np.abs(rng.normal(size=(1500, 65536))).astype(np.float32)   # the widest rows, many per CTA
    assert np.array_equal(gpu_topk(s, 512, ws=True), ora_topk(s, 512))
    # rows that are not 16-byte aligned: scalar loads
    base = torch.from_numpy(rng.normal(size=(20, 1001)).astype(np.float32)).to(DEV)
    view = base[:, 1:]
    idx = qsa.topk(view, 64).cpu().numpy()
    assert np.array_equal(idx, ora_topk(view.cpu().numpy(), 64))


def test_fused_prefill_topk_matches_separate_calls():
    p = wl.make_prefill("fused", [300, 200], [4000, 9000], seed=4)
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    q, k = p.q.to(DEV), p.k.to(DEV)
    ks_d, ke_d = torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV)
    scores = qsa.mqa_prefill(q, k, ks_d, ke_d, p.W)
    want = qsa.topk(scores, 512)
    for rows_in_ws in (p.T, 64, 128, 200):
        ws = torch.empty(qsa.prefill_topk_workspace_size(rows_in_ws, p.W) // 4 + 1, dtype=torch.float32, device=DEV)
        got = qsa.mqa_prefill_topk(q, k, ks_d, ke_d, p.W, 512, ws)
        assert torch.equal(got, want), rows_in_ws
    torch.cuda.synchronize()
    assert qsa.device_error() == 0


def test_fused_prefill_topk_full_config_sampled():
    """The 4 x 4096-row, 102,400-token-prefix workload with top-512: sampled
    rows against the oracle's selection over its fp64 scores."""
    p = wl.make_config(5)
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    ws = torch.empty(qsa.prefill_topk_workspace_size(p.T, p.W) // 4, dtype=torch.float32, device=DEV)
    idx = qsa.mqa_prefill_topk(p.q.to(DEV), p.k.to(DEV), torch.from_numpy(ks).to(DEV),
                               torch.from_numpy(ke).to(DEV), p.W, wl.TOPK_K, ws)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    idx = idx.cpu().numpy()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 4095, 4096, p.T - 1], rng.integers(0, p.T, size=11)]))
    tt = np.repeat(rows, p.W)
    jj = np.tile(np.arange(p.W), len(rows))
    ref = oracle.prefill_entries(p.q, p.k, ks, ke, tt, jj, scale=SCALE).reshape(len(rows), p.W)
    ora_idx = oracle.topk(ref, np.full(len(rows), p.W, dtype=np.int32), wl.TOPK_K)
    loose, _ = prefill_bounds(p.q, p.k, ks, p.W, SCALE, rows=rows)
    for i, r in enumerate(rows):
        topk_sets_agree(idx[r], ora_idx[i], ref[i], loose[i], wl.TOPK_K)


def _fused_vs_separate(p, q, k, k_top=512):
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    ks_d, ke_d = torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV)
    q, k = q.to(DEV), k.to(DEV)
    want = qsa.topk(qsa.mqa_prefill(q, k, ks_d, ke_d, p.W), k_top)
    ws = torch.empty(qsa.prefill_topk_workspace_size(p.T, p.W) // 4 + 1, dtype=torch.float32, device=DEV)
    got = qsa.mqa_prefill_topk(q, k, ks_d, ke_d, p.W, k_top, ws)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    assert torch.equal(got, want)


@pytest.mark.parametrize("sampled_high", [True, False])
def test_fused_prefill_topk_ties_and_skew(sampled_high):
    """Every 16th key scores far above all others (about 190 equal scores
    inside the top 512 of a row) or exactly zero (a block of ties at the
    bottom): the fused entry must still equal top-k over the separate scores,
    ties resolved to the lower column."""
    p = wl.make_prefill("fused_fallback", [96, 70], [12000, 9000], seed=6)
    q = torch.zeros_like(p.q)
    q[:, :, 0] = 1.0
    k = torch.randn(p.k.shape, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16) * 0.1
    k[:, 0] = k[:, 0].abs() + 0.5
    sampled = torch.arange(p.Nk) % 16 == 0
    k[sampled, 0] = 8.0 if sampled_high else 0.0
    k[sampled, 1:] = 0.0
    _fused_vs_separate(p, q, k)


def test_topk_workspace_path_matches_streaming_path_at_full_size():
    """The 4 x 4,096-row, 102,400-token-prefix workload's 16,384 score rows
    (26,624 columns each, from the prefill kernel): the workspace path and
    qsa_topk select exactly the same columns (both are exact selections of
    the same fp32 rows, and every row of the sampled full-parity test checks
    qsa_topk against the oracle)."""
    p = wl.make_config(5)
    ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
    scores = qsa.mqa_prefill(p.q.to(DEV), p.k.to(DEV), torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), p.W)
    want = qsa.topk(scores, wl.TOPK_K)
    ws = torch.empty(qsa.topk_workspace_size(p.T, p.W, wl.TOPK_K), dtype=torch.uint8, device=DEV)
    got = qsa.topk(scores, wl.TOPK_K, workspace=ws)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    assert torch.equal(got, want)
    # a second call over the same workspace (stale lists from the first)
    got2 = qsa.topk(scores, wl.TOPK_K, workspace=ws)
    assert torch.equal(got2, want)
