"""Prefill parity: the CUDA path through the C ABI against the fp64 oracle
(B200 only).  Small cases are compared element by element; the two
full-size workloads on sampled rows, plus properties checked on every
element (mask pattern exact, scores non-negative)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity import compare_scores, prefill_bounds

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
SCALE = 1.0 / np.sqrt(128.0)
DEV = torch.device("cuda")


def intervals(p: wl.PrefillInputs):
    return oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)


def run_full(q, k, ks, ke, W, out=None):
    res = qsa.mqa_prefill(q.to(DEV), k.to(DEV), torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), W,
                          scale=SCALE, out=out)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    gpu = res.cpu().numpy()
    ref = oracle.prefill(q.cpu(), k.cpu(), ks, ke, W, scale=SCALE)
    loose, tight = prefill_bounds(q.cpu(), k.cpu(), ks, W, SCALE)
    return compare_scores(gpu, ref, loose, tight)


def test_intervals_kernel_matches_oracle():
    p = wl.make_prefill("iv", [5, 0, 64, 130, 1, 7], [0, 9, 13, 2000, 3, 1], seed=1)
    ks_o, ke_o = intervals(p)
    ks, ke = qsa.prefill_intervals(p.cu_seqlens_q.to(DEV), p.seq_lens.to(DEV), p.key_offsets.to(DEV), p.T)
    assert np.array_equal(ks.cpu().numpy(), ks_o) and np.array_equal(ke.cpu().numpy(), ke_o)
    for cfg in (4, 5):
        p = wl.make_config(cfg)
        ks_o, ke_o = intervals(p)
        ks, ke = qsa.prefill_intervals(p.cu_seqlens_q.to(DEV), p.seq_lens.to(DEV), p.key_offsets.to(DEV), p.T)
        assert np.array_equal(ks.cpu().numpy(), ks_o) and np.array_equal(ke.cpu().numpy(), ke_o)


@pytest.mark.parametrize("layout", [
    ([64], [128]),                 # one tile each way
    ([100], [1000]),               # ragged rows, partial key tile
    ([37, 91, 5], [0, 517, 260]),  # token tiles straddle sequences
    ([300], [0]),                  # pure causal, rows with no key yet
    ([1], [4]),
    ([200, 200], [2048, 3000]),
])
def test_prefill_small(layout):
    new, pre = layout
    p = wl.make_prefill("small", new, pre, seed=sum(new) + sum(pre))
    ks, ke = intervals(p)
    run_full(p.q, p.k, ks, ke, p.W + 5)


def test_prefill_arbitrary_intervals():
    """Intervals that start below 0, end past Nk, are empty or reversed; W
    cuts some rows short."""
    rng = np.random.default_rng(3)
    T, Nk = 333, 900
    g = torch.Generator().manual_seed(3)
    q = wl.randn_bf16((T, 4, 128), g)
    k = wl.randn_bf16((Nk, 128), g)
    ks = rng.integers(-300, Nk + 50, size=T).astype(np.int32)
    ke = (ks + rng.integers(-50, 700, size=T)).astype(np.int32)
    ks[:4] = [-1000, 0, 5, Nk]
    ke[:4] = [Nk + 1000, 0, 4, Nk + 3]
    run_full(q, k, ks, ke, 512)


def test_prefill_strided_and_no_keys():
    p = wl.make_prefill("strided", [150], [700], seed=5)
    ks, ke = intervals(p)
    qbig = torch.zeros(p.T, 6, 136, dtype=torch.bfloat16)
    qbig[:, :4, :128] = p.q
    q = qbig.to(DEV)[:, :4, :128]
    kbig = torch.zeros(p.Nk, 192, dtype=torch.bfloat16)
    kbig[:, :128] = p.k
    k = kbig.to(DEV)[:, :128]
    out = torch.full((p.T, p.W + 40), 3.0, device=DEV)[:, :p.W + 3]
    run_full(q, k, ks, ke, p.W + 3, out=out)
    # no keys at all: every column is -inf
    res = qsa.mqa_prefill(q, k[:0], torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), 50)
    assert torch.isneginf(res).all()


@pytest.mark.parametrize("cfg", [4, 5])
def test_prefill_full_config_sampled(cfg):
    """Full-size workload in the benchmark's launch configuration: every row's
    mask is checked exactly on the GPU, scores of sampled rows against the
    oracle element by element, and random entries of all other rows."""
    p = wl.make_config(cfg)
    ks, ke = intervals(p)
    out = qsa.mqa_prefill(p.q.to(DEV), p.k.to(DEV), torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), p.W,
                          scale=SCALE)
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    # mask pattern and sign of every element
    lo = torch.from_numpy(np.maximum(ks, 0) - ks).to(DEV)[:, None]
    hi = torch.from_numpy(np.minimum(ke, p.Nk) - ks).to(DEV)[:, None]
    cols = torch.arange(p.W, device=DEV)[None, :]
    want_live = (cols >= lo) & (cols < hi)
    assert torch.equal(torch.isfinite(out), want_live)
    assert torch.equal(torch.isneginf(out), ~want_live)
    assert bool((out[want_live] >= 0).all())
    # sampled rows in full
    rng = np.random.default_rng(cfg)
    T = p.T
    rows = np.unique(np.concatenate([[0, 1, 63, 64, T - 1, T - 64], rng.integers(0, T, size=24),
                                     p.cu_seqlens_q.numpy()[1:-1], p.cu_seqlens_q.numpy()[1:-1] - 1]))
    rows = rows[(rows >= 0) & (rows < T)]
    tt = np.repeat(rows, p.W)
    jj = np.tile(np.arange(p.W), len(rows))
    ref = oracle.prefill_entries(p.q, p.k, ks, ke, tt, jj, scale=SCALE).reshape(len(rows), p.W)
    gpu = out[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    loose, tight = prefill_bounds(p.q, p.k, ks, p.W, SCALE, rows=rows)
    compare_scores(gpu, ref, loose, tight)
    # random entries everywhere
    tt = rng.integers(0, T, size=20000)
    jj = rng.integers(0, p.W, size=20000)
    ref = oracle.prefill_entries(p.q, p.k, ks, ke, tt, jj, scale=SCALE)
    gpu = out[torch.from_numpy(tt).to(DEV), torch.from_numpy(jj).to(DEV)].cpu().numpy()
    live = np.isfinite(ref)
    assert np.array_equal(np.isfinite(gpu), live)
    qn = np.linalg.norm(p.q[torch.from_numpy(tt)].double().numpy(), axis=-1).sum(-1)
    kn = np.linalg.norm(p.k.double().numpy(), axis=-1)
    n = np.clip(ks[tt].astype(np.int64) + jj, 0, p.Nk - 1)
    tol = 4e-3 * SCALE * qn * kn[n] + 1e-6
    assert np.all(np.abs(gpu[live] - ref[live]) <= tol[live])


def test_prefill_repeat_is_bitwise_stable():
    p = wl.make_prefill("rep", [1000], [5000], seed=6)
    ks, ke = intervals(p)
    args = (p.q.to(DEV), p.k.to(DEV), torch.from_numpy(ks).to(DEV), torch.from_numpy(ke).to(DEV), p.W)
    assert torch.equal(qsa.mqa_prefill(*args), qsa.mqa_prefill(*args))
