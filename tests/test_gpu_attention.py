"""Core attention after the indexer (B200 only): block-to-token expansion and
sparse attention through the C ABI against the fp64 oracle.

Expansion is index work and must match exactly.  Attention outputs are bf16
and are compared within a bound derived from the kernel's arithmetic: scores
accumulate 256 bf16 products in fp32 (error at most
ds = 2^-16 * scale * max_j sum_d |q_d k_jd| per row, with headroom), the
probabilities are rounded to bf16 before the PV product (2^-9 relative) and
the output is rounded to bf16 (2^-9 relative), so per element
    |d out| <= (2^-8 + 4 ds) * sum_j p_j |v_jd| + 2^-8 |out| + 1e-6
and |d lse| <= 2 ds + 4e-6 (|lse| + 1).  A second family of cases makes every
score exactly 0 (zero keys) with small-integer values, where the output is
the exact mean of the visible values up to the final bf16 rounding: a token
that is wrongly kept or dropped shows there.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_block_qsa_b200")
DEV = torch.device("cuda")
SCALE = 1.0 / 16.0      # 1 / sqrt(256)


def rows_of(a: wl.AttentionInputs):
    """(request, logical position, request length) of every query row."""
    cu = a.cu_seqlens_q.numpy()
    sl = a.seq_lens.numpy()
    req, pos, length = [], [], []
    for r in range(len(sl)):
        qlen = int(cu[r + 1] - cu[r])
        for i in range(qlen):
            req.append(r)
            pos.append(oracle.logical_position(int(sl[r]), qlen, i))
            length.append(int(sl[r]))
    return np.array(req), np.array(pos), np.array(length)


def gpu_expand(a):
    tok = qsa.expand_block_indices(a.blocks.to(DEV), a.cu_seqlens_q.to(DEV), a.seq_lens.to(DEV))
    torch.cuda.synchronize()
    return tok.cpu()


def gpu_attention(a, tok, gate=None, k_cache=None, v_cache=None, page_table=None):
    kc = a.k_cache if k_cache is None else k_cache
    vc = a.v_cache if v_cache is None else v_cache
    pt = a.page_table if page_table is None else page_table
    out, lse = qsa.sparse_attention(a.q.to(DEV), kc.to(DEV), vc.to(DEV), pt.to(DEV), a.cu_seqlens_q.to(DEV),
                                    a.seq_lens.to(DEV), torch.as_tensor(tok).to(DEV), SCALE,
                                    gate=None if gate is None else gate.to(DEV))
    torch.cuda.synchronize()
    assert qsa.device_error() == 0
    return out.cpu().double().numpy(), lse.cpu().double().numpy()


def bounds(a, tok, ref_out, kc, vc, pt):
    """(out tolerance [T, Hq, 256], lse tolerance [T, Hq]) of the module docstring."""
    req, pos, length = rows_of(a)
    q = a.q.double().numpy()
    K = kc.double().numpy()
    V = vc.double().numpy()
    table = pt.numpy()
    T, Hq = q.shape[:2]
    Hkv = K.shape[2]
    ps = K.shape[1]
    tol = np.zeros((T, Hq, 256))
    ltol = np.zeros((T, Hq))
    for t in range(T):
        js = [int(j) for j in tok[t] if 0 <= j <= pos[t] and j < length[t]]
        rows = []
        for j in js:
            lp = j // ps
            page = int(table[req[t], lp]) if lp < table.shape[1] else -1
            if 0 <= page < K.shape[0]:
                rows.append((page, j % ps))
        if not rows:
            continue
        pg = np.array([r[0] for r in rows])
        rw = np.array([r[1] for r in rows])
        for h in range(Hq):
            g = h // (Hq // Hkv)
            k = K[pg, rw, g]                       # [n, 256]
            v = V[pg, rw, g]
            s = SCALE * (k @ q[t, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            ds = 2.0 ** -16 * SCALE * float(np.max(np.abs(k) @ np.abs(q[t, h])))
            tol[t, h] = (2.0 ** -8 + 4 * ds) * (p @ np.abs(v)) + 2.0 ** -8 * np.abs(ref_out[t, h]) + 1e-6
            ltol[t, h] = 2 * ds + 4e-6 * (abs(np.log(np.exp(s - s.max()).sum()) + s.max()) + 1)
    return tol, ltol


def check_attention(a, tok, gate=None, kc=None, vc=None, pt=None):
    kc = a.k_cache if kc is None else kc
    vc = a.v_cache if vc is None else vc
    pt = a.page_table if pt is None else pt
    req, pos, length = rows_of(a)
    out, lse = gpu_attention(a, tok, gate, kc, vc, pt)
    ref, ref_lse = oracle.sparse_attention(a.q, kc, vc, pt, req, pos, a.seq_lens, tok, scale=SCALE,
                                           gate=None if gate is None else gate.double().numpy())
    tol, ltol = bounds(a, np.asarray(tok), ref, kc, vc, pt)
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), empty), "rows with nothing visible differ"
    assert np.all(out[empty] == 0)
    err = np.abs(out - ref)
    worst = float(np.max(err / tol))
    assert worst <= 1.0, f"output error {worst:.3g}x the bound"
    live = ~empty
    lerr = np.abs(lse[live] - ref_lse[live])
    assert np.all(lerr <= ltol[live]), f"lse error {float(np.max(lerr / ltol[live])):.3g}x the bound"
    return worst


@pytest.mark.parametrize("k", [1, 7, 64, 512])
def test_expand_matches_oracle(k):
    a = wl.make_attention("expand", [3, 130, 4101, 70000], [1, 4, 3, 2], 4, 1, 16, k, seed=k)
    blocks = a.blocks.clone()
    blocks[1, 0] = -1                              # padding in the middle of a row
    blocks[2, -1] = -5
    a.blocks = blocks
    req, pos, length = rows_of(a)
    want = oracle.expand_indices(blocks.numpy(), pos, length)
    got = gpu_expand(a).numpy()
    assert np.array_equal(got, want)


@pytest.mark.parametrize("Hq,Hkv,ps", [(24, 2, 16), (24, 2, 64), (4, 1, 196), (16, 1, 32), (8, 4, 8)])
def test_attention_matches_oracle(Hq, Hkv, ps):
    a = wl.make_attention("attn", [9, 257, 2000, 5003], [1, 4, 2, 3], Hq, Hkv, ps, 40, seed=Hq * 100 + ps)
    req, pos, length = rows_of(a)
    tok = oracle.expand_indices(a.blocks.numpy(), pos, length)
    check_attention(a, tok)


def test_attention_gate_future_tokens_and_missing_pages():
    a = wl.make_attention("attn_mask", [600, 1500], [4, 3], 24, 2, 16, 64, seed=11)
    req, pos, length = rows_of(a)
    tok = oracle.expand_indices(a.blocks.numpy(), pos, length)
    tok[0, 5] = pos[0] + 1                         # a future token: masked
    tok[1, 7] = length[1] + 3                      # past the request: masked
    tok[2, 2:9] = -1                               # padding inside the list
    tok[4, 0] = 1499                               # the last token of request 1, also future for row 4
    pt = a.page_table.clone()
    pt[1, 3] = -1                                  # tokens 48 .. 63 of request 1 have no page
    pt[0, 1] = a.k_cache.shape[0] + 7              # out of the pool
    gate = torch.randn(a.T, 24, generator=torch.Generator().manual_seed(3)) * 2
    check_attention(a, tok, gate=gate, pt=pt)


def test_attention_uniform_scores_give_exact_means():
    """Zero keys: every visible token has probability 1/n exactly, so the
    output is the mean of the visible integer values (bf16 rounding only)."""
    a = wl.make_attention("attn_uniform", [35, 900, 3000], [4, 2, 4], 24, 2, 64, 300, seed=5)
    g = torch.Generator().manual_seed(9)
    kc = torch.zeros_like(a.k_cache)
    vc = torch.randint(-4, 5, a.v_cache.shape, generator=g).to(torch.bfloat16)
    req, pos, length = rows_of(a)
    tok = oracle.expand_indices(a.blocks.numpy(), pos, length)
    tok[3, 0:12] = -1
    out, lse = gpu_attention(a, tok, k_cache=kc, v_cache=vc)
    ref, ref_lse = oracle.sparse_attention(a.q, kc, vc, a.page_table, req, pos, a.seq_lens, tok, scale=SCALE)
    assert np.all(np.abs(out - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
    assert np.allclose(lse, ref_lse, rtol=1e-6, atol=1e-6)


def test_attention_empty_rows_and_single_token():
    a = wl.make_attention("attn_empty", [2, 3, 800], [2, 1, 3], 24, 2, 16, 16, seed=6)
    req, pos, length = rows_of(a)
    tok = oracle.expand_indices(a.blocks.numpy(), pos, length)
    tok[3, :] = -1                                 # nothing listed
    tok[4, :] = -1
    tok[4, 9] = 17                                 # exactly one token: out = v
    out, lse = gpu_attention(a, tok)
    assert np.all(out[3] == 0) and np.all(np.isneginf(lse[3]))
    # rows 0-2 see only open-group tokens of their short requests
    ref, ref_lse = oracle.sparse_attention(a.q, a.k_cache, a.v_cache, a.page_table, req, pos, a.seq_lens, tok,
                                           scale=SCALE)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_lse))
    v17 = a.v_cache[int(a.page_table[2, 1]), 1].double().numpy()      # token 17: page 1, row 1
    for h in range(24):
        assert np.array_equal(out[4, h], v17[h // 12])


def test_attention_split_counts_agree():
    """The same rows scored alone (many splits per row) and inside a large
    batch (one split per row) give results within the bound of each other."""
    a = wl.make_attention("attn_splits", [2100] * 80, [8] * 80, 24, 2, 64, 512, seed=8)
    req, pos, length = rows_of(a)
    tok = oracle.expand_indices(a.blocks.numpy(), pos, length)
    assert qsa.sparse_attention_workspace_size(a.T, 24, 2, tok.shape[1]) > 0
    big, big_lse = gpu_attention(a, tok)
    one = wl.AttentionInputs("one", a.q[:8], a.k_cache, a.v_cache, a.page_table[:1], a.cu_seqlens_q[:2],
                             a.seq_lens[:1], a.blocks[:8])
    small, small_lse = gpu_attention(one, tok[:8])
    assert np.all(np.abs(small - big[:8]) <= 2.0 ** -7 * np.abs(big[:8]) + 2e-3)
    assert np.allclose(small_lse, big_lse[:8], rtol=1e-5, atol=1e-5)
    check_attention(one, tok[:8])
