"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with:

* the cache writer's rule (vLLM qsa_cache.py, "compressed_qsa_slot_mapping":
  a token at logical position p writes compressed row p // 4 only when
  (p + 1) % 4 == 0), simulated token by token;
* the query positions of a decode step being the last Q tokens of the request;
* the prefill FLOP counts printed in the vLLM PR "Separate prefill and decode
  paths for QSA indexer" (section "Microbenchmarks", table "Prefill");
* exact integer brute force on tiny inputs, done by another route (keys are
  first gathered into a dense per-request list by walking the page table,
  visibility comes from the writer simulation, sums are Python integers);
* closed forms, invariants and cross-entry identities of the definition in
  the QSA docs (MATE, section "MQA score");
* a full sort for the top-k selection;
* for the fp8 E4M3 key cache (vLLM qsa_cache.py, the state backend's fp8
  cache dtypes; vLLM qsa_prepare.py, "_to_dst_dtype"): torch's own E4M3
  decoding of all 256 codes and the format's fixed values, exact integer
  brute force with keys that E4M3 holds exactly, and the bf16 entry on keys
  dequantised by torch;
* for fp16 inputs (the QSA docs' second input dtype, section "MQA score"):
  torch's decoding of all 65,536 fp16 patterns, the bf16 entries on values
  both formats hold exactly, and a closed form on a value only fp16 holds.

The same functions run against deliberately broken builds of the oracle
(``test_oracle_mutants.py``) to show that each plausible mistake trips a pin.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "vllm_qsa_indexer_microbench.txt")
SCALE = 1.0 / math.sqrt(128.0)


# ---------------------------------------------------------------- helpers

def keys_written_through(p: int) -> list[int]:
    """Compressed rows in the cache once tokens 0..p have been processed."""
    out = []
    for tok in range(p + 1):
        if (tok + 1) % 4 == 0:
            out.append(tok // 4)
    return out


def int_bf16(shape, lo, hi, rng: np.random.Generator) -> torch.Tensor:
    """Small integers, exactly representable in bf16."""
    return torch.from_numpy(rng.integers(lo, hi + 1, size=shape).astype(np.float32)).to(torch.bfloat16)


def as_int(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float32).numpy().astype(np.int64)


def int_score(q_row_heads: np.ndarray, k_row: np.ndarray) -> int:
    """sum_h max(0, q_h . k) in exact integers (q_row_heads: [4, 128])."""
    total = 0
    for h in range(q_row_heads.shape[0]):
        d = sum(int(a) * int(b) for a, b in zip(q_row_heads[h], k_row))
        total += max(0, d)
    return total


def paged_case(rng, B, Q, page_size, seq_lens, bad_pages=True, extra_w=3, lo=-3, hi=3):
    """Tiny paged decode case with integer data.  Some table entries past the
    visible range, and (optionally) some inside it, are invalid (-1 or past
    the pool)."""
    pages_per_req = [max(1, -(-L // (4 * page_size))) for L in seq_lens]
    num_pages = sum(pages_per_req) + 2
    max_pages = max(pages_per_req) + 1
    perm = rng.permutation(num_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    at = 0
    for b, p in enumerate(pages_per_req):
        table[b, :p] = perm[at:at + p]
        at += p
    if bad_pages and B > 1:
        table[1, 0] = num_pages + 5          # out of range
        if pages_per_req[1] > 1:
            table[1, 1] = -1                  # missing
    q = int_bf16((B, Q, 4, 128), lo, hi, rng)
    k_cache = int_bf16((num_pages, page_size, 1, 128), lo, hi, rng)
    W = max(L // 4 for L in seq_lens) + extra_w
    return q, k_cache, torch.from_numpy(table), torch.tensor(seq_lens, dtype=torch.int32), W


def dense_request_keys(k_cache_int, table_row, page_size, num_pages):
    """The request's keys in logical order, None where the page is invalid."""
    keys = []
    for page in table_row:
        for r in range(page_size):
            keys.append(k_cache_int[page, r, 0] if 0 <= page < num_pages else None)
    return keys


def brute_decode(q, k_cache, table, seq_lens, W):
    qi, ki = as_int(q), as_int(k_cache)
    B, Q = qi.shape[:2]
    out = np.full((B, Q, W), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        keys = dense_request_keys(ki, table[b].tolist(), k_cache.shape[1], k_cache.shape[0])
        positions = list(range(L))[-Q:] if L >= Q else [L - Q + i for i in range(Q)]
        for i, p in enumerate(positions):
            written = keys_written_through(p) if p >= 0 else []
            for n in written:
                if n < W and n < len(keys) and keys[n] is not None:
                    out[b, i, n] = int_score(qi[b, i], keys[n])
    return out


def packed_case(rng, new_tokens, prefixes, lo=-3, hi=3):
    total = [p + n for p, n in zip(prefixes, new_tokens)]
    nkeys = [len(keys_written_through(t - 1)) for t in total]
    T = sum(new_tokens)
    q = int_bf16((T, 4, 128), lo, hi, rng)
    k = int_bf16((sum(nkeys), 128), lo, hi, rng)
    cu = np.concatenate([[0], np.cumsum(new_tokens)]).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(nkeys)[:-1]]).astype(np.int32)
    return q, k, cu, np.array(total, dtype=np.int32), offs, max(nkeys)


# ---------------------------------------------------------------- the mask

def pin_visible_blocks_follow_cache_writer(orc):
    for L in range(0, 41):
        for p in range(0, L):
            written = keys_written_through(p)
            assert written == list(range(len(written)))
            v = orc.visible_blocks(p, L)
            assert v == len(written), (p, L, v, len(written))
        # a padding row (logical position -1) sees nothing
        assert orc.visible_blocks(-1, L) == 0
        # positions past the request are capped at the keys the cache holds
        assert orc.visible_blocks(L + 9, L) == len(keys_written_through(L - 1))


def pin_decode_positions_are_last_tokens(orc):
    for L in range(1, 30):
        for Q in range(1, min(L, 4) + 1):
            expect = list(range(L))[-Q:]
            got = [orc.logical_position(L, Q, i) for i in range(Q)]
            assert got == expect, (L, Q, got, expect)
            vis = orc.decode_visible([L], Q)[0].tolist()
            assert vis == [len(keys_written_through(p)) for p in expect]
    # fewer tokens than query rows: the leading rows have no position
    assert orc.decode_visible([2], 4)[0].tolist() == [0, 0, 0, 0]


def pin_prefill_flops_match_published_table(orc):
    rows = 0
    with open(GOLDEN) as f:
        for line in f:
            parts = line.split()
            if not parts or parts[0] != "prefill":
                continue
            S, n = map(int, parts[1].split("x"))
            prefix = int(parts[2])
            cu = [i * n for i in range(S + 1)]
            ks, ke = orc.prefill_intervals(cu, [prefix + n] * S, [0] * S)
            flop = 2 * 4 * 128 * int((ke.astype(np.int64) - ks).sum())
            for us, printed in ((float(parts[3]), float(parts[5])),
                                (float(parts[4]), float(parts[6]))):
                got = round(flop / us / 1e6, 1)
                assert got == printed, (parts[1], prefix, us, got, printed)
            rows += 1
    assert rows == 12


def pin_prefill_intervals_follow_cache_writer(orc):
    new, pre = [5, 1, 9, 3], [0, 7, 13, 2]
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    total = [a + b for a, b in zip(pre, new)]
    offs = [0, 11, 30, 50]
    ks, ke = orc.prefill_intervals(cu, total, offs)
    t = 0
    for s in range(4):
        for i in range(new[s]):
            p = pre[s] + i
            assert ks[t] == offs[s]
            assert ke[t] - ks[t] == len(keys_written_through(p)), (s, i)
            t += 1


# ---------------------------------------------------------------- the score

def pin_decode_exact_bruteforce(orc):
    rng = np.random.default_rng(1)
    # query lengths past 4 are the prefill rows of a request read from the
    # paged cache (a mixed decode + prefill batch scores them the same way)
    cases = [(1, 1, 8, [37]), (3, 4, 8, [70, 41, 2]), (2, 2, 16, [130, 75]),
             (3, 3, 8, [0, 66, 19]), (2, 4, 16, [64, 3]), (2, 9, 16, [70, 41]), (1, 33, 8, [200]),
             (1, 12, 8, [5])]
    for B, Q, ps, lens in cases:
        q, kc, table, sl, W = paged_case(rng, B, Q, ps, lens)
        got = orc.decode(q, kc, table, sl, W, scale=1.0, threads=2)
        want = brute_decode(q, kc, table.numpy(), sl.numpy(), W)
        assert np.array_equal(got, want), (B, Q, ps, lens)


def pin_prefill_exact_bruteforce(orc):
    rng = np.random.default_rng(2)
    new, pre = [6, 3, 9], [5, 0, 22]
    q, k, cu, total, offs, Wmax = packed_case(rng, new, pre)
    ks, ke = orc.prefill_intervals(cu, total, offs)
    W = Wmax + 2
    got = orc.prefill(q, k, ks, ke, W, scale=1.0, threads=2)
    qi, ki = as_int(q), as_int(k)
    want = np.full((q.shape[0], W), -np.inf)
    t = 0
    for s in range(3):
        for i in range(new[s]):
            for n in keys_written_through(pre[s] + i):
                want[t, n] = int_score(qi[t], ki[offs[s] + n])
            t += 1
    assert np.array_equal(got, want)
    # arbitrary intervals, clipped to the key range, column j holding key ks + j
    T, Nk = q.shape[0], k.shape[0]
    ks2 = rng.integers(-4, Nk, size=T).astype(np.int32)
    ke2 = (ks2 + rng.integers(-2, 9, size=T)).astype(np.int32)
    ke2[0], ks2[1], ke2[1] = Nk + 5, -3, 4
    got2 = orc.prefill(q, k, ks2, ke2, 12, scale=1.0)
    for t in range(T):
        for j in range(12):
            n = int(ks2[t]) + j
            ok = max(int(ks2[t]), 0) <= n < min(int(ke2[t]), Nk)
            want_tj = int_score(qi[t], ki[n]) if ok else -np.inf
            assert got2[t, j] == want_tj, (t, j)


def pin_prefill_entries_match_bruteforce(orc):
    """The listed-entries form of the prefill oracle (the checker of the
    full-size parity tests, which sample rows and columns) against exact
    integer brute force: entries in shuffled order, repeated entries,
    intervals that start below 0, end past the keys, are empty or reversed,
    and columns past each interval."""
    rng = np.random.default_rng(11)
    new, pre = [6, 3, 9], [5, 0, 22]
    q, k, _, _, _, _ = packed_case(rng, new, pre)
    T, Nk = q.shape[0], k.shape[0]
    ks = rng.integers(-4, Nk, size=T).astype(np.int32)
    ke = (ks + rng.integers(-2, 12, size=T)).astype(np.int32)
    ke[0], ks[1], ke[1], ks[2], ke[2] = Nk + 5, -3, 4, 3, 3
    tt, jj = np.meshgrid(np.arange(T), np.arange(T), indexing="ij")
    tt, jj = tt.ravel(), jj.ravel()
    order = rng.permutation(tt.size)
    tt = np.concatenate([tt[order], tt[order[:7]]])
    jj = np.concatenate([jj[order], jj[order[:7]]])
    got = orc.prefill_entries(q, k, ks, ke, tt, jj, scale=1.0, threads=3)
    qi, ki = as_int(q), as_int(k)
    for e in range(tt.size):
        t, j = int(tt[e]), int(jj[e])
        n = int(ks[t]) + j
        ok = max(int(ks[t]), 0) <= n < min(int(ke[t]), Nk)
        want = int_score(qi[t], ki[n]) if ok else -np.inf
        assert got[e] == want, (e, t, j)


def pin_closed_forms(orc):
    T = 3
    q = torch.zeros(T, 4, 128, dtype=torch.bfloat16)
    k = torch.zeros(4, 128, dtype=torch.bfloat16)
    q[0, 2, :] = 1.0                       # one head all ones
    k[0, :] = 1.0                          # key all ones
    k[1, 17] = 1.0                         # key = e_17
    q[1] = torch.tensor(np.random.default_rng(3).normal(size=(4, 128)), dtype=torch.bfloat16)
    q[2] = 1.0
    k[2, :] = -1.0                         # every dot product negative
    ks = np.zeros(T, dtype=np.int32)
    ke = np.full(T, 4, dtype=np.int32)
    s = orc.prefill(q, k, ks, ke, 4, scale=SCALE)
    assert abs(s[0, 0] - math.sqrt(128.0)) <= 1e-12
    want = SCALE * sum(max(float(q[1, h, 17]), 0.0) for h in range(4))
    assert abs(s[1, 1] - want) <= 1e-15
    assert s[2, 2] == 0.0
    assert s[0, 3] == 0.0 and s[1, 3] == 0.0  # zero key
    assert abs(s[2, 0] - 4 * 128 * SCALE) <= 1e-12


def pin_invariants(orc):
    rng = np.random.default_rng(4)
    B, Q, ps, lens = 3, 4, 8, [90, 33, 61]
    q, kc, table, sl, W = paged_case(rng, B, Q, ps, lens, bad_pages=False, lo=-8, hi=8)
    base = orc.decode(q, kc, table, sl, W)
    vis = orc.decode_visible(sl, Q)
    cols = np.arange(W)[None, None, :]
    unmasked = cols < vis[:, :, None]
    assert np.all(base[unmasked] >= 0.0)
    assert np.all(np.isneginf(base[~unmasked]))
    # zero queries give zeros where unmasked
    z = orc.decode(torch.zeros_like(q), kc, table, sl, W)
    assert np.all(z[unmasked] == 0.0) and np.all(np.isneginf(z[~unmasked]))
    # moving pages to other slots of the pool changes nothing
    P = kc.shape[0]
    perm = rng.permutation(P)
    kc2 = torch.empty_like(kc)
    kc2[torch.from_numpy(perm)] = kc
    t2 = table.numpy().copy()
    t2[t2 >= 0] = perm[t2[t2 >= 0]]
    assert np.array_equal(orc.decode(q, kc2, torch.from_numpy(t2), sl, W), base)
    # scaling keys by c > 0 scales scores by c: exactly for powers of two, and
    # exactly for any c once the 1/sqrt(128) multiplier is left out
    for c in (2.0, 0.5):
        sc = orc.decode(q, (kc.float() * c).to(torch.bfloat16), table, sl, W)
        assert np.array_equal(sc[unmasked], c * base[unmasked])
    unscaled = orc.decode(q, kc, table, sl, W, scale=1.0)
    for c in (3.0, 5.0):
        sc = orc.decode(q, (kc.float() * c).to(torch.bfloat16), table, sl, W, scale=1.0)
        assert np.array_equal(sc[unmasked], c * unscaled[unmasked])


def pin_cross_entry_identities(orc):
    rng = np.random.default_rng(5)
    B, Q, ps, lens = 2, 4, 8, [77, 45]
    q, kc, table, sl, W = paged_case(rng, B, Q, ps, lens, bad_pages=False, lo=-8, hi=8)
    spec = orc.decode(q, kc, table, sl, W)
    # spec-decode row i == single-token decode of the request cut after that token
    for i in range(Q):
        sl_i = sl - Q + i + 1
        one = orc.decode(q[:, i:i + 1], kc, table, sl_i, W)
        assert np.array_equal(one[:, 0], spec[:, i]), i
    # paged decode == prefill over the request's keys laid out densely
    vis = orc.decode_visible(sl, Q)
    for b in range(B):
        pages = [p for p in table[b].tolist() if p >= 0]
        dense = torch.cat([kc[p, :, 0, :] for p in pages], dim=0)
        ks = np.zeros(Q, dtype=np.int32)
        ke = vis[b].astype(np.int32)
        pre = orc.prefill(q[b], dense, ks, ke, W)
        assert np.array_equal(pre, spec[b]), b
    # the same keys paged with 16 rows per page instead of 8
    keys = [torch.cat([kc[p, :, 0, :] for p in table[b].tolist() if p >= 0]) for b in range(B)]
    ps2 = 16
    pool, t16 = [], np.full((B, 8), -1, dtype=np.int32)
    for b in range(B):
        kb = keys[b]
        pad = (-kb.shape[0]) % ps2
        kb = torch.cat([kb, torch.zeros(pad, 128, dtype=kb.dtype)])
        for j in range(kb.shape[0] // ps2):
            t16[b, j] = len(pool)
            pool.append(kb[j * ps2:(j + 1) * ps2])
    kc16 = torch.stack(pool)[:, :, None, :]
    assert np.array_equal(orc.decode(q, kc16, torch.from_numpy(t16), sl, W), spec)
    # longer intervals leave earlier columns unchanged
    Tq = q[0]
    ks = np.zeros(Q, dtype=np.int32)
    short = orc.prefill(Tq, keys[0], ks, np.full(Q, 5, dtype=np.int32), 12)
    longer = orc.prefill(Tq, keys[0], ks, np.full(Q, 12, dtype=np.int32), 12)
    assert np.array_equal(short[:, :5], longer[:, :5])


# ---------------------------------------------------------------- top-k

def pin_topk_against_full_sort(orc):
    rng = np.random.default_rng(6)
    rows, width, k = 40, 300, 16
    s = rng.normal(size=(rows, width))
    s[rng.random(size=s.shape) < 0.05] = -np.inf
    lengths = rng.integers(0, width + 1, size=rows).astype(np.int32)
    lengths[:4] = [0, 5, 16, width]
    got = orc.topk(s, lengths, k)
    for r in range(rows):
        L = int(lengths[r])
        cand = np.flatnonzero(np.isfinite(s[r, :L]))
        order = cand[np.argsort(-s[r, cand], kind="stable")][:k]
        want = sorted(order.tolist()) + [-1] * (k - len(order))
        assert got[r].tolist() == want, r


def pin_topk_ties_and_padding(orc):
    k = 4
    s = np.array([
        [1.0] * 10,                                              # all tied: lowest columns
        [0.0, -0.0, 0.0, -0.0, 5.0, 0.0, 0.0, 0.0, 0.0, 0.0],    # signed zeros tie
        [3.0, -np.inf, 2.0, -np.inf, 1.0, 0.0, 0.0, 0.0, 0.0, 0.0],
        [2.0, 1.0, 3.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
    ])
    lengths = np.array([10, 10, 4, 2], dtype=np.int32)
    got = orc.topk(s, lengths, k)
    assert got[0].tolist() == [0, 1, 2, 3]
    assert got[1].tolist() == [0, 1, 2, 4]
    assert got[2].tolist() == [0, 2, -1, -1]    # masked blocks are never selected
    assert got[3].tolist() == [0, 1, -1, -1]
    # NaN is not a candidate either
    s2 = np.array([[np.nan, 1.0, np.nan, 2.0]])
    assert orc.topk(s2, np.array([4], dtype=np.int32), 3)[0].tolist() == [1, 3, -1]


def _repage(kc, table, B, ps2):
    """The requests' keys laid out again with ps2 rows per page (pages in
    reverse order in the pool, -1 past each request's pages)."""
    keys = [torch.cat([kc[p, :, 0, :] for p in table[b].tolist() if p >= 0]) for b in range(B)]
    pool, rows = [], []
    for b in range(B):
        kb = keys[b]
        kb = torch.cat([kb, torch.zeros((-kb.shape[0]) % ps2, 128, dtype=kb.dtype)])
        rows.append([])
        for j in range(kb.shape[0] // ps2):
            rows[b].append(len(pool))
            pool.append(kb[j * ps2:(j + 1) * ps2])
    n = len(pool)
    width = max(len(r) for r in rows) + 1
    t = np.full((B, width), -1, dtype=np.int32)
    for b in range(B):
        t[b, :len(rows[b])] = [n - 1 - p for p in rows[b]]
    kc2 = torch.stack(pool[::-1])[:, :, None, :]
    return kc2, torch.from_numpy(t)


def pin_page_sizes_not_powers_of_two(orc):
    """The production page size 196 (and 12) lays out the same keys: the
    scores must not change, including blocks that straddle page edges."""
    rng = np.random.default_rng(6)
    B, Q, lens = 2, 3, [2000, 900]
    q, kc, table, sl, W = paged_case(rng, B, Q, 8, lens, bad_pages=False)
    ref = orc.decode(q, kc, table, sl, W)
    for ps2 in (196, 12, 64):
        kc2, t2 = _repage(kc, table, B, ps2)
        assert np.array_equal(orc.decode(q, kc2, t2, sl, W), ref), ps2
    assert np.isfinite(ref).sum() > 600


# ---------------------------------------------------------------- fp8 cache

def pin_e4m3_decoder(orc):
    """Every E4M3 code against torch's float8_e4m3fn decoding, and the
    format's fixed points (no infinities, NaN at 0x7f / 0xff, largest finite
    value 448, smallest subnormal 2^-9, smallest normal 2^-6, 1.0 = 0x38)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_to_double(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0
    assert got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6 and got[0x38] == 1.0
    assert got[0x00] == 0.0 and math.copysign(1.0, got[0x80]) == -1.0


def _e4m3_codes(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)


def pin_fp8_decode_exact_bruteforce(orc):
    """Integer keys (exact in E4M3) with k_scale 3 and 1/2: the score is
    k_scale times the exact integer brute force."""
    rng = np.random.default_rng(11)
    cases = [(1, 1, 8, [37]), (3, 4, 8, [70, 41, 2]), (2, 3, 16, [130, 75])]
    for B, Q, ps, lens in cases:
        q, kc, table, sl, W = paged_case(rng, B, Q, ps, lens)
        k8 = _e4m3_codes(kc)
        want = brute_decode(q, kc, table.numpy(), sl.numpy(), W)
        for ks in (3.0, 0.5):
            got = orc.decode_fp8(q, k8, ks, table, sl, W, scale=1.0, threads=2)
            assert np.array_equal(got, want * ks), (B, Q, ps, lens, ks)


def pin_fp8_matches_bf16_on_dequantised_keys(orc):
    """Random finite codes (subnormals and both zeros included) with a
    power-of-two k_scale: every dequantised key is exact in bf16, so the fp8
    entry must equal the bf16 entry on the keys torch dequantises."""
    g = torch.Generator().manual_seed(12)
    B, Q, ps, lens = 3, 2, 16, [300, 41, 200]
    pages = sum(-(-L // (4 * ps)) for L in lens) + 1
    codes = torch.randint(0, 256, (pages, ps, 1, 128), generator=g, dtype=torch.int32)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0x00
    codes[0, 0, 0, :8] = torch.tensor([0x00, 0x80, 0x01, 0x81, 0x07, 0x08, 0x7E, 0xFE])
    k8 = codes.to(torch.uint8)
    ks = 2.0 ** -5
    kbf = (k8.view(torch.float8_e4m3fn).to(torch.float32) * ks).to(torch.bfloat16)
    assert torch.equal(kbf.to(torch.float64), k8.view(torch.float8_e4m3fn).to(torch.float64) * ks)
    q = torch.randn(B, Q, 4, 128, generator=g).to(torch.bfloat16)
    table = torch.full((B, max(-(-L // (4 * ps)) for L in lens)), -1, dtype=torch.int32)
    at = 0
    for b, L in enumerate(lens):
        n = -(-L // (4 * ps))
        table[b, :n] = torch.arange(at, at + n, dtype=torch.int32)
        at += n
    sl = torch.tensor(lens, dtype=torch.int32)
    W = max(lens) // 4 + 5
    got = orc.decode_fp8(q, k8, ks, table, sl, W, threads=2)
    want = orc.decode(q, kbf, table, sl, W, threads=2)
    assert np.array_equal(np.isneginf(got), np.isneginf(want))
    assert np.array_equal(got, want)
    assert np.isfinite(got).sum() > 0


# ---------------------------------------------------------------- fp16 inputs

def pin_f16_decoder(orc):
    """Every fp16 bit pattern against torch's float16 decoding (zeros of
    both signs, subnormals down to 2^-24, the largest finite 65504,
    infinities, NaNs)."""
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.float16).to(torch.float64).numpy()
    got = np.array([orc.f16_to_double(b) for b in range(65536)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x0001] == 2.0 ** -24 and got[0x7BFF] == 65504.0 and got[0x3C00] == 1.0
    assert got[0x7C00] == np.inf and got[0xFC00] == -np.inf
    assert math.copysign(1.0, got[0x8000]) == -1.0


def pin_f16_matches_bf16_on_shared_values(orc):
    """Small integers are exact in both formats: the fp16 decode and prefill
    entries must equal the bf16 ones on them, element for element."""
    rng = np.random.default_rng(21)
    q, kc, table, sl, W = paged_case(rng, 3, 4, 16, [300, 41, 130])
    a = orc.decode(q, kc, table, sl, W, threads=2)
    b = orc.decode(q.to(torch.float16), kc.to(torch.float16), table, sl, W, threads=2)
    assert np.array_equal(a, b) and np.isfinite(a).sum() > 0
    qp, kp, cu, total, offs, maxk = packed_case(rng, [9, 5], [30, 0])
    ks, ke = orc.prefill_intervals(cu, total, offs)
    a = orc.prefill(qp, kp, ks, ke, maxk + 2, threads=2)
    b = orc.prefill(qp.to(torch.float16), kp.to(torch.float16), ks, ke, maxk + 2, threads=2)
    assert np.array_equal(a, b) and np.isfinite(a).sum() > 0


def pin_f16_closed_form(orc):
    """q_0 = (1 + 2^-10) e_0 (exact in fp16, not in bf16) and k = e_0:
    the score is exactly scale * (1 + 2^-10), and 0 with -q."""
    q = torch.zeros(1, 4, 128, dtype=torch.float16)
    q[0, 0, 0] = 1.0 + 2.0 ** -10
    k = torch.zeros(1, 128, dtype=torch.float16)
    k[0, 0] = 1.0
    ks, ke = np.array([0], dtype=np.int32), np.array([1], dtype=np.int32)
    got = orc.prefill(q, k, ks, ke, 1, scale=0.5)
    assert got[0, 0] == 0.5 * (1.0 + 2.0 ** -10)
    assert orc.prefill(-q, k, ks, ke, 1, scale=0.5)[0, 0] == 0.0
    d = orc.decode(q.view(1, 1, 4, 128), k.view(1, 1, 1, 128).expand(1, 8, 1, 128).contiguous(),
                   torch.zeros(1, 1, dtype=torch.int32), torch.tensor([4], dtype=torch.int32), 1, scale=0.5)
    assert d[0, 0, 0] == 0.5 * (1.0 + 2.0 ** -10)


# ---------------------------------------------------------------- core attention

def pin_expand_indices_follow_cache_writer(orc):
    """Block -> token expansion (QSA docs, "Core Attention": token width =
    4 * blocks + 3) against the cache writer's rule: a row keeps the four
    tokens of each selected block, then the tokens written since its last
    complete group."""
    rng = np.random.default_rng(31)
    k = 4
    rows, pos, sl, want = [], [], [], []
    for L in range(1, 34):
        for p in range(0, L):
            written = keys_written_through(p)            # complete blocks at position p
            take = sorted(rng.choice(len(written), size=min(k, len(written)), replace=False).tolist()) \
                if written else []
            if len(take) > 1 and rng.random() < 0.3:
                take = take[:-1]
            blk = take + [-1] * (k - len(take))
            toks = [4 * b + r for b in take for r in range(4)]
            toks += list(range(4 * len(written), p + 1))  # the open group, at most 3 tokens
            assert len(toks) <= 4 * k + 3
            rows.append(blk)
            pos.append(p)
            sl.append(L)
            want.append(toks + [-1] * (4 * k + 3 - len(toks)))
    rows.append([3, -1, 0, -1])                          # a padding row: blocks only
    pos.append(-1)
    sl.append(20)
    want.append([12, 13, 14, 15, 0, 1, 2, 3] + [-1] * 11)
    got = orc.expand_indices(np.array(rows), np.array(pos), np.array(sl))
    assert np.array_equal(got, np.array(want, dtype=np.int32))


def _attn_case(rng, lens, Hq, Hkv, ps, lo=-2, hi=2):
    """Paged K/V pools with small-integer bf16 data, pages permuted."""
    pages_per_req = [max(1, -(-L // ps)) for L in lens]
    num_pages = sum(pages_per_req) + 1
    perm = rng.permutation(num_pages)
    table = np.full((len(lens), max(pages_per_req)), -1, dtype=np.int32)
    at = 0
    for r, n in enumerate(pages_per_req):
        table[r, :n] = perm[at:at + n]
        at += n
    kc = int_bf16((num_pages, ps, Hkv, 256), lo, hi, rng)
    vc = int_bf16((num_pages, ps, Hkv, 256), lo, hi, rng)
    return kc, vc, table


def _dense_kv(cache, table_row, ps, L):
    """K or V of one request in token order [L, Hkv, 256] (a walk of its pages)."""
    return torch.stack([cache[int(table_row[j // ps]), j % ps] for j in range(L)])


def pin_sparse_attention_matches_library_sdpa(orc):
    """When a row's list holds every token it may see (in any order, with -1
    pads, duplicates of nothing, and future tokens that must be masked),
    sparse attention is dense causal attention: torch's
    scaled_dot_product_attention in fp64 on the densely gathered K/V, with the
    grouped heads expanded, and torch.logsumexp for the LSE."""
    rng = np.random.default_rng(32)
    lens, Hq, Hkv, ps = [37, 70], 6, 2, 16
    kc, vc, table = _attn_case(rng, lens, Hq, Hkv, ps)
    rows = [(0, 36), (0, 20), (1, 69), (1, 3), (1, 0)]
    width = 80
    tok = np.full((len(rows), width), -1, dtype=np.int32)
    for t, (r, p) in enumerate(rows):
        toks = list(range(p + 1)) + list(range(p + 1, min(p + 6, lens[r])))   # some future tokens
        toks = rng.permutation(toks).tolist()
        slots = np.sort(rng.choice(width, size=len(toks), replace=False))
        tok[t, slots] = toks
    q = int_bf16((len(rows), Hq, 256), -2, 2, rng)
    scale = 1.0 / 16.0
    out, lse = orc.sparse_attention(q, kc, vc, table, [r for r, _ in rows], [p for _, p in rows], lens, tok,
                                    scale=scale, threads=2)
    group = Hq // Hkv
    for t, (r, p) in enumerate(rows):
        K = _dense_kv(kc, table[r], ps, p + 1).double()          # [n, Hkv, 256]
        V = _dense_kv(vc, table[r], ps, p + 1).double()
        Kh = K.repeat_interleave(group, dim=1).transpose(0, 1)   # [Hq, n, 256]
        Vh = V.repeat_interleave(group, dim=1).transpose(0, 1)
        qq = q[t].double()[:, None, :]                           # [Hq, 1, 256]
        want = torch.nn.functional.scaled_dot_product_attention(qq, Kh, Vh, scale=scale)[:, 0]
        want_lse = torch.logsumexp(scale * (qq @ Kh.transpose(1, 2))[:, 0], dim=-1)
        assert np.allclose(out[t], want.numpy(), rtol=1e-12, atol=1e-12), t
        assert np.allclose(lse[t], want_lse.numpy(), rtol=1e-12, atol=1e-12), t


def pin_sparse_attention_closed_forms(orc):
    rng = np.random.default_rng(33)
    lens, Hq, Hkv, ps = [40], 4, 2, 8
    kc, vc, table = _attn_case(rng, lens, Hq, Hkv, ps)
    kc = torch.zeros_like(kc)                                    # every score 0: uniform weights
    vc[..., 1, :] = vc[..., 0, :] + 100                          # KV head 1 = head 0 + 100
    q = int_bf16((4, Hq, 256), -2, 2, rng)
    width = 6
    tok = np.array([[5, -1, -1, -1, -1, -1],                     # one token: out = v, lse = 0
                    [5, 9, -1, -1, -1, -1],                      # two: the mean, lse = log 2
                    [39, 38, -1, -1, -1, -1],                    # both after the row's position: empty
                    [2, 3, -1, -1, -1, -1]], dtype=np.int32)     # padding row (no request)
    req, pos = [0, 0, 0, -1], [30, 30, 30, 30]
    gate = np.zeros((4, Hq))
    gate[1] = 0.0
    out, lse = orc.sparse_attention(q, kc, vc, table, req, pos, lens, tok, scale=0.5)
    V = _dense_kv(vc, table[0], ps, 40).double().numpy()         # [40, Hkv, 256]
    group = Hq // Hkv
    for h in range(Hq):
        g = h // group
        assert np.array_equal(out[0, h], V[5, g]) and lse[0, h] == 0.0
        assert np.array_equal(out[1, h], (V[5, g] + V[9, g]) / 2) and lse[1, h] == np.log(2.0)
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))
    assert np.all(out[3] == 0) and np.all(np.isneginf(lse[3]))
    # a gate of 0 halves the output exactly (sigmoid(0) = 1/2)
    g_out, g_lse = orc.sparse_attention(q, kc, vc, table, req, pos, lens, tok, scale=0.5, gate=gate)
    assert np.array_equal(g_out[:2], out[:2] / 2) and np.array_equal(g_lse, lse)
    # a missing page drops its tokens: the same as leaving them out of the list
    t2 = table.copy()
    t2[0, 1] = -1                                                # tokens 8..15
    m_out, _ = orc.sparse_attention(q, kc, vc, t2, req, pos, lens, tok, scale=0.5)
    assert np.array_equal(m_out[1], out[0])                      # token 9 gone, token 5 left


ALL_PINS = [
    pin_visible_blocks_follow_cache_writer,
    pin_decode_positions_are_last_tokens,
    pin_prefill_flops_match_published_table,
    pin_prefill_intervals_follow_cache_writer,
    pin_decode_exact_bruteforce,
    pin_prefill_exact_bruteforce,
    pin_prefill_entries_match_bruteforce,
    pin_closed_forms,
    pin_invariants,
    pin_cross_entry_identities,
    pin_page_sizes_not_powers_of_two,
    pin_topk_against_full_sort,
    pin_topk_ties_and_padding,
    pin_e4m3_decoder,
    pin_fp8_decode_exact_bruteforce,
    pin_fp8_matches_bf16_on_dequantised_keys,
    pin_f16_decoder,
    pin_f16_matches_bf16_on_shared_values,
    pin_f16_closed_form,
    pin_expand_indices_follow_cache_writer,
    pin_sparse_attention_matches_library_sdpa,
    pin_sparse_attention_closed_forms,
]
