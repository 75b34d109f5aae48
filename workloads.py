"""Seeded synthetic inputs for the QSA MQA indexer score.

This module only builds inputs: random bf16 queries and keys, context lengths,
paged key pools and their page tables, packed prefill layouts.  It computes
nothing of the score or of its mask; the CUDA path and the CPU oracle each do
that on their own from what is built here.

Shapes follow the QSA docs (MATE, section "MQA score"): queries carry 4 heads
of dimension 128, one compressed key of dimension 128 stands for a group of 4
tokens, and the decode cache is paged as ``[pages, page_size, 1, 128]``.  The
workload sizes follow the vLLM PR "Separate prefill and decode paths for QSA
indexer" (section "Microbenchmarks"): 16 requests with log-normal context
lengths for decode and spec-decode, and long-prefix prefill layouts.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

HEADS = 4              # query heads sharing one compressed key head
DIM = 128              # head dimension
TOKENS_PER_KEY = 4     # tokens behind one compressed key (the compression ratio)


@dataclass
class DecodeInputs:
    """Decode / spec-decode inputs (all tensors on the CPU)."""
    name: str
    q: torch.Tensor            # bf16 [B, Q, 4, 128]
    k_cache: torch.Tensor      # bf16 [num_pages, page_size, 1, 128]
    page_table: torch.Tensor   # int32 [B, max_pages], -1 where unused
    seq_lens: torch.Tensor     # int32 [B], tokens per request (query tokens included)
    page_size: int
    W: int                     # output width (columns per score row)
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return self.q.shape[0]

    @property
    def Q(self) -> int:
        return self.q.shape[1]


@dataclass
class PrefillInputs:
    """Packed prefill inputs (all tensors on the CPU).

    Sequence ``s`` owns query rows ``cu_seqlens_q[s] .. cu_seqlens_q[s+1]`` and
    key rows ``key_offsets[s] ..``; ``seq_lens[s]`` counts all its tokens
    (cached prefix plus the new query tokens).
    """
    name: str
    q: torch.Tensor            # bf16 [T, 4, 128]
    k: torch.Tensor            # bf16 [Nk, 128]
    cu_seqlens_q: torch.Tensor # int32 [S + 1]
    seq_lens: torch.Tensor     # int32 [S]
    key_offsets: torch.Tensor  # int32 [S]
    W: int
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return self.q.shape[0]

    @property
    def Nk(self) -> int:
        return self.k.shape[0]


def _gen(seed: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed)


def randn_bf16(shape, gen: torch.Generator) -> torch.Tensor:
    """N(0, 1) samples rounded to bf16."""
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def lognormal_contexts(n: int, lo: int, hi: int, total: int, seed: int = 0) -> list[int]:
    """``n`` log-normal context lengths with min ``lo``, max ``hi`` and sum ``total``.

    Draws n standard normals, maps them linearly in log space so that the
    smallest becomes ``lo`` and the largest ``hi``, then shifts the interior
    values in log space (bisection) until the rounded lengths sum to ``total``;
    the last few tokens of rounding go to the median element.
    """
    if n == 1:
        return [hi]
    z = torch.randn(n, generator=_gen(seed), dtype=torch.float64).tolist()
    zmin, zmax = min(z), max(z)
    imin, imax = z.index(zmin), z.index(zmax)
    llo, lhi = math.log(lo), math.log(hi)
    base = [llo + (v - zmin) / (zmax - zmin) * (lhi - llo) for v in z]

    def lengths(shift: float) -> list[int]:
        out = []
        for i, b in enumerate(base):
            if i == imin:
                out.append(lo)
            elif i == imax:
                out.append(hi)
            else:
                out.append(int(round(math.exp(min(max(b + shift, llo), lhi)))))
        return out

    a, b = -20.0, 20.0
    for _ in range(200):
        mid = 0.5 * (a + b)
        if sum(lengths(mid)) < total:
            a = mid
        else:
            b = mid
    out = lengths(a)
    interior = sorted((i for i in range(n) if i not in (imin, imax)), key=lambda i: out[i])
    med = interior[len(interior) // 2]
    out[med] += total - sum(out)
    if not (lo <= out[med] <= hi):
        raise ValueError("context lengths cannot meet the requested sum")
    return out


def make_decode(name: str, seq_lens: list[int], Q: int, page_size: int, seed: int,
                W: int | None = None, spare_pages: int = 1, table_pad: int = 0) -> DecodeInputs:
    """Paged decode inputs.

    Each request gets just enough pages to hold keys for all of its tokens
    (``TOKENS_PER_KEY * page_size`` tokens per page); the pool has
    ``spare_pages`` more, and pages are handed out by a random permutation.
    Table entries past a request's pages are -1.  Every pool row is N(0, 1),
    including rows no visible key maps to.
    """
    g = _gen(seed)
    B = len(seq_lens)
    tokens_per_page = TOKENS_PER_KEY * page_size
    pages_per_req = [max(1, -(-L // tokens_per_page)) for L in seq_lens]
    num_pages = sum(pages_per_req) + spare_pages
    max_pages = max(pages_per_req) + table_pad
    q = randn_bf16((B, Q, HEADS, DIM), g)
    k_cache = randn_bf16((num_pages, page_size, 1, DIM), g)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    at = 0
    for b, p in enumerate(pages_per_req):
        table[b, :p] = perm[at:at + p]
        at += p
    if W is None:
        W = max(seq_lens) // TOKENS_PER_KEY
    return DecodeInputs(name=name, q=q, k_cache=k_cache, page_table=table,
                        seq_lens=torch.tensor(seq_lens, dtype=torch.int32),
                        page_size=page_size, W=W,
                        meta={"seed": seed, "context_tokens": list(seq_lens)})


def e4m3_cache(k_cache: torch.Tensor, k_scale: float | None = None) -> tuple[torch.Tensor, float]:
    """An fp8 E4M3 copy of a bf16 key pool, as the cache writer stores it
    (vLLM qsa_prepare.py, "_to_dst_dtype": the bf16 key divided by the cache
    scale, converted to E4M3 by torch).  ``k_scale`` defaults to the pool's
    largest magnitude / 448 (the largest finite E4M3 value), so no code
    saturates and none is NaN.  Returns (uint8 codes of the same shape,
    k_scale)."""
    if k_scale is None:
        amax = float(k_cache.float().abs().max()) if k_cache.numel() else 1.0
        k_scale = amax / 448.0 if amax > 0 else 1.0
    codes = (k_cache.float() / k_scale).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, float(k_scale)


def make_prefill(name: str, new_tokens: list[int], prefixes: list[int], seed: int,
                 W: int | None = None) -> PrefillInputs:
    """Packed prefill inputs: sequence s has ``prefixes[s]`` cached tokens and
    ``new_tokens[s]`` query rows; its keys are the compressed keys of all its
    complete 4-token groups, packed one sequence after another."""
    g = _gen(seed)
    S = len(new_tokens)
    total = [p + n for p, n in zip(prefixes, new_tokens)]
    nkeys = [t // TOKENS_PER_KEY for t in total]
    T = sum(new_tokens)
    q = randn_bf16((T, HEADS, DIM), g)
    k = randn_bf16((sum(nkeys), DIM), g)
    cu = [0]
    for n in new_tokens:
        cu.append(cu[-1] + n)
    offs = [0]
    for n in nkeys[:-1]:
        offs.append(offs[-1] + n)
    if W is None:
        W = max(nkeys)
    return PrefillInputs(name=name, q=q, k=k,
                         cu_seqlens_q=torch.tensor(cu, dtype=torch.int32),
                         seq_lens=torch.tensor(total, dtype=torch.int32),
                         key_offsets=torch.tensor(offs, dtype=torch.int32), W=W,
                         meta={"seed": seed, "new_tokens": list(new_tokens),
                               "prefix_tokens": list(prefixes)})


# The five workloads.  Decode lengths: 16 requests, log-normal, min/mean/max as
# in the vLLM PR's multi-request tables (1,536 / 10,240 / 43,876 and
# 3,508 / 51,200 / 102,400 tokens).  "100K" there is 102,400 tokens.
CONFIG_NAMES = {
    1: "decode_b1_q1_ctx2048_ps16",
    2: "decode_b16_q1_ctx1536-43876_ps64",
    3: "specdecode_b16_q4_ctx3508-102400_ps64",
    4: "prefill_t8192_prefix50144",
    5: "prefill_4x4096_prefix102400_top512",
    6: "core_attention_b16_q4_top512_h24x2_d256_ps64",
    7: "mixed_batch_16decode_plus_prefill2048_after30000_ps64",
}
TOPK_K = 512


def attention_block_sets(a: "AttentionInputs", n: int, seed: int) -> list:
    """n more block selections for the rows of ``a`` (the same rule as
    make_attention: k visible blocks per row uniformly without replacement,
    ascending, -1 padded), so that repeated steps gather different tokens."""
    g = _gen(seed)
    cu = a.cu_seqlens_q.tolist()
    sl = a.seq_lens.tolist()
    k = a.blocks.shape[1]
    out = []
    for _ in range(n):
        blocks = torch.full_like(a.blocks, -1)
        for r in range(len(sl)):
            qlen = cu[r + 1] - cu[r]
            for i in range(qlen):
                pos = sl[r] - qlen + i
                vis = max(0, min((pos + 1) // TOKENS_PER_KEY, sl[r] // TOKENS_PER_KEY))
                m = min(k, vis)
                if m:
                    blocks[cu[r] + i, :m] = torch.randperm(vis, generator=g)[:m].sort().values.to(torch.int32)
        out.append(blocks)
    return out


def make_config(idx: int, seed: int = 0, page_size: int | None = None):
    """Workload idx; for the decode workloads 1-3, page_size (if given)
    replaces the workload's page size (the same contexts, a pool of that
    page size)."""
    name = CONFIG_NAMES[idx]
    if page_size is not None:
        if idx not in (1, 2, 3):
            raise ValueError("a page size applies to the decode workloads 1-3")
        name = name.rsplit("_ps", 1)[0] + f"_ps{page_size}"
    if idx == 1:
        return make_decode(name, [2048], Q=1, page_size=page_size or 16, seed=seed)
    if idx == 2:
        ctx = lognormal_contexts(16, 1536, 43876, 16 * 10240, seed)
        return make_decode(name, ctx, Q=1, page_size=page_size or 64, seed=seed)
    if idx == 3:
        ctx = lognormal_contexts(16, 3508, 102400, 16 * 51200, seed)
        return make_decode(name, ctx, Q=4, page_size=page_size or 64, seed=seed)
    if idx == 4:
        return make_prefill(name, [8192], [50144], seed=seed)
    if idx == 5:
        return make_prefill(name, [4096] * 4, [102400] * 4, seed=seed)
    if idx == 6:
        # the core-attention step after workload 3's indexer: the same 16
        # requests and 4 query rows each, top-512 blocks (2,051 tokens per row),
        # 24 query heads over 2 KV heads of dimension 256, 64-token pages
        ctx = lognormal_contexts(16, 3508, 102400, 16 * 51200, seed)
        return make_attention(name, ctx, [4] * 16, 24, 2, 64, TOPK_K, seed=seed)
    if idx == 7:
        # workload 2's 16 decode requests and one prefill request of 2,048 new
        # rows after 30,000 cached tokens, one paged pool (64-row pages)
        ctx = lognormal_contexts(16, 1536, 43876, 16 * 10240, seed)
        return make_paged_batch(name, ctx, 1, [2048], [30000], 64, seed=seed)
    raise KeyError(idx)


@dataclass
class AttentionInputs:
    """Sparse core-attention inputs (all tensors on the CPU): query rows of R
    requests packed by ``cu_seqlens_q``, paged K and V pools, and the selected
    compressed blocks of every row (ascending, -1 padded)."""
    name: str
    q: torch.Tensor            # bf16 [T, Hq, 256]
    k_cache: torch.Tensor      # bf16 [pages, page_size, Hkv, 256]
    v_cache: torch.Tensor      # bf16 [pages, page_size, Hkv, 256]
    page_table: torch.Tensor   # int32 [R, max_pages]
    cu_seqlens_q: torch.Tensor # int32 [R + 1]
    seq_lens: torch.Tensor     # int32 [R]
    blocks: torch.Tensor       # int32 [T, k]
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return self.q.shape[0]


ATTN_DIM = 256     # core attention head dimension (QSA docs, "Core Attention": D256)


def make_attention(name: str, seq_lens: list[int], qlens: list[int], Hq: int, Hkv: int, page_size: int,
                   k: int, seed: int, spare_pages: int = 1) -> AttentionInputs:
    """Paged K/V pools with N(0, 1) bf16 rows (pages handed out by a random
    permutation, -1 past a request's pages), N(0, 1) queries, and for every
    query row k block indices drawn uniformly without replacement from the
    blocks the row can see (fewer when it sees fewer), ascending, -1 padded.
    Row i of request r sits at position seq_lens[r] - qlens[r] + i."""
    g = _gen(seed)
    R = len(seq_lens)
    pages_per_req = [max(1, -(-L // page_size)) for L in seq_lens]
    num_pages = sum(pages_per_req) + spare_pages
    kc = randn_bf16((num_pages, page_size, Hkv, ATTN_DIM), g)
    vc = randn_bf16((num_pages, page_size, Hkv, ATTN_DIM), g)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.full((R, max(pages_per_req)), -1, dtype=torch.int32)
    at = 0
    for r, n in enumerate(pages_per_req):
        table[r, :n] = perm[at:at + n]
        at += n
    T = sum(qlens)
    q = randn_bf16((T, Hq, ATTN_DIM), g)
    blocks = torch.full((T, k), -1, dtype=torch.int32)
    t = 0
    for r in range(R):
        for i in range(qlens[r]):
            pos = seq_lens[r] - qlens[r] + i
            vis = max(0, min((pos + 1) // TOKENS_PER_KEY, seq_lens[r] // TOKENS_PER_KEY))
            n = min(k, vis)
            if n:
                pick = torch.randperm(vis, generator=g)[:n].sort().values.to(torch.int32)
                blocks[t, :n] = pick
            t += 1
    cu = [0]
    for n in qlens:
        cu.append(cu[-1] + n)
    return AttentionInputs(name=name, q=q, k_cache=kc, v_cache=vc, page_table=table,
                           cu_seqlens_q=torch.tensor(cu, dtype=torch.int32),
                           seq_lens=torch.tensor(seq_lens, dtype=torch.int32), blocks=blocks,
                           meta={"seed": seed, "context_tokens": list(seq_lens), "query_rows": list(qlens),
                                 "heads": (Hq, Hkv), "page_size": page_size, "k": k})


@dataclass
class PagedBatchInputs:
    """A mixed batch read from the paged compressed key cache (all tensors on
    the CPU): D decode requests with Q query rows each, then prefill requests
    with their own numbers of new rows; q packed in that order."""
    name: str
    q: torch.Tensor            # bf16 [T, 4, 128]
    k_cache: torch.Tensor      # bf16 [num_pages, page_size, 1, 128]
    page_table: torch.Tensor   # int32 [R, max_pages]
    cu_seqlens_q: torch.Tensor # int32 [R + 1]
    seq_lens: torch.Tensor     # int32 [R]
    num_decodes: int
    decode_query_len: int
    page_size: int
    W: int
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return self.q.shape[0]


def make_paged_batch(name: str, decode_lens: list[int], Q: int, prefill_new: list[int],
                     prefill_prefix: list[int], page_size: int, seed: int, W: int | None = None) -> PagedBatchInputs:
    """Decode requests of the given context lengths (query rows included)
    followed by prefill requests with `prefill_new` rows after
    `prefill_prefix` cached tokens; one paged pool for all of them (pages
    handed out by a random permutation, one spare, -1 past a request's
    pages), N(0, 1) bf16 queries and keys."""
    g = _gen(seed)
    lens = list(decode_lens) + [p + n for p, n in zip(prefill_prefix, prefill_new)]
    qlens = [Q] * len(decode_lens) + list(prefill_new)
    tokens_per_page = TOKENS_PER_KEY * page_size
    pages_per_req = [max(1, -(-L // tokens_per_page)) for L in lens]
    num_pages = sum(pages_per_req) + 1
    k_cache = randn_bf16((num_pages, page_size, 1, DIM), g)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.full((len(lens), max(pages_per_req)), -1, dtype=torch.int32)
    at = 0
    for r, n in enumerate(pages_per_req):
        table[r, :n] = perm[at:at + n]
        at += n
    q = randn_bf16((sum(qlens), HEADS, DIM), g)
    cu = [0]
    for n in qlens:
        cu.append(cu[-1] + n)
    if W is None:
        W = max(lens) // TOKENS_PER_KEY
    return PagedBatchInputs(name=name, q=q, k_cache=k_cache, page_table=table,
                            cu_seqlens_q=torch.tensor(cu, dtype=torch.int32),
                            seq_lens=torch.tensor(lens, dtype=torch.int32), num_decodes=len(decode_lens),
                            decode_query_len=Q, page_size=page_size, W=W,
                            meta={"seed": seed, "context_tokens": lens, "query_rows": qlens})
