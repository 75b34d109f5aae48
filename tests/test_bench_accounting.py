"""The benchmark's throughput accounting reproduces the numbers printed in the
vLLM PR "Separate prefill and decode paths for QSA indexer" (section
"Microbenchmarks"): decode GB/s from the key, score and query bytes, prefill
TFLOP/s from the causal-visible (row, key) pairs."""
import os

import numpy as np

import bench
import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "vllm_qsa_indexer_microbench.txt")


def rows(kind):
    with open(GOLDEN) as f:
        for line in f:
            p = line.split()
            if p and p[0] == kind:
                yield p


def test_decode_bytes_reproduce_printed_gbps():
    n = 0
    for p in rows("decode"):
        dql, nreq, lo, mean, hi = map(int, p[1:6])
        if nreq == 1:
            ctx = [hi]
            exact = True
        else:  # only min / mean / max are printed: lengths that are multiples of 4 with that sum
            ctx = [mean * nreq]
            exact = False
        b = bench.decode_bytes(ctx, dql) + (nreq - 1) * dql * 1024
        for us, printed in ((float(p[6]), float(p[8])), (float(p[7]), float(p[9]))):
            got = b / us / 1e3
            if exact:
                assert round(got) == printed, (p, got)
            else:
                assert abs(got - printed) <= 1.0, (p, got)
            n += 1
    assert n == 28


def test_prefill_flops_reproduce_printed_tflops():
    n = 0
    for p in rows("prefill"):
        S, new = map(int, p[1].split("x"))
        prefix = int(p[2])
        cu = [i * new for i in range(S + 1)]
        ks, ke = oracle.prefill_intervals(cu, [prefix + new] * S, [0] * S)
        flop = bench.prefill_flops(ks, ke)
        for us, printed in ((float(p[3]), float(p[5])), (float(p[4]), float(p[6]))):
            assert round(flop / us / 1e6, 1) == printed, (p, flop / us / 1e6)
            n += 1
    assert n == 24


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1e9, 1e-3, 1, 1e9) == 1000.0
    assert bench.job_throughput(1e9, 1e-3, 4, 1e9) == 4000.0


def test_source_digest_ignores_comments_and_blank_space(tmp_path, monkeypatch):
    """The DRAM-traffic rows are keyed by bench.source_hash(): a comment or
    blank-space edit must keep the key, a code edit must change it."""
    import shutil
    root = tmp_path / "repo"
    src = root / "sparse_attention_block_qsa_b200" / "csrc"
    shutil.copytree(os.path.join(bench.ROOT, "sparse_attention_block_qsa_b200", "csrc"), src)
    monkeypatch.setattr(bench, "ROOT", str(root))
    base = bench.source_hash()
    f = src / "decode.cuh"
    text = f.read_text()
    f.write_text(text.replace("#pragma once", "// a new comment\n/* and a block\n   comment */\n\n#pragma   once", 1))
    assert bench.source_hash() == base
    f.write_text(text.replace("constexpr int BATCH = 4;", "constexpr int BATCH = 2;", 1))
    assert bench.source_hash() != base


def test_fp8_decode_bytes_count_one_byte_per_key_element():
    ctx = [1536, 10240, 43876, 7]
    keys = sum(L // 4 for L in ctx)
    for dql in (1, 4):
        bf16 = bench.decode_bytes(ctx, dql)
        fp8 = bench.decode_bytes(ctx, dql, 128)
        assert bf16 - fp8 == keys * 128
        assert fp8 == keys * 128 + dql * keys * 4 + len(ctx) * dql * 1024
