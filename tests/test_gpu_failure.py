"""Failure handling on the GPU without a fault: a device-side wait that never
completes must end after its limit, set the library's device error word and
leave the context usable (the kernels' waits are all bounded this way)."""
import time

import pytest
import torch

import oracle
import sparse_attention_block_qsa_b200 as qsa
import workloads as wl
from parity import compare_scores, decode_bounds

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
WAIT_TIMEOUT_BIT = 0x1   # QSA_DEVERR_WAIT_TIMEOUT


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    qsa.device_error()                                   # start from a clear word
    t0 = time.perf_counter()
    qsa.selftest_bounded_wait(20_000_000, arrive=False)  # 20 ms on a phase nothing completes
    bits = qsa.device_error()                            # synchronises
    elapsed = time.perf_counter() - t0
    assert bits & WAIT_TIMEOUT_BIT
    assert elapsed >= 0.02
    # the same context still runs the hot path correctly
    d = wl.make_decode("after_timeout", [517, 2048, 61], Q=2, page_size=16, seed=3)
    out = qsa.mqa_decode(d.q.to(DEV), d.k_cache.to(DEV), d.page_table.to(DEV), d.seq_lens.to(DEV), d.W)
    ref = oracle.decode(d.q, d.k_cache, d.page_table, d.seq_lens, d.W, scale=qsa.SCALE)
    loose, tight = decode_bounds(d.q, d.k_cache, d.page_table, d.W, qsa.SCALE)
    compare_scores(out.cpu().numpy(), ref, loose, tight)
    assert qsa.device_error() == 0


def test_bounded_wait_that_completes_sets_nothing():
    qsa.device_error()
    qsa.selftest_bounded_wait(20_000_000, arrive=True)
    assert qsa.device_error() == 0
