"""Benchmark of the QSA MQA indexer score on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..5] [--impl ours|reference]

One step = one pass of the indexer over one batch of a workload.  By default
all five workloads are timed one after another and printed as ONE JSON line:
the headline is the long-context speculative decode (16 requests, 4 query
tokens each, log-normal contexts of 3,508-102,400 tokens, page size 64), the
workload whose HBM roofline fraction is the decode target; the other four
(single-request decode, 16-request decode, the 8,192-row prefill, the
4 x 4,096-row prefill with top-512, and the core-attention step that follows
the long-context decode: block -> token expansion and sparse attention over
2,051 selected tokens per row) are records under "configs", each with its
own roofline, clocks, end-to-end and CPU-baseline figures.  `--config c`
times one workload only.

For each workload the K timed steps are captured in one CUDA graph and
replayed between CUDA events on the launching stream, after W untimed
warm-up steps; decode steps rotate over enough copies of the inputs that
their total exceeds twice the 126 MB L2, and prefill steps write more than
L2 of scores, so every step reads and writes HBM.

Throughput accounting follows the vLLM PR "Separate prefill and decode
paths for QSA indexer" (section "Microbenchmarks"), whose printed numbers
these formulas reproduce (tests/test_bench_accounting.py):
  decode bytes  = sum_b [(ctx_b // 4) * 256 + DQL * (ctx_b // 4) * 4] + B * DQL * 1024
  prefill FLOPs = 2 * 4 * 128 * sum_t visible(t)

With --gpus N each of N ranks (started by torchrun, or by this script when
no launcher set WORLD_SIZE) runs its own replica of the workload (weak
scaling: the indexer needs no exchange between GPUs); the step time is the
maximum over ranks and the value counts the work of all ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "indexer µs and GB/s (decode) / TFLOP/s (prefill) and % of roofline, 1×B200"
L2_BYTES = 126 * 1024 * 1024
PUBLISHED = {  # the vLLM PR's GB300 numbers for the same workload shapes (context only)
    2: ("GB/s", 1302.0, "vLLM PR microbenchmarks, DQL 1, 16 requests, 1,536/10,240/43,876 tokens, GB300, ps 196"),
    3: ("GB/s", 3374.0, "vLLM PR microbenchmarks, DQL 4, 16 requests, 3,508/51,200/102,400 tokens, GB300, ps 196"),
}


# ------------------------------------------------------------------ accounting

def decode_bytes(seq_lens, dql: int, key_bytes: int = 256) -> int:
    """Algorithmic bytes of one decode step: the visible keys (256 bytes each
    in bf16, 128 in fp8), the fp32 scores of the visible blocks and the bf16
    queries."""
    keys = sum(int(L) // 4 for L in seq_lens)
    return keys * key_bytes + dql * keys * 4 + len(seq_lens) * dql * 1024


def prefill_flops(ks, ke) -> int:
    """2 * 4 heads * 128 features per (row, visible key) pair."""
    return 2 * 4 * 128 * int(np.sum(np.asarray(ke, dtype=np.int64) - np.asarray(ks, dtype=np.int64)))


def read_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# The device sources of each timed kernel (its own header and the shared
# sm_100a helpers).
KERNEL_SOURCES = {
    "decode_kernel": ["decode.cuh", "sm100.cuh"],
    "prefill_kernel": ["prefill.cuh", "sm100.cuh"],
    "topk_pipe_kernel": ["topk.cuh", "sm100.cuh"],
    "topk_filter_kernel": ["topk.cuh", "sm100.cuh"],
    "attn_kernel": ["attention.cuh", "sm100.cuh"],
}


def source_hash(kernel: str | None = None) -> str:
    """Digest of a kernel's device sources (every file of csrc/ when kernel is
    None) with comments and blank space removed, so that it changes exactly
    when that code does."""
    import hashlib
    import re
    src = os.path.join(ROOT, "sparse_attention_block_qsa_b200", "csrc")
    h = hashlib.sha256()
    files = KERNEL_SOURCES.get(kernel) if kernel else None
    for f in sorted(files or os.listdir(src)):
        with open(os.path.join(src, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(f.encode())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:12]


def read_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.md")
    if not os.path.exists(path):
        return None
    sha = source_hash(kernel)
    for line in open(path):
        parts = [p.strip() for p in line.strip().strip("|").split("|")]
        if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload and parts[2] == sha:
            try:
                return int(parts[3])
            except ValueError:
                return None
    return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workloads

class DecodeBench:
    """Decode / spec-decode step: one qsa_mqa_decode launch over one batch."""
    kernel = "decode_kernel"
    bound = "hbm"

    def __init__(self, cfg: int, dev: torch.device, seed: int, fp8: bool = False, page_size: int | None = None,
                 f16: bool = False):
        import sparse_attention_block_qsa_b200 as qsa
        self.qsa = qsa
        self.inp = wl.make_config(cfg, seed=seed, page_size=page_size)
        d = self.inp
        self.fp8 = fp8
        self.k_scale = 1.0
        if fp8:   # the same keys in the fp8 E4M3 cache format
            d.k_cache, self.k_scale = wl.e4m3_cache(d.k_cache)
        if f16:   # the same values as fp16 queries and keys
            d.q, d.k_cache = d.q.to(torch.float16), d.k_cache.to(torch.float16)
        kb = d.k_cache.element_size()
        self.name = d.name + ("_fp8" if fp8 else "") + ("_f16" if f16 else "")
        self.units = decode_bytes(d.seq_lens.tolist(), d.Q, 128 * kb)   # algorithmic bytes per step
        per_copy = d.q.numel() * 2 + d.k_cache.numel() * kb + d.B * d.Q * d.W * 4
        self.copies = max(2, math.ceil(2 * L2_BYTES / per_copy))
        self.dev = dev
        # Timed steps rotate over copies of the key pool and the output (more
        # than twice L2), so keys come from HBM; the queries, lengths and page
        # table are one copy, as in a model step where the previous kernel has
        # just written the queries and every layer reads the same metadata.
        # step_cold rotates every input instead (all of them from HBM).
        self.shared = (d.q.to(dev), d.page_table.to(dev), d.seq_lens.to(dev))
        self.bufs = []
        for _ in range(self.copies):
            self.bufs.append((d.q.to(dev), d.k_cache.to(dev), d.page_table.to(dev), d.seq_lens.to(dev),
                              torch.empty((d.B, d.Q, d.W), dtype=torch.float32, device=dev)))
        self.launches_per_step = 1
        self.h2d = d.q.numel() * 2 + d.k_cache.numel() * kb + (d.page_table.numel() + d.seq_lens.numel()) * 4
        self.d2h = d.B * d.Q * d.W * 4
        self.dtype = "fp8e4m3 keys, bf16 queries" if fp8 else ("f16" if f16 else "bf16")
        self.config = {"workload": self.name, "kv_cache_dtype": "fp8_e4m3" if fp8 else ("fp16" if f16 else "bf16"),
                       "requests": d.B, "query_tokens": d.Q, "page_size": d.page_size,
                       "context_tokens": d.meta["context_tokens"], "W": d.W, "input_copies": self.copies,
                       "l2": f"steps rotate over {self.copies} copies of the key pool and output "
                             f"({self.copies * per_copy / 2**20:.0f} MiB > 2x L2); queries, lengths and page "
                             f"table shared by the steps (L2-resident, as across a model's layers); "
                             f"all_inputs_cold_us rotates every input"}

    def _launch(self, q, kc, pt, sl, out):
        if self.fp8:
            self.qsa.mqa_decode_fp8(q, kc, self.k_scale, pt, sl, self.inp.W, out=out)
        else:
            self.qsa.mqa_decode(q, kc, pt, sl, self.inp.W, out=out)

    def step(self, i: int):
        q, pt, sl = self.shared
        _, kc, _, _, out = self.bufs[i % self.copies]
        self._launch(q, kc, pt, sl, out)

    def step_cold(self, i: int):
        self._launch(*self.bufs[i % self.copies])

    def throughput(self, seconds_per_step: float) -> float:
        return self.units / seconds_per_step / 1e9   # GB/s

    unit = "GB/s"

    def e2e_setup(self):
        d = self.inp
        self.host = [t.pin_memory() for t in (d.q, d.k_cache, d.page_table, d.seq_lens)]
        self.host_out = torch.empty((d.B, d.Q, d.W), dtype=torch.float32).pin_memory()

    def e2e_step(self, i: int):
        q, kc, pt, sl, out = self.bufs[i % self.copies]
        for dst, src in zip((q, kc, pt, sl), self.host):
            dst.copy_(src, non_blocking=True)
        self._launch(q, kc, pt, sl, out)
        self.host_out.copy_(out, non_blocking=True)

    def oracle_step(self, threads: int = 0):
        import oracle
        d = self.inp
        if self.fp8:
            oracle.decode_fp8(d.q, d.k_cache, self.k_scale, d.page_table, d.seq_lens, d.W, threads=threads)
        else:
            oracle.decode(d.q, d.k_cache, d.page_table, d.seq_lens, d.W, threads=threads)

    def oracle_sample(self):
        return 1.0, "one full step (every score of the batch)"


class PrefillBench:
    """Prefill step: qsa_mqa_prefill (configuration 4) or the fused prefill
    + top-512 (configuration 5) over one packed batch."""
    kernel = "prefill_kernel"
    bound = "tensor"
    unit = "TFLOP/s"

    def __init__(self, cfg: int, dev: torch.device, seed: int, f16: bool = False):
        import sparse_attention_block_qsa_b200 as qsa
        self.qsa = qsa
        self.cfg = cfg
        self.inp = p = wl.make_config(cfg, seed=seed)
        if f16:   # the same values as fp16 queries and keys
            p.q, p.k = p.q.to(torch.float16), p.k.to(torch.float16)
        self.f16 = f16
        self.dtype = "f16" if f16 else "bf16"
        self.name = p.name + ("_f16" if f16 else "")
        self.dev = dev
        self.q, self.k = p.q.to(dev), p.k.to(dev)
        self.cu, self.sl, self.ko = p.cu_seqlens_q.to(dev), p.seq_lens.to(dev), p.key_offsets.to(dev)
        self.ks, self.ke = qsa.prefill_intervals(self.cu, self.sl, self.ko, p.T)
        ks_h, ke_h = self.ks.cpu().numpy(), self.ke.cpu().numpy()
        self.units = prefill_flops(ks_h, ke_h)
        self.topk = cfg == 5
        self.out = torch.empty((p.T, p.W), dtype=torch.float32, device=dev)
        if self.topk:
            self.idx = torch.empty((p.T, wl.TOPK_K), dtype=torch.int32, device=dev)
            # the top-k step through qsa_topk_ws: filter, list and exact-pass launches
            self.topk_ws = torch.empty(qsa.topk_workspace_size(p.T, p.W, wl.TOPK_K), dtype=torch.uint8, device=dev)
        self.copies = 1
        self.launches_per_step = 4 if self.topk else 1
        out_bytes = p.T * p.W * 4
        self.h2d = (p.q.numel() + p.k.numel()) * 2 + (p.cu_seqlens_q.numel() + 2 * p.seq_lens.numel()) * 4
        self.d2h = p.T * wl.TOPK_K * 4 if self.topk else out_bytes
        self.config = {"workload": self.name, "sequences": len(p.meta["new_tokens"]),
                       "new_tokens": p.meta["new_tokens"], "prefix_tokens": p.meta["prefix_tokens"],
                       "keys": p.Nk, "W": p.W, "flop_per_step": self.units,
                       "l2": f"each step writes {out_bytes / 2**20:.0f} MiB of scores (> L2)"}
        if self.topk:
            self.config["topk"] = wl.TOPK_K

    def step(self, i: int, mid_event=None):
        p = self.inp
        self.qsa.mqa_prefill(self.q, self.k, self.ks, self.ke, p.W, out=self.out)
        if self.topk:
            if mid_event is not None:
                mid_event.record()
            self.qsa.topk(self.out, wl.TOPK_K, idx=self.idx, workspace=self.topk_ws)

    def throughput(self, seconds_per_step: float) -> float:
        return self.units / seconds_per_step / 1e12

    def topk_bytes(self) -> int:
        """Algorithmic bytes of the top-k step: every score read once, every
        index written once."""
        p = self.inp
        return p.T * p.W * 4 + p.T * wl.TOPK_K * 4

    def time_fused(self, workspace_mib: int = 64, reps: int = 10):
        """qsa_mqa_prefill_topk through a workspace of about `workspace_mib`
        MiB (scores of a chunk of rows stay in the 126 MB L2 between the two
        kernels): median seconds per step over `reps`, CUDA events."""
        if not self.topk:
            return None
        p = self.inp
        ws = torch.empty(workspace_mib * 2**20 // 4, dtype=torch.float32, device=self.dev)
        run = lambda: self.qsa.mqa_prefill_topk(self.q, self.k, self.ks, self.ke, p.W, wl.TOPK_K, ws, idx=self.idx)
        for _ in range(3):
            run()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, e in ev:
            a.record()
            run()
            e.record()
        torch.cuda.synchronize()
        t = statistics.median(a.elapsed_time(e) for a, e in ev) / 1e3
        rows = ((workspace_mib * 2**20 - 4096) // (p.W * 4)) // 64 * 64
        return {"us_per_step": t * 1e6, "workspace_mib": workspace_mib, "rows_per_chunk": int(rows),
                "launches_per_step": 2 * -(-p.T // rows), "tflops": self.units / t / 1e12}

    def e2e_setup(self):
        p = self.inp
        self.host = [t.pin_memory() for t in (p.q, p.k, p.cu_seqlens_q, p.seq_lens, p.key_offsets)]
        shape = (p.T, wl.TOPK_K) if self.topk else (p.T, p.W)
        self.host_out = torch.empty(shape, dtype=torch.int32 if self.topk else torch.float32).pin_memory()

    def e2e_step(self, i: int):
        p = self.inp
        for dst, src in zip((self.q, self.k, self.cu, self.sl, self.ko), self.host):
            dst.copy_(src, non_blocking=True)
        self.qsa.prefill_intervals(self.cu, self.sl, self.ko, p.T, ks=self.ks, ke=self.ke)
        self.step(i)
        self.host_out.copy_(self.idx if self.topk else self.out, non_blocking=True)

    def oracle_sample(self):
        return 64 / self.inp.T, "64 query rows of the batch, every column (scaled to the full batch)"

    def oracle_step(self, threads: int = 0):
        import oracle
        p = self.inp
        ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
        rows = slice(0, 64)
        s = oracle.prefill(p.q[rows], p.k, ks[rows], ke[rows], p.W, threads=threads)
        if self.topk:
            oracle.topk(s, np.full(s.shape[0], p.W, dtype=np.int32), wl.TOPK_K, threads=threads)


class AttentionBench:
    """Core-attention step after the indexer: block -> token expansion and
    split-KV sparse attention (three launches) over one batch of selected
    blocks; steps rotate over several selections so that they gather
    different tokens from the 1.7 GB K/V pool."""
    kernel = "attn_kernel"
    bound = "hbm"
    unit = "GB/s"

    def __init__(self, cfg: int, dev: torch.device, seed: int):
        import sparse_attention_block_qsa_b200 as qsa
        self.qsa = qsa
        self.inp = a = wl.make_config(cfg, seed=seed)
        self.name = a.name
        self.dev = dev
        self.sets = [a.blocks] + wl.attention_block_sets(a, 3, seed + 1000)
        self.copies = len(self.sets)
        self.q = a.q.to(dev)
        self.kc, self.vc = a.k_cache.to(dev), a.v_cache.to(dev)
        self.pt, self.cu, self.sl = a.page_table.to(dev), a.cu_seqlens_q.to(dev), a.seq_lens.to(dev)
        self.blocks = [b.to(dev) for b in self.sets]
        k = a.blocks.shape[1]
        self.tok = torch.empty((a.T, 4 * k + 3), dtype=torch.int32, device=dev)
        Hq, Hkv = a.q.shape[1], a.k_cache.shape[2]
        self.out = torch.empty((a.T, Hq, 256), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((a.T, Hq), dtype=torch.float32, device=dev)
        ws = qsa.sparse_attention_workspace_size(a.T, Hq, Hkv, 4 * k + 3)
        self.ws = torch.empty(ws // 4 + 4, dtype=torch.float32, device=dev)
        self.units, self.flops, self.tokens = self._accounting(a, Hq, Hkv)
        self.launches_per_step = 3
        self.h2d = a.q.numel() * 2 + a.blocks.numel() * 4 + (a.cu_seqlens_q.numel() + a.seq_lens.numel()) * 4
        self.d2h = self.out.numel() * 2 + self.lse.numel() * 4
        self.dtype = "bf16"
        self.config = {"workload": a.name, "requests": len(a.meta["context_tokens"]),
                       "query_rows": a.meta["query_rows"], "heads_q_kv": list(a.meta["heads"]), "head_dim": 256,
                       "page_size": a.meta["page_size"], "blocks_per_row": k, "tokens_per_row": 4 * k + 3,
                       "context_tokens": a.meta["context_tokens"],
                       "kv_pool_bytes": a.k_cache.numel() * 4, "bytes_per_step": self.units,
                       "flop_per_step": self.flops,
                       "l2": f"steps rotate over {self.copies} block selections; each gathers "
                             f"{self.units / 2**20:.0f} MiB of K/V rows from a "
                             f"{a.k_cache.numel() * 4 / 2**30:.1f} GiB pool",
                       "e2e_inputs": "q, selected blocks and request metadata copied in each step; "
                                     "the paged K/V cache is resident model state"}

    @staticmethod
    def _accounting(a, Hq, Hkv):
        """Algorithmic bytes: the distinct K and V rows a request's rows
        select (each read once), the queries, the bf16 outputs and the LSE.
        FLOPs: 4 * 256 per (row, query head, visible token)."""
        cu = a.cu_seqlens_q.tolist()
        sl = a.seq_lens.tolist()
        blocks = a.blocks.numpy()
        uniq = 0
        vis_tokens = 0
        for r in range(len(sl)):
            toks = set()
            qlen = cu[r + 1] - cu[r]
            for i in range(qlen):
                t = cu[r] + i
                pos = sl[r] - qlen + i
                v = max(0, min((pos + 1) // 4, sl[r] // 4))
                row = {4 * int(b) + j for b in blocks[t] if b >= 0 for j in range(4)}
                row |= set(range(4 * v, pos + 1))
                toks |= row
                vis_tokens += len(row)
            uniq += len(toks)
        T = a.T
        bytes_ = uniq * Hkv * 2 * 512 + T * Hq * 256 * 2 * 2 + T * Hq * 4
        return bytes_, 4 * Hq * 256 * vis_tokens, vis_tokens

    def _launch(self, blocks):
        self.qsa.expand_block_indices(blocks, self.cu, self.sl, token_idx=self.tok)
        self.qsa.sparse_attention(self.q, self.kc, self.vc, self.pt, self.cu, self.sl, self.tok, 1.0 / 16.0,
                                  out=self.out, lse=self.lse, workspace=self.ws)

    def step(self, i: int):
        self._launch(self.blocks[i % self.copies])

    def throughput(self, seconds_per_step: float) -> float:
        return self.units / seconds_per_step / 1e9

    def e2e_setup(self):
        a = self.inp
        self.host = [t.pin_memory() for t in (a.q, a.cu_seqlens_q, a.seq_lens)]
        self.host_blocks = [b.pin_memory() for b in self.sets]
        self.host_out = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
        self.host_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()

    def e2e_step(self, i: int):
        for dst, src in zip((self.q, self.cu, self.sl), self.host):
            dst.copy_(src, non_blocking=True)
        b = self.blocks[i % self.copies]
        b.copy_(self.host_blocks[i % self.copies], non_blocking=True)
        self._launch(b)
        self.host_out.copy_(self.out, non_blocking=True)
        self.host_lse.copy_(self.lse, non_blocking=True)

    def oracle_sample(self):
        return 8 / self.inp.T, "8 query rows (two requests), all 24 heads (scaled to the full batch)"

    def oracle_step(self, threads: int = 0):
        import oracle
        a = self.inp
        rows = slice(0, 8)
        cu = a.cu_seqlens_q.tolist()
        sl = a.seq_lens.tolist()
        req, pos, ln = [], [], []
        for r in range(2):
            qlen = cu[r + 1] - cu[r]
            for i in range(qlen):
                req.append(r)
                pos.append(oracle.logical_position(sl[r], qlen, i))
                ln.append(sl[r])
        tok = oracle.expand_indices(a.blocks[rows].numpy(), pos, ln)
        oracle.sparse_attention(a.q[rows], a.k_cache, a.v_cache, a.page_table, req, pos, a.seq_lens, tok,
                                scale=1.0 / 16.0, threads=threads)


class MixedBench:
    """A mixed decode + prefill batch from the paged cache in one
    qsa_mqa_paged_batch call (decode kernel, metadata kernel, prefill kernel,
    fix-up: four launches chained with programmatic dependent launches)."""
    kernel = "prefill_kernel"
    bound = "hbm+tensor"
    unit = "us"

    def __init__(self, cfg: int, dev: torch.device, seed: int):
        import sparse_attention_block_qsa_b200 as qsa
        self.qsa = qsa
        self.inp = b = wl.make_config(cfg, seed=seed)
        self.name = b.name
        self.dev = dev
        D, Q = b.num_decodes, b.decode_query_len
        sl = b.seq_lens.tolist()
        cu = b.cu_seqlens_q.tolist()
        self.dec_bytes, self.pre_flops = self.accounting(b)
        ws = qsa.paged_batch_workspace_size(len(sl), D, Q, b.T, b.W)
        per_copy = b.q.numel() * 2 + b.k_cache.numel() * 2 + b.T * b.W * 4
        self.copies = max(2, math.ceil(2 * L2_BYTES / per_copy))
        self.bufs = [(b.q.to(dev), b.k_cache.to(dev), b.page_table.to(dev), b.cu_seqlens_q.to(dev),
                      b.seq_lens.to(dev), torch.empty((b.T, b.W), dtype=torch.float32, device=dev),
                      torch.empty(ws // 4 + 4, dtype=torch.float32, device=dev)) for _ in range(self.copies)]
        self.units = 1.0
        self.launches_per_step = 4
        self.h2d = (b.q.numel() + b.k_cache.numel()) * 2 + (b.page_table.numel() + len(sl) + len(cu)) * 4
        self.d2h = b.T * b.W * 4
        self.dtype = "bf16"
        self.config = {"workload": b.name, "decode_requests": D, "decode_query_len": Q,
                       "prefill_rows": b.T - D * Q, "context_tokens": sl, "page_size": b.page_size, "W": b.W,
                       "decode_bytes": self.dec_bytes, "prefill_flop": self.pre_flops, "input_copies": self.copies,
                       "l2": f"steps rotate over {self.copies} input copies "
                             f"({self.copies * per_copy / 2**20:.0f} MiB > 2x L2)"}

    @staticmethod
    def accounting(b):
        """Decode bytes of the decode requests (the vLLM PR's formula) and
        prefill FLOPs of the prefill rows (2 * 4 * 128 per visible key, the
        row at position p seeing min((p + 1) // 4, L // 4) keys)."""
        D, Q = b.num_decodes, b.decode_query_len
        sl = b.seq_lens.tolist()
        cu = b.cu_seqlens_q.tolist()
        vis = 0
        for r in range(D, len(sl)):
            qlen = cu[r + 1] - cu[r]
            for i in range(qlen):
                pos = sl[r] - qlen + i
                vis += max(0, min((pos + 1) // 4, sl[r] // 4, b.W))
        return decode_bytes(sl[:D], Q), 2 * 4 * 128 * vis

    def _launch(self, q, kc, pt, cu, sl, out, ws):
        b = self.inp
        self.qsa.mqa_paged_batch(q, kc, pt, cu, sl, b.num_decodes, b.decode_query_len, b.W, out=out, workspace=ws)

    def step(self, i: int):
        self._launch(*self.bufs[i % self.copies])

    def throughput(self, seconds_per_step: float) -> float:
        return seconds_per_step * 1e6

    def roofline(self, seconds_per_step: float, peaks: dict) -> dict:
        """The step against the sum of its parts' roofline times: the decode
        bytes at the HBM copy bandwidth, plus the prefill rows' bound, the
        larger of their FLOPs at the bf16 peak and their fp32 score rows
        (W columns each) at the HBM bandwidth."""
        b = self.inp
        pre_rows = b.T - b.num_decodes * b.decode_query_len
        pre = max(self.pre_flops / (peaks["bf16_tflops"] * 1e12), pre_rows * b.W * 4 / (peaks["hbm_gbs"] * 1e9))
        ideal = self.dec_bytes / (peaks["hbm_gbs"] * 1e9) + pre
        return {"bound": self.bound, "ideal_us": ideal * 1e6, "achieved_us": seconds_per_step * 1e6,
                "frac": ideal / seconds_per_step, "unit": "us", "traffic": None,
                "peak": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"]},
                "peak_source": peaks["source"]}

    def e2e_setup(self):
        b = self.inp
        self.host = [t.pin_memory() for t in (b.q, b.k_cache, b.page_table, b.cu_seqlens_q, b.seq_lens)]
        self.host_out = torch.empty((b.T, b.W), dtype=torch.float32).pin_memory()

    def e2e_step(self, i: int):
        bufs = self.bufs[i % self.copies]
        for dst, src in zip(bufs[:5], self.host):
            dst.copy_(src, non_blocking=True)
        self._launch(*bufs)
        self.host_out.copy_(bufs[5], non_blocking=True)

    def oracle_sample(self):
        b = self.inp
        return 64 / b.T, "the 16 decode rows and 48 prefill rows, every column (scaled to the full batch by rows)"

    def oracle_step(self, threads: int = 0):
        import oracle
        b = self.inp
        D, Q = b.num_decodes, b.decode_query_len
        oracle.decode(b.q[:D * Q].reshape(D, Q, 4, 128), b.k_cache, b.page_table[:D], b.seq_lens[:D], b.W,
                      threads=threads)
        r = D
        first = int(b.cu_seqlens_q[r])
        n = int(b.cu_seqlens_q[r + 1]) - first
        rows = b.q[first + n - 48:first + n].reshape(1, 48, 4, 128)
        # the last 48 rows of the prefill request: a request cut to those rows
        cut = b.seq_lens[r:r + 1].clone()
        oracle.decode(rows, b.k_cache, b.page_table[r:r + 1], cut, b.W, threads=threads)


def make_bench(cfg: int, dev, seed: int, fp8: bool = False, page_size: int | None = None, f16: bool = False):
    if fp8 and cfg not in (1, 2, 3):
        raise ValueError("the fp8 key cache applies to the decode configurations 1-3")
    if page_size is not None and cfg not in (1, 2, 3):
        raise ValueError("--page-size applies to the decode configurations 1-3")
    if f16 and cfg not in (1, 2, 3, 4):
        raise ValueError("--f16 applies to the decode configurations 1-3 and the prefill configuration 4")
    if cfg in (1, 2, 3):
        return DecodeBench(cfg, dev, seed, fp8, page_size, f16)
    if cfg == 6:
        return AttentionBench(cfg, dev, seed)
    if cfg == 7:
        return MixedBench(cfg, dev, seed)
    return PrefillBench(cfg, dev, seed, f16)


# ------------------------------------------------------------------ timing

def sync_all(world: int):
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over the ranks (step times are reported as the slowest rank's)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step: float, seconds_per_step: float, world: int, scale: float) -> float:
    """Whole-job throughput: every rank processes its own batch of `units_per_step`."""
    return units_per_step * world / seconds_per_step / scale


def time_graph(b, steps: int, world: int, soak_s: float = 0.0, sampler: ClockSampler | None = None):
    """Capture `steps` steps in one graph; return (seconds per step, seconds
    per step of the dominant kernel, clocks)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(steps):
                b.step(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
    t_end = time.time() + soak_s
    while time.time() < t_end:
        g.replay()
        torch.cuda.synchronize()
    sync_all(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    g.replay()
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler is not None else None
    sync_all(world)
    elapsed = start.elapsed_time(end) / 1e3
    del g
    return elapsed / steps, clocks


def time_kernel_split(b, reps: int = 10):
    """For a two-kernel step: per-kernel seconds (prefill, top-k), events
    around each kernel on the launching stream."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, m, e in ev:
        a.record()
        b.step(0, mid_event=m)
        e.record()
    torch.cuda.synchronize()
    pre = statistics.median(a.elapsed_time(m) for a, m, _ in ev) / 1e3
    top = statistics.median(m.elapsed_time(e) for _, m, e in ev) / 1e3
    return pre, top


def time_e2e(b, steps: int, warmup: int, world: int):
    b.e2e_setup()
    for i in range(warmup):
        b.e2e_step(i)
    sync_all(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        b.e2e_step(i)
    end.record()
    torch.cuda.synchronize()
    sync_all(world)
    return start.elapsed_time(end) / 1e3 / steps


def cpu_baseline(b, budget_s: float = 10.0) -> dict:
    import oracle
    threads = oracle.default_threads()
    frac, what = b.oracle_sample()
    b.oracle_step(threads)          # builds / loads the oracle, warms caches
    n, t0 = 0, time.perf_counter()
    while True:
        b.oracle_step(threads)
        n += 1
        if time.perf_counter() - t0 >= budget_s or n >= 100000:
            break
    per_sample = (time.perf_counter() - t0) / n
    per_step = per_sample / frac
    return {"value": b.throughput(per_step), "unit": b.unit, "cores": threads, "kind": "oracle",
            "sample": f"{what}; {n} repetitions, {per_sample:.3f} s each, fp64 C oracle on {threads} host threads",
            "seconds_per_step": per_step}


# ------------------------------------------------------------------ main

HEADLINE = 3            # the long-context spec-decode workload: the decode roofline target
ALL_CONFIGS = [3, 1, 2, 4, 5, 6, 7]


def run_reference(args, rank: int, world: int):
    """The oracle as the reference arm, timed on the host cores."""
    if rank != 0:
        return
    import oracle
    inp_bench = _HostOnly(args.config or HEADLINE, args.kv_fp8, args.page_size, args.f16)
    threads = oracle.default_threads()
    frac, what = inp_bench.oracle_sample()
    for _ in range(args.warmup):
        inp_bench.oracle_step(threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        inp_bench.oracle_step(threads)
    per_sample = (time.perf_counter() - t0) / args.steps
    per_step = per_sample / frac
    value = inp_bench.throughput(per_step)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": inp_bench.unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": inp_bench.unit != "us", "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": inp_bench.config,
            "cpu_baseline": {"value": value, "unit": inp_bench.unit, "cores": threads, "kind": "oracle",
                             "sample": f"{what}; fp64 C oracle on {threads} host threads"},
            "e2e": {"value": value, "unit": inp_bench.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class _HostOnly:
    """Inputs and accounting of a workload without any GPU state."""

    def __init__(self, cfg: int, fp8: bool = False, page_size: int | None = None, f16: bool = False):
        self.cfg = cfg
        self.inp = wl.make_config(cfg, page_size=page_size if cfg in (1, 2, 3) else None)
        self.fp8 = fp8 and cfg in (1, 2, 3)
        self.f16 = f16 and cfg in (1, 2, 3, 4)
        self.k_scale = 1.0
        if cfg == 7:
            self.unit = "us"
            self.config = {"workload": self.inp.name, "W": self.inp.W}
        elif cfg == 6:
            a = self.inp
            self.units, _, _ = AttentionBench._accounting(a, a.q.shape[1], a.k_cache.shape[2])
            self.unit = "GB/s"
            self.config = {"workload": a.name, "query_rows": a.meta["query_rows"], "blocks_per_row": a.blocks.shape[1]}
        elif cfg in (1, 2, 3):
            d = self.inp
            if self.fp8:
                d.k_cache, self.k_scale = wl.e4m3_cache(d.k_cache)
            if self.f16:
                d.q, d.k_cache = d.q.to(torch.float16), d.k_cache.to(torch.float16)
            self.units = decode_bytes(d.seq_lens.tolist(), d.Q, 128 * d.k_cache.element_size())
            self.unit = "GB/s"
            self.config = {"workload": d.name + ("_fp8" if self.fp8 else "") + ("_f16" if self.f16 else ""),
                           "kv_cache_dtype": "fp8_e4m3" if self.fp8 else ("fp16" if self.f16 else "bf16"),
                           "requests": d.B, "query_tokens": d.Q, "page_size": d.page_size, "W": d.W}
        else:
            import oracle
            p = self.inp
            if self.f16:
                p.q, p.k = p.q.to(torch.float16), p.k.to(torch.float16)
            ks, ke = oracle.prefill_intervals(p.cu_seqlens_q, p.seq_lens, p.key_offsets)
            self.units = prefill_flops(ks, ke)
            self.unit = "TFLOP/s"
            self.topk = cfg == 5
            self.config = {"workload": p.name + ("_f16" if self.f16 else ""), "keys": p.Nk, "W": p.W}

    def throughput(self, s):
        if self.unit == "us":
            return s * 1e6
        return self.units / s / (1e9 if self.unit == "GB/s" else 1e12)

    def oracle_sample(self):
        if self.cfg == 7:
            return MixedBench.oracle_sample(self)
        if self.cfg == 6:
            return AttentionBench.oracle_sample(self)
        if self.cfg in (1, 2, 3):
            return 1.0, "one full step (every score of the batch)"
        return 64 / self.inp.T, "64 query rows of the batch, every column (scaled to the full batch)"

    def oracle_step(self, threads):
        if self.cfg == 7:
            MixedBench.oracle_step(self, threads)
        elif self.cfg == 6:
            AttentionBench.oracle_step(self, threads)
        elif self.cfg in (1, 2, 3):
            DecodeBench.oracle_step(self, threads)
        else:
            PrefillBench.oracle_step(self, threads)


def measure(cfg: int, args, world: int, rank: int, local: int, cpu_budget_s: float) -> dict | None:
    """Time one workload: W eager warm-up steps, then K steps in one CUDA
    graph between CUDA events (max over ranks); the same steps end to end
    through the public binding; the oracle on the host cores (rank 0, N = 1).
    Returns rank 0's record (None on the other ranks)."""
    dev = torch.device("cuda", local)
    b = make_bench(cfg, dev, seed=rank, fp8=args.kv_fp8 and cfg in (1, 2, 3),
                   page_size=args.page_size if cfg in (1, 2, 3) else None,
                   f16=args.f16 and cfg in (1, 2, 3, 4))
    for i in range(args.warmup):
        b.step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    per_step, clocks = time_graph(b, args.steps, world, soak_s=args.soak, sampler=sampler)
    per_step = max_over_ranks(per_step, world)
    kernel_s = per_step
    extra = {}
    if hasattr(b, "step_cold"):
        class _Cold:
            step = staticmethod(b.step_cold)
        cold_s, _ = time_graph(_Cold, args.steps, world)
        extra["all_inputs_cold_us"] = max_over_ranks(cold_s, world) * 1e6
    if getattr(b, "topk", False):
        pre, top = time_kernel_split(b)
        pre, top = max_over_ranks(pre, world), max_over_ranks(top, world)
        kernel_s = pre
        topk_bytes = b.topk_bytes()
        peaks = read_peaks()
        extra["kernels"] = {
            "prefill_us": pre * 1e6, "topk_us": top * 1e6,
            "topk": {"bound": "hbm", "achieved": topk_bytes / top / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": topk_bytes / top / 1e9 / peaks["hbm_gbs"], "bytes_per_step": topk_bytes,
                     "traffic": read_traffic("topk_filter_kernel", b.name)}}
        fused = b.time_fused()
        if fused is not None:
            extra["fused_l2_workspace"] = fused
            # the same call with a workspace of 512 MiB: fewer, fuller chunks
            extra["fused_512mib_workspace"] = b.time_fused(workspace_mib=512)
    e2e_s = max_over_ranks(time_e2e(b, args.steps, 3, world), world)
    from sparse_attention_block_qsa_b200 import device_error
    dev_err = device_error()
    rec = None
    if rank == 0:
        peaks = read_peaks()
        value = b.throughput(per_step) * (world if b.unit != "us" else 1)
        if hasattr(b, "roofline"):
            pass
        elif b.bound == "hbm":
            achieved = b.units / kernel_s / 1e9
            peak, unit = peaks["hbm_gbs"], "GB/s"
        else:
            # the kernel runs for seconds under the power cap (soak, then the
            # timed replay): the sustained dense bf16 figure is its peak
            achieved = b.units / kernel_s / 1e12
            peak, unit = peaks["bf16_tflops_sustained"], "TFLOP/s"
        if hasattr(b, "roofline"):
            roofline = b.roofline(kernel_s, peaks)
        else:
            which = "sustained" if b.bound == "tensor" else "copy"
            roofline = {"bound": b.bound, "achieved": achieved, "peak": peak, "unit": unit,
                        "frac": achieved / peak, "traffic": read_traffic(b.kernel, b.name), "kernel": b.kernel,
                        "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json {which} figure)"
                        if peaks["source"] == "measured" else "fallback"}
            if b.bound == "tensor":
                roofline["frac_of_burst"] = achieved / peaks["bf16_tflops"]
        pub = None if (args.kv_fp8 or args.page_size or args.f16) else PUBLISHED.get(cfg)
        conf = dict(b.config)
        if pub:
            conf["published_reference"] = pub[2]
        rec = {"workload": b.name, "value": value, "unit": b.unit, "ms_per_step": per_step * 1e3,
               "higher_is_better": b.unit != "us",
               "us_per_step": per_step * 1e6,
               "vs_baseline": (value / pub[1]) if pub and pub[0] == b.unit else None,
               "dtype": getattr(b, "dtype", "bf16"), "config": conf, "roofline": roofline,
               "e2e": {"value": b.throughput(e2e_s) * (world if b.unit != "us" else 1), "unit": b.unit,
                       "h2d_bytes_per_step": b.h2d,
                       "d2h_bytes_per_step": b.d2h, "ms_per_step": e2e_s * 1e3},
               "gpu_launches": args.steps * b.launches_per_step, "clocks": clocks, "device_error": dev_err}
        rec.update(extra)
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(b, cpu_budget_s)
            cb.pop("seconds_per_step", None)
            rec["cpu_baseline"] = cb
    del b
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def relaunch(n: int) -> int:
    """`--gpus N` without a launcher: start N replica ranks of this script
    with torch.distributed.run on 127.0.0.1 and return its exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = launch_command(sys.argv[1:], n, port)
    return subprocess.run(cmd).returncode


def launch_command(argv: list[str], n: int, port: int, script: str | None = None) -> list[str]:
    """torchrun command line that starts `script` (this file) on n ranks of one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr=127.0.0.1", f"--master-port={port}", script or os.path.abspath(__file__), *argv]


def check_world(gpus: int, env) -> tuple[int, int, int]:
    """(world, rank, local rank) of this process; the world size must be the
    requested GPU count."""
    world = int(env.get("WORLD_SIZE", "1"))
    if world != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but WORLD_SIZE={world}; launch one rank per GPU "
                         f"(or run without a launcher and let --gpus start the ranks)")
    return world, int(env.get("RANK", "0")), int(env.get("LOCAL_RANK", "0"))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=None, choices=[1, 2, 3, 4, 5, 6, 7],
                    help="one workload only (default: all five, the long-context spec-decode one as the headline)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-fp8", action="store_true", help="decode over the fp8 E4M3 key cache")
    ap.add_argument("--page-size", type=int, default=None,
                    help="decode workloads over a pool of this page size (e.g. 196) instead of their own")
    ap.add_argument("--f16", action="store_true", help="fp16 queries and keys (decode workloads and workload 4)")
    ap.add_argument("--soak", type=float, default=1.5, help="seconds of load before each timed region")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args.gpus))
    world, rank, local = check_world(args.gpus, os.environ)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    configs = [args.config] if args.config else ALL_CONFIGS
    records = {}
    for i, cfg in enumerate(configs):
        records[cfg] = measure(cfg, args, world, rank, local, cpu_budget_s=10.0 if i == 0 else 5.0)
    # the default run also times the spec-decode workload over 196-row pages,
    # the page size the vLLM PR's microbenchmarks use
    variants = []
    if not args.config and not (args.page_size or args.f16 or args.kv_fp8):
        v = argparse.Namespace(**vars(args))
        v.page_size = 196
        variants.append(measure(HEADLINE, v, world, rank, local, cpu_budget_s=5.0))

    if rank == 0:
        head = records[configs[0]]
        line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "us_per_step": head["us_per_step"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": head["vs_baseline"], "dtype": head["dtype"], "data": "synthetic",
                "config": head["config"],
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "roofline": head["roofline"], "e2e": head["e2e"],
                "gpu_launches": sum(r["gpu_launches"] for r in list(records.values()) + variants),
                "clocks": head["clocks"], "device_error": max(r["device_error"] for r in list(records.values()) + variants)}
        for key in ("kernels", "fused_l2_workspace", "fused_512mib_workspace", "all_inputs_cold_us", "cpu_baseline"):
            if key in head:
                line[key] = head[key]
        if len(configs) > 1:
            line["configs"] = {records[c]["workload"]: records[c] for c in configs[1:]}
            line["configs"].update({r["workload"]: r for r in variants})
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
