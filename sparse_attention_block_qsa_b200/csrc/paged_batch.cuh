// A mixed decode + prefill batch scored from the paged compressed key cache
// in one call: the step before the score kernels (per-row positions, visible
// counts and key intervals, computed on the device as in vLLM qsa_cache.py's
// metadata kernel), then the two score kernels, chained with programmatic
// dependent launches (vLLM's metadata kernel uses the same mechanism,
// "gdc_wait" / "gdc_launch_dependents").
//
//  * gather_kernel (the metadata step): requests D .. R-1 are prefills.  Each
//    CTA scans their key counts n_r = min(seq_len_r / 4, W) into offsets in
//    shared memory; rows of prefill requests get ks = offset of their
//    request, ke = ks + min(visible, n_r); and the prefill keys are copied
//    from their pages into a packed array (a missing page's keys are zeroed
//    and masked afterwards), so that the tcgen05 prefill kernel reads them
//    with TMA tiles.  Keys are small next to the scores they feed (256 bytes
//    per key against 4 bytes per row), so the copy costs little.
//  * fixup_kernel: the scores of keys whose page is missing become -inf
//    (one CTA per prefill request, one page entry per lane; nothing to do
//    when every page is there).
#pragma once

#include "sm100.cuh"

namespace qsa {
namespace batch {

constexpr int THREADS = 256;
constexpr int MAX_PREFILL = 8192;   // prefill requests per call (their prefix lives in shared memory)

struct Params {
  const int32_t* cu;         // int32 [R + 1]
  const int32_t* seq_lens;   // int32 [R]
  int32_t R, D;              // requests; the first D are decodes
  int64_t row0;              // first prefill row (D * decode query length)
  int64_t T;
  const uint16_t* k_cache;
  int64_t num_pages;
  int32_t page_size;
  int64_t k_page_stride, k_row_stride;
  const int32_t* page_table;
  int64_t pt_stride;
  int32_t max_pages;
  int32_t W;
  uint16_t* packed;          // bf16 [capacity, 128]
  int32_t* ks;               // int32 [T - row0]
  int32_t* ke;
  float* out;                // fp32 scores [T, W]
  int64_t out_stride;
};

constexpr size_t SMEM_BYTES = sizeof(int32_t) * (MAX_PREFILL + 1);

__device__ __forceinline__ void pdl_wait_then_release() {
  // Wait until the previous kernel on the stream has completed and its writes
  // are visible (a no-op without a programmatic dependency), then let the
  // next one begin launching.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ int keys_of(const Params& p, int r) {
  return min(max(__ldg(p.seq_lens + r), 0) >> 2, p.W);
}

// Block-wide exclusive prefix of the prefill requests' key counts into pre[0..P].
__device__ __forceinline__ void scan_keys(const Params& p, int32_t* pre) {
  __shared__ int32_t warp_sum[THREADS / 32];
  const int P = p.R - p.D;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t carry = 0;
  for (int base = 0; base < P; base += THREADS) {
    const int i = base + tid;
    const int32_t v = i < P ? keys_of(p, p.D + i) : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sum[warp] = x;
    __syncthreads();
    int32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) {
      before += w < warp ? warp_sum[w] : 0;
      all += warp_sum[w];
    }
    if (i < P) pre[i] = carry + before + x - v;
    carry += all;
    __syncthreads();
  }
  if (tid == 0) pre[P] = carry;
  __syncthreads();
}

__global__ void __launch_bounds__(THREADS) gather_kernel(const Params p) {
  extern __shared__ int32_t pre[];
  pdl_wait_then_release();
  scan_keys(p, pre);
  const int P = p.R - p.D;
  const int64_t nthreads = (int64_t)gridDim.x * THREADS;
  const int64_t gtid = (int64_t)blockIdx.x * THREADS + threadIdx.x;

  // ---- key intervals of the prefill rows
  for (int64_t t = p.row0 + gtid; t < p.T; t += nthreads) {
    int lo = p.D, hi = p.R - 1;  // last request whose first row is <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)__ldg(p.cu + mid) <= t) lo = mid;
      else hi = mid - 1;
    }
    const int first = __ldg(p.cu + lo);
    const int qlen = __ldg(p.cu + lo + 1) - first;
    const int L = max(__ldg(p.seq_lens + lo), 0);
    const int pos = L - qlen + (int)(t - first);
    const int vis = max(0, min((pos + 1) >> 2, L >> 2));
    const int32_t off = pre[lo - p.D];
    p.ks[t - p.row0] = off;
    p.ke[t - p.row0] = off + min(vis, pre[lo - p.D + 1] - off);
  }

  // ---- the prefill keys, packed: a half-warp copies one 256-byte key row
  const int64_t total = pre[P];
  const int64_t nhalf = nthreads >> 4;
  const int hl = threadIdx.x & 15;
  for (int64_t i = gtid >> 4; i < total; i += nhalf) {
    int lo = 0, hi = P - 1;  // prefill request holding packed key i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)pre[mid] <= i) lo = mid;
      else hi = mid - 1;
    }
    const int r = p.D + lo;
    const int n = (int)(i - pre[lo]);
    const int lp = n / p.page_size;
    const int page = lp < p.max_pages ? __ldg(p.page_table + (int64_t)r * p.pt_stride + lp) : -1;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (page >= 0 && (int64_t)page < p.num_pages) {
      const uint16_t* src = p.k_cache + (int64_t)page * p.k_page_stride + (int64_t)(n - lp * p.page_size) * p.k_row_stride;
      v = __ldg(reinterpret_cast<const uint4*>(src) + hl);
    }
    reinterpret_cast<uint4*>(p.packed + i * 128)[hl] = v;
  }
}

// One CTA per prefill request: -inf over the scores of keys whose page is
// missing.  Each lane checks one page entry, so a warp covers 32 pages per
// round trip; the (rare) missing pages are then handled one at a time by the
// whole warp.
__global__ void __launch_bounds__(THREADS) fixup_kernel(const Params p) {
  pdl_wait_then_release();
  const int r = p.D + blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = max(__ldg(p.seq_lens + r), 0);
  const int n_r = min(L >> 2, p.W);
  const int first = __ldg(p.cu + r);
  const int qlen = __ldg(p.cu + r + 1) - first;
  const int pages = (n_r + p.page_size - 1) / p.page_size;
  for (int lp0 = warp * 32; lp0 < pages; lp0 += THREADS) {
    const int lp = lp0 + lane;
    bool missing = false;
    if (lp < pages) {
      const int page = lp < p.max_pages ? __ldg(p.page_table + (int64_t)r * p.pt_stride + lp) : -1;
      missing = !(page >= 0 && (int64_t)page < p.num_pages);
    }
    unsigned m = __ballot_sync(0xffffffffu, missing);
    while (m) {
      const int k0 = (lp0 + __ffs(m) - 1) * p.page_size, k1 = min(k0 + p.page_size, n_r);
      m &= m - 1;
      for (int i = 0; i < qlen; ++i) {
        const int pos = L - qlen + i;
        const int vis = max(0, min((pos + 1) >> 2, L >> 2));
        float* row = p.out + (int64_t)(first + i) * p.out_stride;
        for (int j = k0 + lane; j < min(k1, vis); j += 32) row[j] = -INFINITY;
      }
    }
  }
}

}  // namespace batch
}  // namespace qsa
