// Per-row top-k block selection over score rows (the caller's selection
// step in the QSA docs, MATE, and the top-512/1024/2048 selection that the
// vLLM PR's review thread discusses).
//
// One CTA per row.  The row is read once from HBM (16-byte loads when the
// row is aligned), turned into order-preserving 32-bit keys and, when it
// fits, kept in shared memory.  The k-th largest key is then found exactly
// by narrowing a key range with 1024-bin histograms (at most 4 passes over
// the cached row); every pass bins only the keys still inside the range, so
// a few hot bins never serialise the whole row.  A final ordered pass writes
// the selected column indices in ascending order: all keys above the
// threshold, then threshold keys from the lowest column up until k are
// taken.  -inf and NaN scores are never candidates; -0.0 counts as +0.0.
#pragma once

#include "sm100.cuh"

namespace qsa {
namespace topk {

constexpr int THREADS = 512;
constexpr int NWARPS = THREADS / 32;
constexpr int BINS = 1024;
constexpr int LOG2_BINS = 10;
constexpr int MAX_CACHED_W = 49152;  // row cache of up to 192 KB

struct Params {
  const float* scores;
  int64_t stride;
  const int32_t* lengths;  // may be null
  int32_t W;
  int32_t k;
  int32_t* idx;
  int64_t idx_stride;
  int32_t vec4;            // rows are 16-byte aligned: use float4 loads
};

// Order-preserving key of a score; 0 marks "not a candidate".
__device__ __forceinline__ uint32_t score_key(float x) {
  if (!(x > -INFINITY)) return 0u;  // -inf and NaN
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;     // -0.0 -> +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct Smem {
  uint32_t hist[BINS];
  uint32_t red[NWARPS * 2];
  uint32_t sel_lo, sel_hi, sel_need, sel_done;
};

// Inclusive block scan of two counters at once; totals returned.
__device__ __forceinline__ void block_scan2(uint32_t& a, uint32_t& b, uint32_t* red, uint32_t& ta,
                                            uint32_t& tb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t ya = __shfl_up_sync(0xffffffffu, a, o);
    const uint32_t yb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) {
      a += ya;
      b += yb;
    }
  }
  if (lane == 31) {
    red[warp] = a;
    red[NWARPS + warp] = b;
  }
  __syncthreads();
  uint32_t ba = 0, bb = 0;
  ta = 0;
  tb = 0;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) {
    const uint32_t ra = red[w], rb = red[NWARPS + w];
    if (w < warp) {
      ba += ra;
      bb += rb;
    }
    ta += ra;
    tb += rb;
  }
  __syncthreads();
  a += ba;
  b += bb;
}

template <bool CACHED>
__global__ void __launch_bounds__(THREADS)
    topk_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  uint32_t* cache = reinterpret_cast<uint32_t*>(smem_raw + sizeof(Smem));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r = blockIdx.x;
  const float* row = p.scores + r * p.stride;
  int32_t* out = p.idx + r * p.idx_stride;
  int len = p.W;
  if (p.lengths != nullptr) len = min(max(__ldg(p.lengths + r), 0), p.W);

  auto key_at = [&](int j) -> uint32_t { return CACHED ? cache[j] : score_key(__ldg(row + j)); };

  // ---- pass 0: load, count candidates, min / max key
  uint32_t cnt = 0, kmin = 0xffffffffu, kmax = 0u;
  auto take = [&](int j, float x) {
    const uint32_t key = score_key(x);
    if (CACHED) cache[j] = key;
    if (key) {
      ++cnt;
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
  };
  if (p.vec4) {
    const int n4 = len >> 2;
    const float4* row4 = reinterpret_cast<const float4*>(row);
    for (int i = tid; i < n4; i += THREADS) {
      const float4 x = __ldcs(row4 + i);
      take(4 * i, x.x);
      take(4 * i + 1, x.y);
      take(4 * i + 2, x.z);
      take(4 * i + 3, x.w);
    }
    for (int j = 4 * n4 + tid; j < len; j += THREADS) take(j, __ldcs(row + j));
  } else {
    for (int j = tid; j < len; j += THREADS) take(j, __ldcs(row + j));
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    S.red[warp] = cnt;
    S.hist[warp] = kmin;
    S.hist[NWARPS + warp] = kmax;
  }
  __syncthreads();
  uint32_t total = 0;
  kmin = 0xffffffffu;
  kmax = 0u;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) {
    total += S.red[w];
    kmin = min(kmin, S.hist[w]);
    kmax = max(kmax, S.hist[NWARPS + w]);
  }
  __syncthreads();

  const uint32_t k = (uint32_t)p.k;
  uint32_t thr;       // threshold key: every key above it is taken
  uint32_t need;      // how many keys equal to thr are taken (lowest columns first)
  if (total <= k) {
    thr = 1u;         // every candidate (keys >= 1) ...
    need = 0xffffffffu;
  } else {
    // ---- narrow [lo, hi] until it holds a single key value, tracking how
    // many keys of the range are still to be taken from the top
    uint32_t lo = kmin, hi = kmax;
    need = k;
    // each pass shrinks the range by 2^10 at least: 4 passes cover 32 bits
    for (int pass = 0; pass < 6 && lo < hi; ++pass) {
      if (tid == 0) {
        S.sel_lo = lo;
        S.sel_hi = hi;
        S.sel_need = need;
      }
      const uint64_t span = (uint64_t)hi - lo + 1;
      int shift = 0;
      while (((span - 1) >> shift) >= (uint64_t)BINS) ++shift;  // largest bin index < BINS
      for (int i = tid; i < BINS; i += THREADS) S.hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < len; j += THREADS) {
        const uint32_t key = key_at(j);
        if (key >= lo && key <= hi) atomicAdd(&S.hist[(key - lo) >> shift], 1u);
      }
      __syncthreads();
      // bins from the top: thread t owns bins [2t, 2t+2)
      uint32_t mine = S.hist[2 * tid] + S.hist[2 * tid + 1];
      uint32_t dummy = 0, tot, tdummy;
      uint32_t incl = mine;
      block_scan2(incl, dummy, S.red, tot, tdummy);
      const uint32_t above = tot - incl;  // keys in bins above mine
      if (above < need && need <= above + mine) {
        uint32_t acc = above;
        int bin = 2 * tid + 1;
        if (acc + S.hist[bin] < need) {
          acc += S.hist[bin];
          bin = 2 * tid;
        }
        S.sel_lo = lo + ((uint32_t)bin << shift);
        const uint64_t top = (uint64_t)S.sel_lo + ((uint64_t)1 << shift) - 1;
        S.sel_hi = (uint32_t)min((uint64_t)hi, top);
        S.sel_need = need - acc;
      }
      __syncthreads();
      lo = S.sel_lo;
      hi = S.sel_hi;
      need = S.sel_need;
      __syncthreads();
    }
    if (lo < hi && tid == 0) record_device_error(QSA_DEVERR_SELECT);
    thr = lo;
  }

  // ---- ordered selection: contiguous column chunks per thread (odd length
  // so that the threads of a warp read different banks)
  int chunk = (len + THREADS - 1) / THREADS;
  chunk |= 1;
  const int c0 = min(tid * chunk, len), c1 = min(c0 + chunk, len);
  uint32_t gt = 0, eq = 0;
  for (int j = c0; j < c1; ++j) {
    const uint32_t key = key_at(j);
    gt += key > thr;
    eq += key == thr;
  }
  uint32_t gt_incl = gt, eq_incl = eq, gt_tot, eq_tot;
  block_scan2(gt_incl, eq_incl, S.red, gt_tot, eq_tot);
  const uint32_t eq_before = eq_incl - eq;
  uint32_t pos = (gt_incl - gt) + min(eq_before, need);
  uint32_t eq_seen = eq_before;
  for (int j = c0; j < c1; ++j) {
    const uint32_t key = key_at(j);
    bool sel = key > thr;
    if (key == thr) {
      sel = eq_seen < need;
      ++eq_seen;
    }
    if (sel && pos < k) out[pos++] = j;
  }
  const uint32_t taken = gt_tot + min(eq_tot, need);
  for (uint32_t s = taken + tid; s < k; s += THREADS) out[s] = -1;
}

}  // namespace topk
}  // namespace qsa
