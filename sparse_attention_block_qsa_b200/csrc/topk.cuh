// Per-row top-k block selection over score rows (the caller's selection
// step in the QSA docs, MATE, and the top-512/1024/2048 selection that the
// vLLM PR's review thread discusses).
//
// Persistent CTAs, each over a contiguous range of rows (neighbouring query
// rows score alike).  Per row:
//  * Fast path: one streaming read of the row (batched 16-byte loads); a
//    float compare against a threshold predicted from the previous row's
//    exact k-th value (x 0.9) and a warp ballot append the few scores above
//    it to a shared-memory candidate list.  If that list holds at least k
//    and at most CAP scores, it contains every selected column, and the
//    exact selection runs on it alone.
//  * Exact path (first row of a CTA, or a prediction that missed): a
//    histogram of the top 13 bits of order-preserving keys over the row
//    finds the bin holding the k-th key; a second read (from L2) marks every
//    key of a higher bin and gathers the boundary bin into the list.  A
//    pathological boundary bin (more than CAP keys) is narrowed with further
//    passes over the row.
//  * On the list, histogram levels over key bits (13, 10 and 9 bits) give
//    the exact threshold key: keys above it are taken, keys equal to it are
//    ties taken from the lowest column up.  A popcount scan over a column
//    bitmap writes the selected columns in ascending order, then -1 padding.
// -inf and NaN scores are never candidates; -0.0 counts as +0.0.  The result
// does not depend on the prediction, only the speed does.
#pragma once

#include "sm100.cuh"

namespace qsa {
namespace topk {

constexpr int THREADS = 512;
constexpr int NWARPS = THREADS / 32;
constexpr int CTAS_PER_SM = 2;
constexpr int HBITS = 13;
constexpr int HBINS = 1 << HBITS;
constexpr int HSHIFT = 32 - HBITS;
constexpr int CAP = 4096;             // candidate list capacity
constexpr int SEG = CAP / NWARPS;     // list slots owned by each warp
constexpr int MAX_W = 65536;
constexpr int BM_WORDS = MAX_W / 32;
constexpr int NBINS_FINE = 1024;      // fallback narrowing histogram
constexpr uint32_t ZERO_KEY = 0x80000000u;
constexpr float PREDICT_MARGIN = 0.9f;

struct Params {
  const float* scores;
  int64_t stride;
  const int32_t* lengths;  // may be null
  int64_t rows;
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

// Score value of a key (keys of candidates only).
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

struct Smem {
  uint32_t hist[HBINS];
  uint32_t gt[BM_WORDS];    // columns taken
  uint32_t tie[BM_WORDS];   // columns whose key equals the threshold
  uint32_t cand_key[CAP];
  int32_t cand_idx[CAP];
  uint32_t red[2 * NWARPS];
  uint32_t seg_cnt[NWARPS];  // filled slots of each warp's segment
  uint32_t n_cand;
  uint32_t zeros;
  uint32_t total;
  uint32_t sel_bin;
  uint32_t sel_above;
  uint32_t lo, hi, need;
};

constexpr size_t SMEM_BYTES = sizeof(Smem);

// Inclusive block scan of two counters; totals returned.
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

// Visit every column j < len with its score; all threads of the block take
// every step together (columns past len arrive as -inf), so f may use
// warp-collective operations.  Loads are issued in batches of 8 x 16 bytes.
template <typename F>
__device__ __forceinline__ void for_each_score(const Params& p, const float* row, int len, F&& f) {
  const int tid = threadIdx.x;
  if (p.vec4) {
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = (len + 3) >> 2;
    constexpr int U = 8;
    for (int i0 = 0; i0 < n4; i0 += U * THREADS) {
      float4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * THREADS + tid;
        x[u] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (4 * i + 3 < len) {
          x[u] = __ldg(row4 + i);
        } else if (4 * i < len) {  // ragged end: scalar loads stay inside the row
          x[u].x = __ldg(row + 4 * i);
          if (4 * i + 1 < len) x[u].y = __ldg(row + 4 * i + 1);
          if (4 * i + 2 < len) x[u].z = __ldg(row + 4 * i + 2);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = 4 * (i0 + u * THREADS + tid);
        f(j, x[u].x);
        f(j + 1, x[u].y);
        f(j + 2, x[u].z);
        f(j + 3, x[u].w);
      }
    }
  } else {
    for (int j0 = 0; j0 < len; j0 += THREADS) {
      const int j = j0 + tid;
      f(j, j < len ? __ldg(row + j) : -INFINITY);
    }
  }
}

// Exact threshold among the candidate list (warp w's keys fill slots
// [w * SEG, w * SEG + seg_cnt[w])): histogram levels over key bits [31:19],
// [18:9] and [8:0], starting at `level` with the bits above it equal to
// those of `lo`.  On return lo is the threshold key and nd the number of its
// copies to take.
__device__ __forceinline__ void resolve_list(Smem& S, int level, uint32_t& lo, uint32_t& nd) {
  const int tid = threadIdx.x;
#pragma unroll 1
  for (; level < 3; ++level) {
    const int shift = level == 0 ? 19 : level == 1 ? 9 : 0;
    const int nbits = level == 0 ? 13 : level == 1 ? 10 : 9;
    const uint32_t nb = 1u << nbits;
    const uint32_t keep = level == 0 ? 0u : ~((1u << (shift + nbits)) - 1u);  // bits fixed so far
    for (uint32_t i = tid; i < nb; i += THREADS) S.hist[i] = 0;
    if (tid == 0) {
      S.lo = lo;
      S.need = nd;
    }
    __syncthreads();
    for (uint32_t i = tid; i < CAP; i += THREADS) {
      if ((i % SEG) >= S.seg_cnt[i / SEG]) continue;
      const uint32_t key = S.cand_key[i];
      if ((key & keep) == (lo & keep)) atomicAdd(&S.hist[(key >> shift) & (nb - 1u)], 1u);
    }
    __syncthreads();
    const uint32_t per = nb / THREADS > 0 ? nb / THREADS : 1u;
    uint32_t mine = 0;
    if (tid * per < nb)
      for (uint32_t i = 0; i < per; ++i) mine += S.hist[tid * per + i];
    uint32_t incl = mine, dummy = 0, tot, td;
    block_scan2(incl, dummy, S.red, tot, td);
    const uint32_t above = tot - incl;  // keys in higher bins
    if (above < nd && nd <= above + mine) {
      uint32_t acc = above;
      uint32_t bin = tid * per + per - 1;
      while (acc + S.hist[bin] < nd) {
        acc += S.hist[bin];
        --bin;
      }
      S.lo = (lo & keep) | (bin << shift);
      S.need = nd - acc;
    }
    __syncthreads();
    lo = S.lo;
    nd = S.need;
    __syncthreads();
  }
}

// Mark the list's keys above the threshold as taken and its threshold
// copies as ties.
__device__ __forceinline__ void mark_list(Smem& S, uint32_t thr) {
  for (uint32_t i = threadIdx.x; i < CAP; i += THREADS) {
    if ((i % SEG) >= S.seg_cnt[i / SEG]) continue;
    const uint32_t key = S.cand_key[i];
    const int32_t j = S.cand_idx[i];
    if (key > thr) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    else if (key == thr) atomicOr(&S.tie[j >> 5], 1u << (j & 31));
  }
}

// Append (key, column) to this warp's list segment when `hit`; the count
// lives in a register of every lane.  Returns false once the segment is
// full (further keys are dropped and counted).
__device__ __forceinline__ void warp_append(Smem& S, bool hit, uint32_t key, int j, uint32_t& count) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t m = __ballot_sync(0xffffffffu, hit);
  if (m) {
    const uint32_t pos = count + __popc(m & ((1u << lane) - 1u));
    if (hit && pos < SEG) {
      S.cand_key[warp * SEG + pos] = key;
      S.cand_idx[warp * SEG + pos] = j;
    }
    count += __popc(m);
  }
}

// Selection of one row into the bitmaps; returns the threshold key (0 when
// every candidate is taken) and, in need_tie, how many of its copies count.
__device__ __forceinline__ uint32_t select_row(const Params& p, Smem& S, const float* row, int len, float pred,
                                               uint32_t& need_tie) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t k = (uint32_t)p.k;
  need_tie = 0;

  // ---- fast path: gather the scores at or above the predicted threshold
  if (pred > 0.f) {
    uint32_t count = 0;
    for_each_score(p, row, len, [&](int j, float x) {
      const bool hit = x >= pred;
      warp_append(S, hit, hit ? score_key(x) : 0u, j, count);
    });
    if (lane == 0) S.seg_cnt[threadIdx.x >> 5] = min(count, (uint32_t)SEG);
    const uint32_t full = __reduce_or_sync(0xffffffffu, count > SEG ? 1u : 0u);
    const uint32_t cnt = __reduce_add_sync(0xffffffffu, lane == 0 ? count : 0u);
    if (lane == 0) {
      atomicAdd(&S.n_cand, cnt);
      if (full) atomicOr(&S.total, 0x80000000u);  // a segment overflowed
    }
    __syncthreads();
    const uint32_t n = S.n_cand;
    const bool overflow = S.total & 0x80000000u;
    if (!overflow && n >= k) {
      uint32_t lo = 0, nd = k;
      resolve_list(S, 0, lo, nd);
      mark_list(S, lo);
      need_tie = nd;
      return lo;
    }
    __syncthreads();  // everyone has read the counters before they are reset
    if (tid == 0) {
      S.n_cand = 0;
      S.total = 0;
    }
    __syncthreads();
  }

  // ---- exact path, pass A: histogram of the top 13 key bits
  uint32_t cnt = 0, zc = 0;
  for_each_score(p, row, len, [&](int j, float x) {
    const uint32_t key = score_key(x);
    if (key) {
      ++cnt;
      if (key == ZERO_KEY) ++zc;
      else atomicAdd(&S.hist[key >> HSHIFT], 1u);
    }
  });
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  zc = __reduce_add_sync(0xffffffffu, zc);
  if (lane == 0) {
    atomicAdd(&S.total, cnt);
    if (zc) atomicAdd(&S.zeros, zc);
  }
  __syncthreads();
  if (tid == 0) S.hist[ZERO_KEY >> HSHIFT] += S.zeros;
  __syncthreads();
  const uint32_t total = S.total;
  const bool take_all = total <= k;
  if (!take_all) {
    uint32_t mine = 0;  // thread t owns bins [16t, 16t + 16)
#pragma unroll
    for (int i = 0; i < 16; ++i) mine += S.hist[16 * tid + i];
    uint32_t incl = mine, dummy = 0, tot, td;
    block_scan2(incl, dummy, S.red, tot, td);
    const uint32_t above = tot - incl;
    if (above < k && k <= above + mine) {
      uint32_t acc = above;
      int bin = 16 * tid + 15;
      while (acc + S.hist[bin] < k) {
        acc += S.hist[bin];
        --bin;
      }
      S.sel_bin = (uint32_t)bin;
      S.sel_above = acc;
    }
    __syncthreads();
  }
  const uint32_t sel_bin = take_all ? 0u : S.sel_bin;
  const uint32_t need = take_all ? 0u : k - S.sel_above;  // keys to take from the boundary bin

  // ---- exact path, pass B: mark higher bins, gather the boundary bin
  uint32_t count = 0;
  for_each_score(p, row, len, [&](int j, float x) {
    const uint32_t key = score_key(x);
    const uint32_t bin = key >> HSHIFT;
    if (key && (take_all || bin > sel_bin)) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    warp_append(S, key && !take_all && bin == sel_bin, key, j, count);
  });
  if (lane == 0) S.seg_cnt[threadIdx.x >> 5] = min(count, (uint32_t)SEG);
  const uint32_t full = __reduce_or_sync(0xffffffffu, count > SEG ? 1u : 0u);
  if (lane == 0 && full) atomicOr(&S.n_cand, 1u);  // a segment overflowed
  __syncthreads();
  if (take_all) return 0u;
  uint32_t lo = sel_bin << HSHIFT, nd = need;
  if (S.n_cand == 0) {
    resolve_list(S, 1, lo, nd);
    mark_list(S, lo);
    need_tie = nd;
    return lo;
  }
  // narrow [lo, hi] inside the boundary bin until one key value is left
  uint32_t hi = lo | ((1u << HSHIFT) - 1u);
  for (int pass = 0; pass < 4 && lo < hi; ++pass) {
    const uint64_t span = (uint64_t)hi - lo + 1;
    int shift = 0;
    while (((span - 1) >> shift) >= (uint64_t)NBINS_FINE) ++shift;  // largest bin index < NBINS_FINE
    for (int i = tid; i < NBINS_FINE; i += THREADS) S.hist[i] = 0;
    if (tid == 0) {
      S.lo = lo;
      S.hi = hi;
      S.need = nd;
    }
    __syncthreads();
    for_each_score(p, row, len, [&](int j, float x) {
      const uint32_t key = score_key(x);
      if (key >= lo && key <= hi) atomicAdd(&S.hist[(key - lo) >> shift], 1u);
    });
    __syncthreads();
    const uint32_t mine = S.hist[2 * tid] + S.hist[2 * tid + 1];
    uint32_t incl = mine, dummy = 0, tot, td;
    block_scan2(incl, dummy, S.red, tot, td);
    const uint32_t above = tot - incl;
    if (above < nd && nd <= above + mine) {
      uint32_t acc = above;
      int bin = 2 * tid + 1;
      if (acc + S.hist[bin] < nd) {
        acc += S.hist[bin];
        bin = 2 * tid;
      }
      S.lo = lo + ((uint32_t)bin << shift);
      S.hi = (uint32_t)min((uint64_t)hi, (uint64_t)S.lo + ((uint64_t)1 << shift) - 1);
      S.need = nd - acc;
    }
    __syncthreads();
    lo = S.lo;
    hi = S.hi;
    nd = S.need;
    __syncthreads();
  }
  if (lo < hi && tid == 0) record_device_error(QSA_DEVERR_SELECT);
  const uint32_t thr = lo, top = (sel_bin << HSHIFT) | ((1u << HSHIFT) - 1u);
  for_each_score(p, row, len, [&](int j, float x) {
    const uint32_t key = score_key(x);
    if (key > thr && key <= top) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    else if (key == thr && key) atomicOr(&S.tie[j >> 5], 1u << (j & 31));
  });
  need_tie = nd;
  return thr;
}

__global__ void __launch_bounds__(THREADS, CTAS_PER_SM) topk_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x;
  const uint32_t k = (uint32_t)p.k;
  const int64_t r_begin = (int64_t)blockIdx.x * p.rows / gridDim.x;
  const int64_t r_end = (int64_t)(blockIdx.x + 1) * p.rows / gridDim.x;
  float pred = 0.f;  // predicted lower bound of the k-th score (0: none)

  for (int64_t r = r_begin; r < r_end; ++r) {
    const float* row = p.scores + r * p.stride;
    int32_t* out = p.idx + r * p.idx_stride;
    int len = p.W;
    if (p.lengths != nullptr) len = min(max(__ldg(p.lengths + r), 0), p.W);
    const int nwords = (len + 31) >> 5;

    for (int i = tid; i < HBINS; i += THREADS) S.hist[i] = 0;
    for (int i = tid; i < nwords; i += THREADS) S.gt[i] = S.tie[i] = 0;
    if (tid == 0) {
      S.n_cand = 0;
      S.zeros = 0;
      S.total = 0;
    }
    __syncthreads();

    uint32_t need_tie;
    const uint32_t thr = select_row(p, S, row, len, pred, need_tie);
    __syncthreads();
    // next row: a little below this row's k-th score (positive scores only)
    const float tv = thr ? key_value(thr) : 0.f;
    pred = (thr & 0x80000000u) && tv > 0.f ? tv * PREDICT_MARGIN : 0.f;

    // ---- ordered output: contiguous bitmap words per thread
    const int wpt = (nwords + THREADS - 1) / THREADS;
    const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);
    uint32_t ties = 0;
    for (int w = w0; w < w1; ++w) ties += __popc(S.tie[w]);
    uint32_t t_incl = ties, d0 = 0, t_tot, d_tot;
    block_scan2(t_incl, d0, S.red, t_tot, d_tot);
    const uint32_t ties_before = t_incl - ties;
    uint32_t tie_left = need_tie > ties_before ? need_tie - ties_before : 0u;  // ties this thread may take
    uint32_t sel = 0;
    for (int w = w0; w < w1; ++w) {
      uint32_t tw = S.tie[w];
      while (tw && (uint32_t)__popc(tw) > tie_left) tw &= ~(1u << (31 - __clz(tw)));  // keep the lowest
      tie_left -= (uint32_t)__popc(tw);
      S.tie[w] = tw;
      sel += (uint32_t)__popc(S.gt[w] | tw);
    }
    uint32_t s_incl = sel, d1 = 0, s_tot, d1_tot;
    block_scan2(s_incl, d1, S.red, s_tot, d1_tot);
    uint32_t pos = s_incl - sel;
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = S.gt[w] | S.tie[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < k) out[pos] = w * 32 + b;
        ++pos;
      }
    }
    for (uint32_t s = min(s_tot, k) + tid; s < k; s += THREADS) out[s] = -1;
    __syncthreads();  // bitmaps and histogram are reused by the next row
  }
}

}  // namespace topk
}  // namespace qsa
