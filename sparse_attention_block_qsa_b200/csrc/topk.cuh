// Per-row top-k block selection over score rows (the caller's selection
// step in the QSA docs, MATE, and the top-512/1024/2048 selection that the
// vLLM PR's review thread discusses).
//
// Persistent CTAs, each over a contiguous range of rows (neighbouring query
// rows score alike).  Two kernels share the selection logic:
//  * topk_pipe_kernel (rows 16-byte aligned, W a multiple of 4), two CTAs per
//    SM: a producer warp streams the rows as 16 KB bulk copies, filtering
//    warps build each row's candidate list while selecting warps resolve the
//    previous row (described beside the kernel).
//  * topk_rows_kernel (any alignment): 8 warps read each row with batched
//    loads themselves.
// Per row:
//  * Fast path: every score is compared with a threshold predicted from an
//    earlier row's exact k-th value (x 0.9); a lane holding a score at or
//    above it appends it to its warp's segment of a candidate list (about 4%
//    of the scores; the common case costs a compare per score).  If the list
//    holds at least k scores and no segment overflowed, it holds every
//    selected column and the selection runs on it alone: one histogram over
//    [predicted key, largest key] finds the boundary bin; a warp ranks the
//    boundary bin's keys (larger first, then lower column) when they are few,
//    otherwise further histograms narrow the bin.
//  * Exact path (no prediction yet, or one that missed): a histogram of the
//    top 11 bits of order-preserving keys over the row finds the bin holding
//    the k-th key; a second read of the row marks every key of a higher bin
//    and gathers the boundary bin, resolved with 11- and 10-bit histograms; a
//    pathological boundary bin is narrowed with further passes over the row.
//    Its exact k-th value becomes the next prediction.
//  * A popcount scan over a column bitmap writes the selected columns in
//    ascending order, then -1 padding.
// -inf and NaN scores are never candidates; -0.0 counts as +0.0.  The result
// does not depend on the prediction, only the speed does.
#pragma once

#include <cstddef>

#include "sm100.cuh"

namespace qsa {
namespace topk {

constexpr int THREADS = 256;          // selecting threads (both kernels)
constexpr int NWARPS = THREADS / 32;
constexpr int ROWS_CTAS_PER_SM = 4;
constexpr int HBITS = 11;
constexpr int HBINS = 1 << HBITS;
constexpr int HSHIFT = 32 - HBITS;
constexpr int CAP = 2048;             // candidate list capacity
constexpr int SEG = CAP / NWARPS;     // list slots owned by each warp
constexpr int MAX_W = 65536;
constexpr int BM_WORDS = MAX_W / 32;
constexpr int NBINS_FINE = 1024;      // narrowing histogram
constexpr int FBINS = 2048;           // fast-path histogram
constexpr uint32_t ZERO_KEY = 0x80000000u;
constexpr float PREDICT_MARGIN = 0.9f;
constexpr int CHUNK = 4096;           // floats per ring slot (16 KB)
static_assert(FBINS == HBINS, "the fast path and the exact path share one histogram");

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
  float* pred_state;       // per-CTA predictions carried between launches (may be null)
  const int32_t* row_list;    // rows kernel: if set, only these rows (exact path), row_count of them
  const uint32_t* row_count;
  uint8_t* ws;                // two-pass kernels: the caller's workspace (tp_layout)
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

// Shared state of the selection (both kernels).
struct Sel {
  uint32_t hist[HBINS];
  uint32_t gt[BM_WORDS];    // columns taken
  uint32_t tie[BM_WORDS];   // columns whose key equals the threshold
  uint32_t cand_key[CAP];
  int32_t cand_idx[CAP];
  uint32_t red[2 * NWARPS];
  uint32_t seg_cnt[NWARPS];  // keys appended by each warp (may pass SEG: overflow)
  uint32_t small_key[32];
  int32_t small_idx[32];
  uint32_t n_small;
  uint32_t kmax;
  uint32_t zeros;
  uint32_t total;
  uint32_t sel_bin;
  uint32_t sel_above;
  uint32_t lo, hi, need;
  int abort;
  int stop;  // abort as seen by the selecting warps at a row boundary
};

struct BlockSync {
  __device__ static void sync() { __syncthreads(); }
};
struct ConsumerSync {  // the selecting threads only (the producer warp keeps streaming)
  __device__ static void sync() { named_barrier_sync(1, THREADS); }
};

// Inclusive scan of two counters over the selecting threads; totals returned.
template <class Sync>
__device__ __forceinline__ void block_scan2(uint32_t& a, uint32_t& b, uint32_t* red, uint32_t& ta, uint32_t& tb) {
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
  Sync::sync();
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
  Sync::sync();
  a += ba;
  b += bb;
}

// Visit every column j < len of a row in global memory with its score; all
// selecting threads take every step together (columns past len arrive as
// -inf), so f may use warp-collective operations.  Loads are issued in
// batches of 4 x 16 bytes per thread.
template <typename F>
__device__ __forceinline__ void for_each_score(const Params& p, const float* row, int len, F&& f) {
  const int tid = threadIdx.x;
  if (p.vec4) {
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = (len + 3) >> 2;
    constexpr int U = 4;
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

// Fast path for one score: at or above the predicted (positive) threshold it
// goes to this warp's list segment; its key is then simply the float bits
// with the top bit set.
__device__ __forceinline__ void fast_put(Sel& S, float x, int j, uint32_t& pos, uint32_t& kmax) {
  const uint32_t key = __float_as_uint(x) | 0x80000000u;
  const int warp = threadIdx.x >> 5;
  if (pos < SEG) {
    S.cand_key[warp * SEG + pos] = key;
    S.cand_idx[warp * SEG + pos] = j;
  }
  kmax = max(kmax, key);
  ++pos;
}

__device__ __forceinline__ void fast_visit4(Sel& S, float4 x, int j0, float pred, uint32_t& kmax) {
  const bool h0 = x.x >= pred, h1 = x.y >= pred, h2 = x.z >= pred, h3 = x.w >= pred;
  if (h0 | h1 | h2 | h3) {
    uint32_t pos = atomicAdd(&S.seg_cnt[threadIdx.x >> 5], (uint32_t)h0 + h1 + h2 + h3);
    if (h0) fast_put(S, x.x, j0, pos, kmax);
    if (h1) fast_put(S, x.y, j0 + 1, pos, kmax);
    if (h2) fast_put(S, x.z, j0 + 2, pos, kmax);
    if (h3) fast_put(S, x.w, j0 + 3, pos, kmax);
  }
}

__device__ __forceinline__ void fast_visit1(Sel& S, float x, int j, float pred, uint32_t& kmax) {
  if (x >= pred) {
    uint32_t pos = atomicAdd(&S.seg_cnt[threadIdx.x >> 5], 1u);
    fast_put(S, x, j, pos, kmax);
  }
}

// Append (key, column) to this warp's list segment when `hit` (all lanes
// call it together).
__device__ __forceinline__ void warp_append(Sel& S, bool hit, uint32_t key, int j) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t m = __ballot_sync(0xffffffffu, hit);
  if (m) {
    uint32_t base = 0;
    if (lane == 0) base = atomicAdd(&S.seg_cnt[warp], (uint32_t)__popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    const uint32_t pos = base + __popc(m & ((1u << lane) - 1u));
    if (hit && pos < SEG) {
      S.cand_key[warp * SEG + pos] = key;
      S.cand_idx[warp * SEG + pos] = j;
    }
  }
}

// Keys in the list and whether a segment overflowed (read after a barrier).
__device__ __forceinline__ uint32_t list_size(const Sel& S, bool& overflow) {
  uint32_t n = 0;
  overflow = false;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) {
    n += S.seg_cnt[w];
    overflow |= S.seg_cnt[w] > (uint32_t)SEG;
  }
  return n;
}

template <typename F>
__device__ __forceinline__ void for_each_candidate(Sel& S, F&& f) {
  for (uint32_t i = threadIdx.x; i < CAP; i += THREADS)
    if ((i % SEG) < min(S.seg_cnt[i / SEG], (uint32_t)SEG)) f(S.cand_key[i], S.cand_idx[i]);
}

// Narrow [lo, hi] (keys of the candidate list, or of the row when row !=
// nullptr) with 1024-bin histograms until one key value is left; nd is the
// number of keys to take from the top of the range and on return the number
// of threshold copies to take.
template <class Sync>
__device__ __forceinline__ void narrow(const Params& p, Sel& S, const float* row, int len, uint32_t& lo,
                                       uint32_t& hi, uint32_t& nd) {
  const int tid = threadIdx.x;
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
    Sync::sync();
    auto count = [&](uint32_t key) {
      if (key >= lo && key <= hi) atomicAdd(&S.hist[(key - lo) >> shift], 1u);
    };
    if (row) for_each_score(p, row, len, [&](int, float x) { count(score_key(x)); });
    else for_each_candidate(S, [&](uint32_t key, int32_t) { count(key); });
    Sync::sync();
    constexpr int per = NBINS_FINE / THREADS;
    uint32_t mine = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) mine += S.hist[per * tid + i];
    uint32_t incl = mine, dummy = 0, tot, td;
    block_scan2<Sync>(incl, dummy, S.red, tot, td);
    const uint32_t above = tot - incl;
    if (above < nd && nd <= above + mine) {
      uint32_t acc = above;
      int bin = per * tid + per - 1;
      while (acc + S.hist[bin] < nd) {
        acc += S.hist[bin];
        --bin;
      }
      S.lo = lo + ((uint32_t)bin << shift);
      S.hi = (uint32_t)min((uint64_t)hi, (uint64_t)S.lo + ((uint64_t)1 << shift) - 1);
      S.need = nd - acc;
    }
    Sync::sync();
    lo = S.lo;
    hi = S.hi;
    nd = S.need;
    Sync::sync();
  }
  if (lo < hi && tid == 0) record_device_error(QSA_DEVERR_SELECT);
}

// Bin of the k-th largest key of a 2048-bin histogram; thread t owns bins
// [8t, 8t + 8).  Writes S.sel_bin and S.sel_above (keys in higher bins).
template <class Sync>
__device__ __forceinline__ void find_bin(Sel& S, uint32_t k) {
  constexpr int per = HBINS / THREADS;
  const int tid = threadIdx.x;
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) mine += S.hist[per * tid + i];
  uint32_t incl = mine, dummy = 0, tot, td;
  block_scan2<Sync>(incl, dummy, S.red, tot, td);
  const uint32_t above = tot - incl;
  if (above < k && k <= above + mine) {
    uint32_t acc = above;
    int bin = per * tid + per - 1;
    while (acc + S.hist[bin] < k) {
      acc += S.hist[bin];
      --bin;
    }
    S.sel_bin = (uint32_t)bin;
    S.sel_above = acc;
  }
  Sync::sync();
}

// Fast-path resolution on the candidate list (all keys >= key_lo, at least
// k of them, S.hist zeroed): marks the selected columns.  With kth != nullptr
// the k-th largest key is returned there too.
template <class Sync>
__device__ __forceinline__ void resolve_candidates(const Params& p, Sel& S, uint32_t key_lo, uint32_t& thr,
                                                   uint32_t& need_tie, uint32_t* kth = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t k = (uint32_t)p.k;
  const uint32_t kmax = S.kmax;
  const uint64_t span = (uint64_t)kmax - key_lo + 1;
  int shift = 0;
  while (((span - 1) >> shift) >= (uint64_t)FBINS) ++shift;
  for_each_candidate(S, [&](uint32_t key, int32_t) { atomicAdd(&S.hist[(key - key_lo) >> shift], 1u); });
  Sync::sync();
  find_bin<Sync>(S, k);
  const uint32_t B = S.sel_bin, nb = S.hist[B], needB = k - S.sel_above;
  const uint32_t blo = key_lo + (B << shift);
  const uint32_t bhi = (uint32_t)min((uint64_t)kmax, (uint64_t)blo + ((uint64_t)1 << shift) - 1);
  // keys above the boundary bin are taken; its own keys are set aside
  for_each_candidate(S, [&](uint32_t key, int32_t j) {
    if (key > bhi) {
      atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    } else if (key >= blo && nb <= 32) {
      const uint32_t pos = atomicAdd(&S.n_small, 1u);
      S.small_key[pos] = key;
      S.small_idx[pos] = j;
    }
  });
  Sync::sync();
  if (nb <= 32) {
    if (tid < 32) {  // one warp ranks the boundary keys: larger first, then lower column
      const bool have = (uint32_t)lane < nb;
      const uint32_t key = have ? S.small_key[lane] : 0u;
      const int32_t j = have ? S.small_idx[lane] : INT32_MAX;
      uint32_t rank = 0;
      for (int o = 0; o < 32; ++o) {
        const uint32_t ko = __shfl_sync(0xffffffffu, key, o);
        const int32_t jo = __shfl_sync(0xffffffffu, j, o);
        rank += (ko > key) || (ko == key && jo < j);
      }
      if (have && rank < needB) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
      if (kth != nullptr && have && rank == needB - 1) S.lo = key;
    }
    if (kth != nullptr) {
      Sync::sync();
      *kth = S.lo;
    }
    thr = 0;
    need_tie = 0;
    return;
  }
  uint32_t lo = blo, hi = bhi, nd = needB;
  narrow<Sync>(p, S, nullptr, 0, lo, hi, nd);
  for_each_candidate(S, [&](uint32_t key, int32_t j) {
    if (key > lo && key <= bhi) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    else if (key == lo) atomicOr(&S.tie[j >> 5], 1u << (j & 31));
  });
  thr = lo;
  need_tie = nd;
  if (kth != nullptr) *kth = lo;
}

// Exact threshold among the list keys of the boundary bin: histogram levels
// over key bits [20:10] and [9:0] below the bin's 11 bits.
template <class Sync>
__device__ __forceinline__ void resolve_bin(Sel& S, uint32_t& lo, uint32_t& nd) {
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int level = 0; level < 2; ++level) {
    const int shift = level == 0 ? 10 : 0;
    const int nbits = level == 0 ? 11 : 10;
    const uint32_t nb = 1u << nbits;
    const uint32_t keep = ~((1u << (shift + nbits)) - 1u);  // bits fixed so far
    for (uint32_t i = tid; i < nb; i += THREADS) S.hist[i] = 0;
    if (tid == 0) {
      S.lo = lo;
      S.need = nd;
    }
    Sync::sync();
    for_each_candidate(S, [&](uint32_t key, int32_t) {
      if ((key & keep) == (lo & keep)) atomicAdd(&S.hist[(key >> shift) & (nb - 1u)], 1u);
    });
    Sync::sync();
    const uint32_t per = nb / THREADS;
    uint32_t mine = 0;
    for (uint32_t i = 0; i < per; ++i) mine += S.hist[tid * per + i];
    uint32_t incl = mine, dummy = 0, tot, td;
    block_scan2<Sync>(incl, dummy, S.red, tot, td);
    const uint32_t above = tot - incl;
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
    Sync::sync();
    lo = S.lo;
    nd = S.need;
    Sync::sync();
  }
}

// Exact selection reading the row from global memory; when have_hist the
// 11-bit histogram of the row (pass A) is already in S.hist / S.total.
template <class Sync>
__device__ __forceinline__ void exact_select(const Params& p, Sel& S, const float* row, int len, bool have_hist,
                                             uint32_t& thr, uint32_t& need_tie) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t k = (uint32_t)p.k;
  thr = 0;
  need_tie = 0;
  if (!have_hist) {
    for (int i = tid; i < HBINS; i += THREADS) S.hist[i] = 0;
    if (tid == 0) {
      S.zeros = 0;
      S.total = 0;
    }
    Sync::sync();
    uint32_t cnt = 0, zc = 0;
    for_each_score(p, row, len, [&](int, float x) {
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
    Sync::sync();
  }
  if (tid == 0) S.hist[ZERO_KEY >> HSHIFT] += S.zeros;
  if (tid < NWARPS) S.seg_cnt[tid] = 0;
  Sync::sync();
  const uint32_t total = S.total;
  const bool take_all = total <= k;
  if (!take_all) find_bin<Sync>(S, k);
  const uint32_t sel_bin = take_all ? 0u : S.sel_bin;
  const uint32_t need = take_all ? 0u : k - S.sel_above;  // keys to take from the boundary bin
  // pass B: mark higher bins, gather the boundary bin
  for_each_score(p, row, len, [&](int j, float x) {
    const uint32_t key = score_key(x);
    const uint32_t bin = key >> HSHIFT;
    if (key && (take_all || bin > sel_bin)) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    warp_append(S, key && !take_all && bin == sel_bin, key, j);
  });
  Sync::sync();
  if (take_all) return;
  bool overflow;
  list_size(S, overflow);
  uint32_t lo = sel_bin << HSHIFT, nd = need;
  const uint32_t top = lo | ((1u << HSHIFT) - 1u);
  if (!overflow) {
    resolve_bin<Sync>(S, lo, nd);
  } else {
    uint32_t hi = top;
    narrow<Sync>(p, S, row, len, lo, hi, nd);
  }
  auto mark = [&](uint32_t key, int32_t j) {
    if (key > lo && key <= top) atomicOr(&S.gt[j >> 5], 1u << (j & 31));
    else if (key == lo && key) atomicOr(&S.tie[j >> 5], 1u << (j & 31));
  };
  if (!overflow) for_each_candidate(S, mark);
  else for_each_score(p, row, len, [&](int j, float x) { mark(score_key(x), j); });
  thr = lo;
  need_tie = nd;
}

// Bitmap -> ascending column list (ties beyond need_tie dropped from the top),
// -1 padding; the bitmap words are cleared for the next row on the way.
template <class Sync>
__device__ __forceinline__ void write_row(const Params& p, Sel& S, int32_t* out, int nwords, uint32_t need_tie) {
  const int tid = threadIdx.x;
  const uint32_t k = (uint32_t)p.k;
  const int wpt = (nwords + THREADS - 1) / THREADS;
  const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);
  uint32_t ties = 0, sel = 0;
  for (int w = w0; w < w1; ++w) {
    ties += __popc(S.tie[w]);
    sel += __popc(S.gt[w]);
  }
  uint32_t t_incl = ties, g_incl = sel, t_tot, g_tot;
  block_scan2<Sync>(t_incl, g_incl, S.red, t_tot, g_tot);
  uint32_t pos, s_tot = g_tot;
  if (t_tot > 0) {  // keep the lowest need_tie ties
    const uint32_t ties_before = t_incl - ties;
    uint32_t tie_left = need_tie > ties_before ? need_tie - ties_before : 0u;
    sel = 0;
    for (int w = w0; w < w1; ++w) {
      uint32_t tw = S.tie[w];
      while (tw && (uint32_t)__popc(tw) > tie_left) tw &= ~(1u << (31 - __clz(tw)));
      tie_left -= (uint32_t)__popc(tw);
      S.tie[w] = tw;
      sel += (uint32_t)__popc(S.gt[w] | tw);
    }
    uint32_t s_incl = sel, d1 = 0, d1_tot;
    block_scan2<Sync>(s_incl, d1, S.red, s_tot, d1_tot);
    pos = s_incl - sel;
  } else {
    pos = g_incl - sel;
  }
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = S.gt[w] | S.tie[w];
    S.gt[w] = 0;
    S.tie[w] = 0;
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < k) out[pos] = w * 32 + b;
      ++pos;
    }
  }
  for (uint32_t s = min(s_tot, k) + tid; s < k; s += THREADS) out[s] = -1;
}

__device__ __forceinline__ float next_prediction(uint32_t thr) {
  const float tv = thr ? key_value(thr) : 0.f;
  return (thr & 0x80000000u) && tv > 0.f ? tv * PREDICT_MARGIN : 0.f;
}

__device__ __forceinline__ int row_len(const Params& p, int64_t r) {
  return p.lengths != nullptr ? min(max(__ldg(p.lengths + r), 0), p.W) : p.W;
}

// Reset the per-row state that the fast path relies on (before a barrier).
__device__ __forceinline__ void start_row(Sel& S) {
  const int tid = threadIdx.x;
  for (int i = tid; i < HBINS; i += THREADS) S.hist[i] = 0;
  if (tid < NWARPS) S.seg_cnt[tid] = 0;
  if (tid == 0) {
    S.kmax = 0;
    S.zeros = 0;
    S.total = 0;
    S.n_small = 0;
  }
}

// -------------------------------------------------------------- general kernel

__global__ void __launch_bounds__(THREADS, ROWS_CTAS_PER_SM) topk_rows_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Sel& S = *reinterpret_cast<Sel*>(smem_raw);
  const int tid = threadIdx.x;
  const uint32_t k = (uint32_t)p.k;
  const int64_t r_begin = (int64_t)blockIdx.x * p.rows / gridDim.x;
  const int64_t r_end = (int64_t)(blockIdx.x + 1) * p.rows / gridDim.x;
  float pred = p.pred_state ? p.pred_state[blockIdx.x] : 0.f;
  for (int i = tid; i < BM_WORDS; i += THREADS) S.gt[i] = S.tie[i] = 0;

  // list mode: the rows another pass could not resolve, exact path only
  const uint32_t n_list = p.row_list ? *(volatile const uint32_t*)p.row_count : 0u;
  const int64_t i_begin = p.row_list ? blockIdx.x : r_begin;
  const int64_t i_end = p.row_list ? (int64_t)n_list : r_end;
  const int64_t i_step = p.row_list ? gridDim.x : 1;
  if (p.row_list) pred = 0.f;
  for (int64_t i = i_begin; i < i_end; i += i_step) {
    const int64_t r = p.row_list ? (int64_t)p.row_list[i] : i;
    const float* row = p.scores + r * p.stride;
    const int len = row_len(p, r);
    start_row(S);
    __syncthreads();
    uint32_t thr = 0, need_tie = 0;
    bool done = false;
    if (pred > 0.f) {
      uint32_t kmax = 0;
      for_each_score(p, row, len, [&](int j, float x) { fast_visit1(S, x, j, pred, kmax); });
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if ((tid & 31) == 0) atomicMax(&S.kmax, kmax);
      __syncthreads();
      bool overflow;
      if (list_size(S, overflow) >= k && !overflow) {
        resolve_candidates<BlockSync>(p, S, __float_as_uint(pred) | 0x80000000u, thr, need_tie);
        done = true;
      }
      __syncthreads();
    }
    if (!done) exact_select<BlockSync>(p, S, row, len, false, thr, need_tie);
    __syncthreads();
    if (!done && !p.row_list) pred = next_prediction(thr);  // a miss refreshes the prediction
    write_row<BlockSync>(p, S, p.idx + r * p.idx_stride, (len + 31) >> 5, need_tie);
    __syncthreads();
  }
  if (p.pred_state && !p.row_list && tid == 0) p.pred_state[blockIdx.x] = pred;
}

constexpr size_t ROWS_SMEM_BYTES = sizeof(Sel);

// -------------------------------------------------------------- pipelined kernel
//
// topk_pipe_kernel (rows 16-byte aligned, W a multiple of 4), two CTAs per
// SM.  Resolving a row (short phases between barriers) takes about as long as
// streaming it (measured: ~13k cycles each per row at W = 26,624), so when
// the same warps do both, the copies stall while a row resolves.  Here the
// roles are split so the two overlap:
//  * a producer warp streams the CTA's rows as 16 KB bulk copies into a
//    3-slot ring, without pausing between rows;
//  * 8 filtering warps compare every score with the prediction and append
//    candidates to a staging list (warp w owns list segment w; positions
//    from a warp scan of the lanes' counts);
//  * 8 selecting warps (threads 0..255, the helpers above) take the staged
//    list of row r (copying it frees the staging list for row r+1) and
//    resolve it while the filtering warps already read row r+1.
// A row whose list misses (fewer than k candidates, or a full segment) is
// filtered once more from L2 by the selecting warps with the threshold moved
// toward its k-th value (x 0.85 below, x 1.08 above the prediction), and only
// if that misses too goes to the exact path; rows without a prediction take
// the exact path.  The prediction used for row r+1 is the one known when its
// filtering starts (a miss refreshes it, as in the rows kernel).

constexpr int PIPE_SEL_WARPS = NWARPS;   // threads 0 .. 255
constexpr int PIPE_FILT_WARPS = 8;
constexpr int PIPE_FILT_THREADS = PIPE_FILT_WARPS * 32;
constexpr int PIPE_SEGS = NWARPS / PIPE_FILT_WARPS;      // list segments per filtering warp
constexpr int PIPE_WARP_CAP = PIPE_SEGS * SEG;
constexpr int PIPE_THREADS = (PIPE_SEL_WARPS + PIPE_FILT_WARPS + 1) * 32;
constexpr int PIPE_CTAS_PER_SM = 2;
constexpr int PNST = 3;                  // ring slots
constexpr uint32_t FILTER_BAR = 2;       // named barrier of the filtering warps
constexpr float REFILTER_DOWN = 0.85f;
constexpr float REFILTER_UP = 1.08f;
static_assert(PIPE_SEGS * PIPE_FILT_WARPS == NWARPS, "the filtering warps own every list segment");

struct PipeList {   // one row's candidates as the filtering warps leave them
  uint32_t key[CAP];
  int32_t idx[CAP];
  uint32_t cnt[PIPE_FILT_WARPS];  // entries appended by each filtering warp (may pass PIPE_WARP_CAP)
  uint32_t kmax;
  float pred;                     // the threshold the row was filtered with (0: none)
  int stop;
};

struct PipeSmem {
  float ring[PNST * CHUNK];
  uint64_t full[PNST];
  uint64_t empty[PNST];
  uint64_t list_full;
  uint64_t list_empty;
  float pred_next;                // the latest prediction (written by the selecting warps)
  PipeList F;
  Sel sel;
};

constexpr size_t PIPE_SMEM_BYTES = sizeof(PipeSmem) + 128;
static_assert(PIPE_CTAS_PER_SM * (PIPE_SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs fit an SM's shared memory");

__global__ void __launch_bounds__(PIPE_THREADS, PIPE_CTAS_PER_SM) topk_pipe_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  PipeSmem& M = *reinterpret_cast<PipeSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  Sel& S = M.sel;
  PipeList& F = M.F;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t k = (uint32_t)p.k;
  const int64_t r_begin = (int64_t)blockIdx.x * p.rows / gridDim.x;
  const int64_t r_end = (int64_t)(blockIdx.x + 1) * p.rows / gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < PNST; ++s) {
      mbar_init(&M.full[s], 1);
      mbar_init(&M.empty[s], PIPE_FILT_WARPS);
    }
    mbar_init(&M.list_full, 1);
    mbar_init(&M.list_empty, 1);
    M.pred_next = p.pred_state ? p.pred_state[blockIdx.x] : 0.f;
    S.abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < BM_WORDS; i += PIPE_THREADS) S.gt[i] = S.tie[i] = 0;
  __syncthreads();

  if (warp == PIPE_SEL_WARPS + PIPE_FILT_WARPS) {
    // ================= producer: every chunk of every row, back to back
    if (lane == 0) {
      uint32_t it = 0;
      for (int64_t r = r_begin; r < r_end && !*(volatile int*)&S.abort; ++r) {
        const int len4 = (row_len(p, r) + 3) & ~3;  // within the row: W is a multiple of 4
        const float* row = p.scores + r * p.stride;
        for (int c0 = 0; c0 < len4; c0 += CHUNK, ++it) {
          const int s = it % PNST;
          if (!mbar_wait(&M.empty[s], ((it / PNST) & 1) ^ 1, &S.abort)) {
            if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
            break;
          }
          const uint32_t bytes = (uint32_t)min(CHUNK, len4 - c0) * 4u;
          mbar_arrive_expect_tx(&M.full[s], bytes);
          asm volatile(
              "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  smem_addr(M.ring + s * CHUNK)),
              "l"(row + c0), "r"(bytes), "r"(smem_addr(&M.full[s]))
              : "memory");
        }
      }
      // the last copy into every slot must land before the block may retire
      for (uint32_t i = it > (uint32_t)PNST ? it - PNST : 0u; i < it; ++i)
        if (!mbar_wait(&M.full[i % PNST], (i / PNST) & 1, nullptr)) break;
    }
    __syncwarp();
    return;
  }

  if (warp >= PIPE_SEL_WARPS) {
    // ================= filtering warps
    const int fw = warp - PIPE_SEL_WARPS, ftid = tid - PIPE_SEL_WARPS * 32;
    uint32_t it = 0;
    for (int64_t r = r_begin; r < r_end; ++r) {
      const uint32_t i_row = (uint32_t)(r - r_begin);
      if (ftid == 0) {
        // the staging list is free once the selecting warps copied the previous row
        if (!mbar_wait(&M.list_empty, (i_row & 1) ^ 1, &S.abort) && atomicExch(&S.abort, 1) == 0)
          record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
        F.pred = *(volatile float*)&M.pred_next;
        F.kmax = 0;
        F.stop = *(volatile int*)&S.abort;
      }
      named_barrier_sync(FILTER_BAR, PIPE_FILT_THREADS);
      if (F.stop) break;
      const float pred = F.pred;
      const bool fast = pred > 0.f;
      const int len = row_len(p, r);
      const int len4 = (len + 3) & ~3;
      uint32_t kmax = 0, count = 0;  // count: this warp's list entries (warp-uniform)
      for (int c0 = 0; c0 < len4; c0 += CHUNK, ++it) {
        const int s = it % PNST;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&M.full[s], (it / PNST) & 1, &S.abort));
        if (!ok) {
          if (lane == 0 && atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
        } else if (fast) {
          const float4* ring4 = reinterpret_cast<const float4*>(M.ring + s * CHUNK);
          const bool tail = c0 + CHUNK > len;
          constexpr int U = CHUNK / 4 / PIPE_FILT_THREADS;  // float4 per thread per chunk
          uint32_t mask = 0;  // bit 4u + e: score e of this lane's u-th float4 is a candidate
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int f = u * PIPE_FILT_THREADS + ftid;
            float4 x = ring4[f];
            const int j0 = c0 + 4 * f;
            if (tail) {
              if (j0 >= len) x.x = -INFINITY;
              if (j0 + 1 >= len) x.y = -INFINITY;
              if (j0 + 2 >= len) x.z = -INFINITY;
              if (j0 + 3 >= len) x.w = -INFINITY;
            }
            mask |= (uint32_t)(x.x >= pred) << (4 * u) | (uint32_t)(x.y >= pred) << (4 * u + 1) |
                    (uint32_t)(x.z >= pred) << (4 * u + 2) | (uint32_t)(x.w >= pred) << (4 * u + 3);
          }
          const uint32_t nl = __popc(mask);
          uint32_t incl = nl;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          uint32_t pos = count + incl - nl;
          count += __shfl_sync(0xffffffffu, incl, 31);
          while (mask) {
            const int b = __ffs(mask) - 1;
            mask &= mask - 1;
            const int f = (b >> 2) * PIPE_FILT_THREADS + ftid;
            const float x = M.ring[s * CHUNK + 4 * f + (b & 3)];
            const uint32_t key = __float_as_uint(x) | 0x80000000u;  // x >= pred > 0
            if (pos < (uint32_t)PIPE_WARP_CAP) {
              F.key[fw * PIPE_WARP_CAP + pos] = key;
              F.idx[fw * PIPE_WARP_CAP + pos] = c0 + 4 * f + (b & 3);
            }
            kmax = max(kmax, key);
            ++pos;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&M.empty[s]);
      }
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) {
        atomicMax(&F.kmax, kmax);
        F.cnt[fw] = count;
      }
      named_barrier_sync(FILTER_BAR, PIPE_FILT_THREADS);
      if (ftid == 0) mbar_arrive(&M.list_full);
    }
    return;
  }

  // ================= 8 selecting warps
  for (int64_t r = r_begin; r < r_end; ++r) {
    const uint32_t i_row = (uint32_t)(r - r_begin);
    const float* row = p.scores + r * p.stride;
    const int len = row_len(p, r);
    start_row(S);
    if (tid == 0) {
      if (!mbar_wait(&M.list_full, i_row & 1, &S.abort) && atomicExch(&S.abort, 1) == 0)
        record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
      S.stop = *(volatile int*)&S.abort;
    }
    ConsumerSync::sync();
    if (S.stop) break;
    // take the staged list: segment 2w + h of filtering warp w holds its
    // entries h * SEG .. h * SEG + SEG - 1
    const float pred = F.pred;
    uint32_t n = 0;
    bool overflow = false;
#pragma unroll
    for (int w = 0; w < PIPE_FILT_WARPS; ++w) {
      n += F.cnt[w];
      overflow |= F.cnt[w] > (uint32_t)PIPE_WARP_CAP;
    }
    const bool hit = pred > 0.f && n >= k && !overflow;
    if (hit) {
      for (int i = tid; i < CAP; i += THREADS) {
        const uint32_t c = F.cnt[i / PIPE_WARP_CAP], slot = (uint32_t)(i % PIPE_WARP_CAP);
        if (slot < c) {
          S.cand_key[i] = F.key[i];
          S.cand_idx[i] = F.idx[i];
        }
      }
      if (tid < NWARPS) {
        const uint32_t c = F.cnt[tid / PIPE_SEGS];
        const uint32_t first = (uint32_t)(tid % PIPE_SEGS) * SEG;
        S.seg_cnt[tid] = c > first ? min(c - first, (uint32_t)SEG) : 0u;
      }
      if (tid == 0) S.kmax = F.kmax;
    }
    ConsumerSync::sync();
    if (tid == 0) mbar_arrive(&M.list_empty);  // the filtering warps may stage the next row

    uint32_t thr = 0, need_tie = 0, kth = 0;
    bool done = false, refreshed = false;
    if (hit) {
      resolve_candidates<ConsumerSync>(p, S, __float_as_uint(pred) | 0x80000000u, thr, need_tie);
      done = true;
    } else if (pred > 0.f) {
      // filter the row once more (from L2) with the threshold moved toward its k-th value
      const float t2 = n < k ? pred * REFILTER_DOWN : pred * REFILTER_UP;
      uint32_t km = 0;
      for_each_score(p, row, len, [&](int j, float x) { fast_visit1(S, x, j, t2, km); });
      km = __reduce_max_sync(0xffffffffu, km);
      if (lane == 0) atomicMax(&S.kmax, km);
      ConsumerSync::sync();
      bool ov2;
      if (list_size(S, ov2) >= k && !ov2) {
        resolve_candidates<ConsumerSync>(p, S, __float_as_uint(t2) | 0x80000000u, thr, need_tie, &kth);
        done = true;
        refreshed = true;
      }
      ConsumerSync::sync();
    }
    if (!done) {
      exact_select<ConsumerSync>(p, S, row, len, false, thr, need_tie);
      kth = thr;
      refreshed = true;
    }
    ConsumerSync::sync();
    if (refreshed && tid == 0) M.pred_next = next_prediction(kth);  // a miss refreshes the prediction
    write_row<ConsumerSync>(p, S, p.idx + r * p.idx_stride, (len + 31) >> 5, need_tie);
    ConsumerSync::sync();
  }
  if (p.pred_state && tid == 0) p.pred_state[blockIdx.x] = M.pred_next;
}

// -------------------------------------------------------------- two-pass kernels (caller workspace)
//
// With a workspace (qsa_topk_ws) the aligned-row selection runs in three
// launches, so that no CTA both streams a row and resolves one:
//  * topk_filter_kernel (four CTAs per SM): a producer warp streams the rows
//    as 16 KB bulk copies into a 3-slot ring; 8 filtering warps compare every
//    score with the prediction, write the candidates (key and column) to the
//    row's list in the workspace (up to 4096: warp w owns list segment w of
//    512, positions from a warp scan) and count them in a 256-bin histogram
//    of key offsets above the prediction (bins of 2^15 key steps: one
//    binade, the last bin taking everything above).  At the end of a row the
//    histogram gives the bin of its k-th key, so the prediction for the next
//    row follows every row: 0.88 x the bin's lower edge, kept unchanged while
//    it stays within 0.8 .. 0.93 of that edge (on the 4 x 4,096-row
//    workload's rows: ~1,200 candidates per row, 1.7% of rows short of k and
//    none over a segment; 0.85 .. 0.75 .. 0.9 gave 1,480 candidates and 0.4%
//    short, a little slower overall).  A row without a prediction, with fewer
//    than k candidates or with a full segment is marked for the exact pass.
//  * topk_list_kernel: one warp per row, no block barriers: the stored
//    histogram gives the boundary bin, one pass over the list marks the
//    columns of higher bins in the warp's column bitmap and sets the boundary
//    bin's entries aside, the warp ranks those (at most 32, else the row goes
//    to the exact pass; larger key first, then lower column) and writes the
//    bitmap out in ascending order.
//  * topk_rows_kernel in list mode: the exact path over the marked rows.

constexpr int TP_FILT_WARPS = 8;
constexpr int TP_THREADS = (TP_FILT_WARPS + 1) * 32;
constexpr int TP_CTAS_PER_SM = 4;
constexpr int TP_NST = 3;
constexpr int TP_CAP = 4096;          // staged candidates per row (global memory, so roomier than CAP)
constexpr int TP_SEG = TP_CAP / TP_FILT_WARPS;
constexpr int TP_BINS = 256;
constexpr int TP_SHIFT = 15;
constexpr float TP_MARGIN = 0.88f;
constexpr float TP_KEEP_LO = 0.8f;
constexpr float TP_KEEP_HI = 0.93f;
constexpr uint32_t TP_FILTER_BAR = 1;
constexpr int TP_LIST_WARPS = 8;
constexpr int TP_LIST_CTAS_PER_SM = 4;

struct TpRowHdr {        // one row's staged list (64 bytes)
  uint32_t cnt[TP_FILT_WARPS];  // entries appended by each filtering warp (may pass TP_SEG)
  uint32_t kmax;
  float pred;            // the threshold the row was filtered with
  uint32_t status;       // 0: the list holds every selected column; 1: exact pass
  uint32_t pad[5];
};
static_assert(sizeof(TpRowHdr) == 64, "row header size");

// Workspace of the two-pass kernels for `rows` rows (offsets multiples of 256 bytes).
struct TpLayout {
  size_t hdr, hist, ent, count, list, pred, total;
};
constexpr int TP_PRED_FLOATS = 1024;   // per-CTA predictions carried from one call to the next
__host__ __device__ inline size_t tp_round(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline TpLayout tp_layout(int64_t rows) {
  TpLayout L;
  const size_t r = rows > 0 ? (size_t)rows : 0;
  L.hdr = 0;
  L.hist = tp_round(L.hdr + r * sizeof(TpRowHdr));
  L.ent = tp_round(L.hist + r * TP_BINS * 4);   // uint2 {key, column} per staged candidate
  L.count = tp_round(L.ent + r * TP_CAP * 8);
  L.list = tp_round(L.count + 4);
  L.pred = tp_round(L.list + r * 4);
  L.total = tp_round(L.pred + TP_PRED_FLOATS * 4);
  return L;
}

__device__ __forceinline__ uint32_t tp_bin(uint32_t key, uint32_t key_lo) {
  return min((key - key_lo) >> TP_SHIFT, (uint32_t)(TP_BINS - 1));
}

struct TpSmem {
  float ring[TP_NST * CHUNK];
  uint64_t full[TP_NST];
  uint64_t empty[TP_NST];
  uint32_t hist[TP_BINS];
  uint32_t cnt[TP_FILT_WARPS];
  uint32_t kmax;
  float pred;        // this row's threshold
  float pred_next;   // the next row's
  int abort;
  int stop;
};
constexpr size_t TP_SMEM_BYTES = sizeof(TpSmem) + 128;

__global__ void __launch_bounds__(TP_THREADS, TP_CTAS_PER_SM) topk_filter_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  TpSmem& M = *reinterpret_cast<TpSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t k = (uint32_t)p.k;
  const TpLayout L = tp_layout(p.rows);
  TpRowHdr* hdrs = reinterpret_cast<TpRowHdr*>(p.ws + L.hdr);
  uint32_t* ghist = reinterpret_cast<uint32_t*>(p.ws + L.hist);
  uint2* gent = reinterpret_cast<uint2*>(p.ws + L.ent);
  const int64_t r_begin = (int64_t)blockIdx.x * p.rows / gridDim.x;
  const int64_t r_end = (int64_t)(blockIdx.x + 1) * p.rows / gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < TP_NST; ++s) {
      mbar_init(&M.full[s], 1);
      mbar_init(&M.empty[s], TP_FILT_WARPS);
    }
    M.abort = 0;
    // a prediction left in the workspace by an earlier call (any bit pattern:
    // only the speed depends on it)
    const float carried = p.pred_state ? p.pred_state[blockIdx.x] : 0.f;
    M.pred_next = carried > 0.f && carried < 3.0e38f ? carried : 0.f;
    if (blockIdx.x == 0) *reinterpret_cast<uint32_t*>(p.ws + L.count) = 0u;  // the exact pass's row count
    fence_mbar_init();
  }
  for (int i = tid; i < TP_BINS; i += TP_THREADS) M.hist[i] = 0;
  __syncthreads();

  if (warp == TP_FILT_WARPS) {
    // ================= producer: every chunk of every row, back to back
    if (lane == 0) {
      uint32_t it = 0;
      for (int64_t r = r_begin; r < r_end && !*(volatile int*)&M.abort; ++r) {
        const int len4 = (row_len(p, r) + 3) & ~3;  // within the row: W is a multiple of 4
        const float* row = p.scores + r * p.stride;
        for (int c0 = 0; c0 < len4; c0 += CHUNK, ++it) {
          const int s = it % TP_NST;
          if (!mbar_wait(&M.empty[s], ((it / TP_NST) & 1) ^ 1, &M.abort)) {
            if (atomicExch(&M.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
            break;
          }
          const uint32_t bytes = (uint32_t)min(CHUNK, len4 - c0) * 4u;
          mbar_arrive_expect_tx(&M.full[s], bytes);
          asm volatile(
              "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  smem_addr(M.ring + s * CHUNK)),
              "l"(row + c0), "r"(bytes), "r"(smem_addr(&M.full[s]))
              : "memory");
        }
      }
      // the last copy into every slot must land before the block may retire
      for (uint32_t i = it > (uint32_t)TP_NST ? it - TP_NST : 0u; i < it; ++i)
        if (!mbar_wait(&M.full[i % TP_NST], (i / TP_NST) & 1, nullptr)) break;
    }
    __syncwarp();
    return;
  }

  // ================= 8 filtering warps
  const int fw = warp;
  uint32_t it = 0;
  for (int64_t r = r_begin; r < r_end; ++r) {
    if (tid == 0) {
      M.pred = M.pred_next;
      M.kmax = 0;
      M.stop = *(volatile int*)&M.abort;
    }
    named_barrier_sync(TP_FILTER_BAR, TP_FILT_WARPS * 32);
    if (M.stop) break;
    const float pred = M.pred;
    const bool fast = pred > 0.f;
    const uint32_t key_lo = __float_as_uint(pred) | 0x80000000u;
    const int len = row_len(p, r);
    const int len4 = (len + 3) & ~3;
    uint2* ent = gent + r * TP_CAP + fw * TP_SEG;
    uint32_t kmax = 0, count = 0;  // kmax: largest candidate key (every score's without a prediction)
    for (int c0 = 0; c0 < len4; c0 += CHUNK, ++it) {
      const int s = it % TP_NST;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&M.full[s], (it / TP_NST) & 1, &M.abort));
      if (!ok) {
        if (lane == 0 && atomicExch(&M.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
      } else {
        const float4* ring4 = reinterpret_cast<const float4*>(M.ring + s * CHUNK);
        const bool tail = c0 + CHUNK > len;
        constexpr int U = CHUNK / 4 / (TP_FILT_WARPS * 32);  // float4 per thread per chunk
        uint32_t mask = 0;  // bit 4u + e: score e of this lane's u-th float4 is a candidate
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int f = u * TP_FILT_WARPS * 32 + tid;
          float4 x = ring4[f];
          const int j0 = c0 + 4 * f;
          if (tail) {
            if (j0 >= len) x.x = -INFINITY;
            if (j0 + 1 >= len) x.y = -INFINITY;
            if (j0 + 2 >= len) x.z = -INFINITY;
            if (j0 + 3 >= len) x.w = -INFINITY;
          }
          if (fast) {
            mask |= (uint32_t)(x.x >= pred) << (4 * u) | (uint32_t)(x.y >= pred) << (4 * u + 1) |
                    (uint32_t)(x.z >= pred) << (4 * u + 2) | (uint32_t)(x.w >= pred) << (4 * u + 3);
          } else {
            kmax = max(kmax, max(max(score_key(x.x), score_key(x.y)), max(score_key(x.z), score_key(x.w))));
          }
        }
        if (fast) {
          const uint32_t nl = __popc(mask);
          uint32_t incl = nl;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          uint32_t pos = count + incl - nl;
          count += __shfl_sync(0xffffffffu, incl, 31);
          while (mask) {
            const int b = __ffs(mask) - 1;
            mask &= mask - 1;
            const int f = (b >> 2) * TP_FILT_WARPS * 32 + tid;
            const float x = M.ring[s * CHUNK + 4 * f + (b & 3)];
            const uint32_t key = __float_as_uint(x) | 0x80000000u;  // x >= pred > 0
            atomicAdd(&M.hist[tp_bin(key, key_lo)], 1u);
            if (pos < (uint32_t)TP_SEG) ent[pos] = make_uint2(key, (uint32_t)(c0 + 4 * f + (b & 3)));
            kmax = max(kmax, key);
            ++pos;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&M.empty[s]);
    }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
      M.cnt[fw] = count;
      atomicMax(&M.kmax, kmax);
    }
    named_barrier_sync(TP_FILTER_BAR, TP_FILT_WARPS * 32);
    // ---- end of the row: header, histogram, the next row's prediction
    uint32_t n = 0;
    bool overflow = false;
#pragma unroll
    for (int w = 0; w < TP_FILT_WARPS; ++w) {
      n += M.cnt[w];
      overflow |= M.cnt[w] > (uint32_t)TP_SEG;
    }
    const bool exact = !fast || n < k || overflow;
    ghist[r * TP_BINS + tid] = M.hist[tid];
    if (warp == 0) {
      float next = M.pred_next;
      if (!fast) {
        const uint32_t km = M.kmax;  // the row's largest score: a first guess
        next = (km & 0x80000000u) && key_value(km) > 0.f ? 0.5f * key_value(km) : 0.f;
      } else if (n < k) {
        next = 2 * n >= k ? pred * 0.8f : 0.f;  // far too high (a stale carried value): start over from the max
      } else {
        // the bin holding the k-th candidate (lane l: bins 255 - 8l .. 248 - 8l)
        uint32_t c[TP_BINS / 32], sum = 0;
#pragma unroll
        for (int b = 0; b < TP_BINS / 32; ++b) {
          c[b] = M.hist[TP_BINS - 1 - (TP_BINS / 32) * lane - b];
          sum += c[b];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - sum;
        uint32_t bsel = 0, acc = excl;
        bool found = false;
#pragma unroll
        for (int b = 0; b < TP_BINS / 32; ++b) {
          const bool here = !found && acc + c[b] >= k;
          if (here) bsel = TP_BINS - 1 - (TP_BINS / 32) * lane - b;
          if (!found && !here) acc += c[b];
          found = found || here;
        }
        const unsigned who = __ballot_sync(0xffffffffu, excl < k && k <= incl);
        bsel = __shfl_sync(0xffffffffu, bsel, who ? __ffs(who) - 1 : 0);
        if (bsel == (uint32_t)(TP_BINS - 1)) {
          next = pred * 1.5f;  // the k-th key lies a binade or more above the threshold
        } else {
          const float edge = key_value(key_lo + (bsel << TP_SHIFT));
          if (!(pred >= TP_KEEP_LO * edge && pred <= TP_KEEP_HI * edge)) next = TP_MARGIN * edge;
        }
      }
      if (lane == 0) {
        M.pred_next = next;
        TpRowHdr h;
#pragma unroll
        for (int w = 0; w < TP_FILT_WARPS; ++w) h.cnt[w] = M.cnt[w];
        h.kmax = M.kmax;
        h.pred = pred;
        h.status = exact ? 1u : 0u;
#pragma unroll
        for (int i = 0; i < 5; ++i) h.pad[i] = 0;
        hdrs[r] = h;
      }
    }
    named_barrier_sync(TP_FILTER_BAR, TP_FILT_WARPS * 32);
    M.hist[tid] = 0;  // the next row's histogram (appends begin after the next barrier)
  }
  if (p.pred_state && tid == 0) p.pred_state[blockIdx.x] = M.pred_next;
}

// Per-warp shared memory of the list kernel: the small buffers, then a column
// bitmap of tp_bitmap_words(W) words.
struct TpListWarp {
  uint32_t small_key[32];
  int32_t small_col[32];
  uint32_t n_small;
  uint32_t pad[3];
  uint32_t bm[1];          // tp_bitmap_words(W) words
};
__host__ __device__ inline int tp_bitmap_words(int W) { return (((W + 31) >> 5) + 3) & ~3; }
__host__ __device__ inline size_t tp_list_warp_bytes(int W) {
  return offsetof(TpListWarp, bm) + (size_t)tp_bitmap_words(W) * 4;
}

__global__ void __launch_bounds__(TP_LIST_WARPS * 32, TP_LIST_CTAS_PER_SM) topk_list_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  TpListWarp& S = *reinterpret_cast<TpListWarp*>(smem_raw + (size_t)warp * tp_list_warp_bytes(p.W));
  const int bmw = tp_bitmap_words(p.W);
  const uint32_t k = (uint32_t)p.k;
  const TpLayout L = tp_layout(p.rows);
  const TpRowHdr* hdrs = reinterpret_cast<const TpRowHdr*>(p.ws + L.hdr);
  const uint32_t* ghist = reinterpret_cast<const uint32_t*>(p.ws + L.hist);
  const uint2* gent = reinterpret_cast<const uint2*>(p.ws + L.ent);
  uint32_t* miss_count = reinterpret_cast<uint32_t*>(p.ws + L.count);
  int32_t* miss_rows = reinterpret_cast<int32_t*>(p.ws + L.list);
  for (int i = lane; i < bmw; i += 32) S.bm[i] = 0;
  if (lane == 0) S.n_small = 0;
  __syncwarp();
  const int64_t nw = (int64_t)gridDim.x * TP_LIST_WARPS;
  for (int64_t r = (int64_t)blockIdx.x * TP_LIST_WARPS + warp; r < p.rows; r += nw) {
    // the row's header and histogram in one round trip
    const TpRowHdr* h = hdrs + r;
    const uint32_t status = __ldg(&h->status);
    const float hpred = __ldg(&h->pred);
    const uint32_t cnt_l = lane < TP_FILT_WARPS ? __ldg(&h->cnt[lane]) : 0u;
    uint32_t c[TP_BINS / 32];
#pragma unroll
    for (int b = 0; b < TP_BINS / 32; ++b) c[b] = __ldg(ghist + r * TP_BINS + TP_BINS - 1 - (TP_BINS / 32) * lane - b);
    uint32_t B = 0, needB = 0;
    bool exact = status != 0u;
    if (!exact) {
      // the bin of the k-th candidate and how many of its entries to take
      uint32_t sum = 0;
#pragma unroll
      for (int b = 0; b < TP_BINS / 32; ++b) sum += c[b];
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - sum;
      uint32_t bsel = 0, acc = excl, csel = 0;
      bool found = false;
#pragma unroll
      for (int b = 0; b < TP_BINS / 32; ++b) {
        const bool here = !found && acc + c[b] >= k;
        if (here) {
          bsel = TP_BINS - 1 - (TP_BINS / 32) * lane - b;
          csel = c[b];
        }
        if (!found && !here) acc += c[b];
        found = found || here;
      }
      const unsigned who = __ballot_sync(0xffffffffu, excl < k && k <= incl);
      const int src = who ? __ffs(who) - 1 : 0;
      B = __shfl_sync(0xffffffffu, bsel, src);
      needB = k - __shfl_sync(0xffffffffu, acc, src);
      const uint32_t nb = __shfl_sync(0xffffffffu, csel, src);
      exact = who == 0u || B == (uint32_t)(TP_BINS - 1) || nb > 32u;
    }
    if (exact) {
      if (lane == 0) miss_rows[atomicAdd(miss_count, 1u)] = (int32_t)r;
      continue;
    }
    const uint32_t key_lo = __float_as_uint(hpred) | 0x80000000u;
    // one pass over the list: higher bins are taken, the boundary bin is set
    // aside.  Entry e of the row (segments back to back) is slot e - pre[s]
    // of segment s; each lane loads TP_BATCH entries before using any.
    const uint32_t my_cnt = min(cnt_l, (uint32_t)TP_SEG);
    uint32_t pre_incl = my_cnt;
#pragma unroll
    for (int o = 1; o < TP_FILT_WARPS; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, pre_incl, o);
      if (lane >= o) pre_incl += y;
    }
    const uint32_t n_all = __shfl_sync(0xffffffffu, pre_incl, TP_FILT_WARPS - 1);
    const uint32_t pre_excl = pre_incl - my_cnt;
    uint32_t first[TP_FILT_WARPS];  // first entry of each segment
#pragma unroll
    for (int sgm = 0; sgm < TP_FILT_WARPS; ++sgm) first[sgm] = __shfl_sync(0xffffffffu, pre_excl, sgm);
    const uint2* rent = gent + r * TP_CAP;
    constexpr int TP_BATCH = 16;
    for (uint32_t e0 = 0; e0 < n_all; e0 += 32 * TP_BATCH) {
      uint32_t key[TP_BATCH];
      int col[TP_BATCH];
#pragma unroll
      for (int u = 0; u < TP_BATCH; ++u) {
        const uint32_t e = e0 + u * 32 + lane;
        // segment of entry e: the last segment whose first entry is <= e
        uint32_t slot = 0;
#pragma unroll
        for (int sgm = 0; sgm < TP_FILT_WARPS; ++sgm)
          if (e >= first[sgm]) slot = (uint32_t)sgm * TP_SEG + (e - first[sgm]);
        const uint2 v = e < n_all ? __ldg(rent + slot) : make_uint2(0u, 0u);
        key[u] = v.x;
        col[u] = (int)v.y;
      }
#pragma unroll
      for (int u = 0; u < TP_BATCH; ++u) {
        if (e0 + u * 32 + lane < n_all) {
          const uint32_t b = tp_bin(key[u], key_lo);
          const int j = col[u];
          if (b > B) {
            atomicOr(&S.bm[j >> 5], 1u << (j & 31));
          } else if (b == B) {
            const uint32_t q = atomicAdd(&S.n_small, 1u);
            S.small_key[q] = key[u];
            S.small_col[q] = j;
          }
        }
      }
    }
    __syncwarp();
    {
      // rank the boundary entries: larger key first, then lower column
      const uint32_t nb = S.n_small;
      const bool have = (uint32_t)lane < nb;
      const uint32_t key = have ? S.small_key[lane] : 0u;
      const int32_t j = have ? S.small_col[lane] : INT32_MAX;
      uint32_t rank = 0;
      for (uint32_t o = 0; o < nb; ++o) {
        const uint32_t ko = S.small_key[o];
        const int32_t jo = S.small_col[o];
        rank += (ko > key) || (ko == key && jo < j);
      }
      if (have && rank < needB) atomicOr(&S.bm[j >> 5], 1u << (j & 31));
    }
    __syncwarp();
    if (lane == 0) S.n_small = 0;
    // the bitmap out in ascending order (exactly k bits are set); words cleared on the way
    const int len = row_len(p, r);
    const int nwords = (len + 31) >> 5;
    const int wpl = (nwords + 31) >> 5;
    const int w0 = min(lane * wpl, nwords), w1 = min(w0 + wpl, nwords);
    uint32_t cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += (uint32_t)__popc(S.bm[w]);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t pos = incl - cnt;
    int32_t* out = p.idx + r * p.idx_stride;
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = S.bm[w];
      S.bm[w] = 0;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < k) out[pos] = w * 32 + b;
        ++pos;
      }
    }
    __syncwarp();
  }
}

}  // namespace topk
}  // namespace qsa
