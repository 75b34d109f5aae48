// Prefill indexer scores: packed query rows against shared keys, one key
// interval per row (QSA docs, MATE, section "MQA score": "qsa_mqa_prefill
// takes packed queries, shared keys and per-row key intervals").
//
// A dense bf16 contraction, so it runs on the 5th-generation tensor cores:
//  * Keys are the UMMA M side (128 keys per tile, TMEM lane = key) and the
//    64 query tokens x 4 heads of a token tile are the N side (N = 256), so
//    each epilogue thread owns one key and finds the 4 head products of a
//    token in 4 adjacent TMEM columns: the head sum needs no shuffles.
//  * The token tile's queries (64 KB) stay in shared memory while 128-key
//    tiles stream through a 4-stage TMA ring; two 256-column TMEM
//    accumulators let the epilogue of one tile overlap the MMAs of the next.
//  * Work = every (token tile, key tile) pair that meets at least one row's
//    interval, in token-tile order.  Each CTA computes that list from ks/ke
//    itself and takes an equal contiguous share of it, so the grid is
//    balanced to one tile and never needs a grid-wide barrier.
//  * Warp 0 issues TMA, warp 1 issues tcgen05.mma, warps 2-9 run the
//    epilogue: ReLU, head sum, scale, interval mask, coalesced fp32 stores.
//    Before their first tile they write -inf into the columns of their share
//    of rows that no key covers.
#pragma once

#include "sm100.cuh"

namespace qsa {
namespace prefill {

constexpr int BM = 128;              // keys per tile (UMMA M)
constexpr int BT = 64;               // tokens per tile
constexpr int BN = BT * 4;           // UMMA N
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + EPI_WARPS * 32;
constexpr int NUM_WARPS = NUM_THREADS / 32;
constexpr int KHALF_BYTES = BM * 128;
constexpr int K_STAGE_BYTES = 2 * KHALF_BYTES;
constexpr int QHALF_BYTES = BN * 128;
constexpr int Q_BYTES = 2 * QHALF_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int MAX_TT = 2048;         // token tiles per launch
constexpr int64_t MAX_ROWS_PER_LAUNCH = (int64_t)MAX_TT * BT;
constexpr uint32_t IDESC = umma_idesc_bf16_f32(BM, BN);

struct Params {
  const int32_t* ks;   // rows of this launch
  const int32_t* ke;
  int32_t q_row0;      // first query row of this launch in the query tensor map
  int64_t T;           // rows in this launch
  int64_t Nk;
  float scale;
  float* out;
  int64_t out_stride;
  int32_t W;
};

struct SharedState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t q_full;
  uint64_t q_empty;
  uint32_t tmem_base;
  int abort;
  uint32_t prod_issued;
  uint32_t mma_consumed;
  uint32_t prefix[MAX_TT + 1];  // exclusive prefix of key tiles per token tile
  int32_t kt_lo[MAX_TT];        // first key tile of each token tile
};

constexpr size_t SMEM_BYTES = 1024 + Q_BYTES + STAGES * K_STAGE_BYTES + sizeof(SharedState);

// Keys row t scores: [lo, hi) = [max(ks,0), min(ke, Nk, ks + W)), empty when
// hi <= lo.  Columns are relative to ks, so keys at column >= W are skipped.
__device__ __forceinline__ void row_range(const Params& p, int64_t t, int32_t& ks, int32_t& lo, int32_t& hi) {
  ks = __ldg(p.ks + t);
  const int32_t ke = __ldg(p.ke + t);
  const int64_t l = ks > 0 ? ks : 0;
  int64_t h = ke < p.Nk ? (int64_t)ke : p.Nk;
  const int64_t wcut = (int64_t)ks + p.W;
  if (wcut < h) h = wcut;
  if (h < l) h = l;
  lo = (int32_t)l;
  hi = (int32_t)h;
}

struct Walk {
  int tt;   // token tile
  int i;    // key tile index within the token tile's range
};

__device__ __forceinline__ int tile_count(const SharedState& S, int tt) {
  return (int)(S.prefix[tt + 1] - S.prefix[tt]);
}

__device__ __forceinline__ void walk_next(const SharedState& S, int ntt, Walk& w) {
  ++w.i;
  while (w.tt < ntt && w.i >= tile_count(S, w.tt)) {
    w.i = 0;
    ++w.tt;
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_tile = smem;
  uint8_t* k_stages = smem + Q_BYTES;
  SharedState& S = *reinterpret_cast<SharedState*>(k_stages + STAGES * K_STAGE_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int ntt = (int)((p.T + BT - 1) / BT);

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], EPI_WARPS);
    }
    mbar_init(&S.q_full, 1);
    mbar_init(&S.q_empty, 1);
    S.abort = 0;
    S.prod_issued = 0;
    S.mma_consumed = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == 1) tmem_alloc(&S.tmem_base, TMEM_COLS);

  // ---- plan: key-tile range of every token tile (4 tiles per warp pass)
  for (int tt0 = warp * 4; tt0 < ntt; tt0 += NUM_WARPS * 4) {
    int32_t lo_v[8], hi_v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int tt = tt0 + (k >> 1);
      const int64_t t = (int64_t)tt * BT + (k & 1) * 32 + lane;
      lo_v[k] = INT32_MAX;
      hi_v[k] = INT32_MIN;
      if (tt < ntt && t < p.T) {
        int32_t ks, lo, hi;
        row_range(p, t, ks, lo, hi);
        if (hi > lo) {
          lo_v[k] = lo;
          hi_v[k] = hi;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tt = tt0 + j;
      const int lo = __reduce_min_sync(0xffffffffu, min(lo_v[2 * j], lo_v[2 * j + 1]));
      const int hi = __reduce_max_sync(0xffffffffu, max(hi_v[2 * j], hi_v[2 * j + 1]));
      if (lane == 0 && tt < ntt) {
        if (hi > lo) {
          S.kt_lo[tt] = lo / BM;
          S.prefix[tt + 1] = (uint32_t)((hi + BM - 1) / BM - lo / BM);
        } else {
          S.kt_lo[tt] = 0;
          S.prefix[tt + 1] = 0;
        }
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefix over token tiles (counts sit in prefix[1..ntt])
    const int per = (ntt + 31) / 32;
    const int b0 = lane * per, b1 = min(b0 + per, ntt);
    uint32_t sum = 0;
    for (int i = b0; i < b1; ++i) sum += S.prefix[i + 1];
    uint32_t x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    // each lane rewrites only the slots it read: prefix[i+1] becomes the
    // running sum through token tile i
    uint32_t run = x - sum;
    for (int i = b0; i < b1; ++i) {
      run += S.prefix[i + 1];
      S.prefix[i + 1] = run;
    }
    if (lane == 0) S.prefix[0] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;
  const uint32_t total = S.prefix[ntt];
  const uint32_t u_begin = (uint32_t)((uint64_t)c * total / G);
  const uint32_t u_end = (uint32_t)((uint64_t)(c + 1) * total / G);
  const uint32_t n_units = u_end - u_begin;
  Walk start{ntt, 0};
  if (n_units > 0) {
    int lo = 0, hi = ntt - 1;  // last tt with prefix[tt] <= u_begin
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (S.prefix[mid] <= u_begin) lo = mid;
      else hi = mid - 1;
    }
    start.tt = lo;
    start.i = (int)(u_begin - S.prefix[lo]);
    while (start.tt < ntt && start.i >= tile_count(S, start.tt)) {
      start.i -= tile_count(S, start.tt);
      ++start.tt;
    }
  }

  if (warp == 0) {
    // =========================== TMA producer
    if (lane == 0) {
      Walk w = start;
      int cur_tt = -1;
      uint32_t q_loads = 0;
      for (uint32_t it = 0; it < n_units; ++it) {
        if (w.tt != cur_tt) {
          if (q_loads > 0 && !mbar_wait(&S.q_empty, (q_loads - 1) & 1, &S.abort)) {
            if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&S.q_full, Q_BYTES);
          tma_load_3d(q_tile, &S.q_full, &tm_q, 0, 0, p.q_row0 + w.tt * BT);
          tma_load_3d(q_tile + QHALF_BYTES, &S.q_full, &tm_q, 64, 0, p.q_row0 + w.tt * BT);
          ++q_loads;
          cur_tt = w.tt;
        }
        const int s = it % STAGES;
        if (!mbar_wait(&S.empty[s], ((it / STAGES) & 1) ^ 1, &S.abort)) {
          if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          break;
        }
        const int kt = S.kt_lo[w.tt] + w.i;
        mbar_arrive_expect_tx(&S.full[s], K_STAGE_BYTES);
        uint8_t* dst = k_stages + s * K_STAGE_BYTES;
        tma_load_2d(dst, &S.full[s], &tm_k, 0, kt * BM);
        tma_load_2d(dst + KHALF_BYTES, &S.full[s], &tm_k, 64, kt * BM);
        S.prod_issued = it + 1;
        walk_next(S, ntt, w);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // =========================== MMA issuer
    if (lane == 0) {
      Walk w = start;
      int cur_tt = -1;
      uint32_t q_uses = 0;
      uint32_t last = 0xffffffffu;
      const uint32_t qbase = smem_addr(q_tile);
      for (uint32_t it = 0; it < n_units; ++it) {
        if (w.tt != cur_tt) {
          if (cur_tt >= 0) umma_commit(&S.q_empty);  // old queries free once prior MMAs finish
          if (!mbar_wait(&S.q_full, q_uses & 1, &S.abort)) {
            if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
            break;
          }
          ++q_uses;
          cur_tt = w.tt;
        }
        const int s = it % STAGES, a = it & 1;
        if (!mbar_wait(&S.full[s], (it / STAGES) & 1, &S.abort) ||
            !mbar_wait(&S.acc_empty[a], ((it >> 1) & 1) ^ 1, &S.abort)) {
          if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t kbase = smem_addr(k_stages + s * K_STAGE_BYTES);
        const uint32_t d = tmem_base + a * BN;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t half = kk >> 2, within = (kk & 3) * 32;
          umma_bf16(d, umma_desc_sw128(kbase + half * KHALF_BYTES + within),
                    umma_desc_sw128(qbase + half * QHALF_BYTES + within), IDESC, kk > 0 ? 1u : 0u);
        }
        umma_commit(&S.empty[s]);
        umma_commit(&S.acc_full[a]);
        last = it;
        S.mma_consumed = it + 1;
        walk_next(S, ntt, w);
      }
      if (last != 0xffffffffu && !mbar_wait(&S.acc_full[last & 1], (last >> 1) & 1, nullptr))
        record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // =========================== epilogue (warps 2..9)
    const int e = warp - 2;          // 0..7
    const int quad = warp & 3;       // TMEM lanes this warp may read
    const int half = e >> 2;         // which 32 tokens of the tile
    // -inf for columns no key covers, rows spread over all epilogue warps
    {
      const int64_t gw = (int64_t)c * EPI_WARPS + e, nw = (int64_t)G * EPI_WARPS;
      for (int64_t t = gw; t < p.T; t += nw) {
        int32_t ks, lo, hi;
        row_range(p, t, ks, lo, hi);
        const int64_t vlo = min((int64_t)lo - ks, (int64_t)p.W);
        const int64_t vhi = max((int64_t)hi - ks, vlo);
        float* row = p.out + t * p.out_stride;
        for (int64_t j = lane; j < vlo; j += 32) row[j] = -INFINITY;
        for (int64_t j = vhi + lane; j < p.W; j += 32) row[j] = -INFINITY;
      }
    }
    Walk w = start;
    int cur_tt = -1;
    // this warp's 32 rows of the current token tile: lane l holds row l
    int32_t r_ks = 0, r_lo = 0, r_hi = 0;
    bool fast_rows = false;   // all 32 rows present with one ks
    int32_t w_max_lo = 0, w_min_hi = 0;
    for (uint32_t it = 0; it < n_units; ++it) {
      if (w.tt != cur_tt) {
        const int64_t t = (int64_t)w.tt * BT + half * 32 + lane;
        r_ks = 0;
        r_lo = 0;
        r_hi = 0;
        if (t < p.T) row_range(p, t, r_ks, r_lo, r_hi);
        const int32_t ks0 = __shfl_sync(0xffffffffu, r_ks, 0);
        fast_rows = __all_sync(0xffffffffu, t < p.T && r_ks == ks0);
        w_max_lo = __reduce_max_sync(0xffffffffu, r_lo);
        w_min_hi = __reduce_min_sync(0xffffffffu, r_hi);
        cur_tt = w.tt;
      }
      const int a = it & 1;
      // the TMEM loads below are warp-collective: leave together or not at all
      if (!__all_sync(0xffffffffu, mbar_wait(&S.acc_full[a], (it >> 1) & 1, &S.abort))) {
        if (lane == 0 && atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
        break;
      }
      tc_fence_after();
      float v[128];
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + a * BN + half * 128;
      tmem_ld32(taddr + 0, v);
      tmem_ld32(taddr + 32, v + 32);
      tmem_ld32(taddr + 64, v + 64);
      tmem_ld32(taddr + 96, v + 96);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[a]);

      const int kt = S.kt_lo[w.tt] + w.i;
      const int n0 = kt * BM;
      const int n = n0 + quad * 32 + lane;
      const int64_t t0 = (int64_t)w.tt * BT + half * 32;
      if (fast_rows && n0 >= w_max_lo && n0 + BM <= w_min_hi) {
        // every (row, key) of this warp's block is scored: no mask needed
        float* o = p.out + t0 * p.out_stride + (n - __shfl_sync(0xffffffffu, r_ks, 0));
#pragma unroll
        for (int i = 0; i < 32; ++i)
          o[i * p.out_stride] = head_sum_relu(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], p.scale);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int32_t ks_i = __shfl_sync(0xffffffffu, r_ks, i);
          const int32_t lo_i = __shfl_sync(0xffffffffu, r_lo, i);
          const int32_t hi_i = __shfl_sync(0xffffffffu, r_hi, i);
          if (n >= lo_i && n < hi_i)
            p.out[(t0 + i) * p.out_stride + (n - ks_i)] =
                head_sum_relu(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], p.scale);
        }
      }
      walk_next(S, ntt, w);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (S.abort && tid == 0) {
    for (uint32_t it = S.mma_consumed; it < S.prod_issued; ++it)
      if (!mbar_wait(&S.full[it % STAGES], (it / STAGES) & 1, nullptr)) break;
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace prefill
}  // namespace qsa
