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
//    tiles stream through a 3-stage TMA ring; two 256-column TMEM
//    accumulators let the epilogue of one tile overlap the MMAs of the next.
//  * Work = every (token tile, key tile) pair that meets at least one row's
//    interval, in token-tile order.  Each CTA computes that list from ks/ke
//    itself and takes an equal contiguous share of it, so the grid is
//    balanced to one tile and never needs a grid-wide barrier.
//  * Warp 0 issues TMA, warp 1 issues tcgen05.mma, warps 2-17 run the
//    epilogue: ReLU, head sum, scale, interval mask.  The epilogue has 32K
//    accumulator values per tile to turn into 8K scores in the time the
//    tensor core takes for the next tile, so it is kept short: a packed
//    fp32x2 add in the head sum, and each warp writes its 16 x 32 block of
//    scores into its own 2 KB of shared memory and stores it with one TMA
//    tensor store (no per-element address arithmetic).  Blocks whose rows
//    differ in ks, or whose first column is not 16-byte aligned, use plain
//    coalesced stores instead.
//  * Between tiles each epilogue warp writes -inf into the uncovered columns
//    of one row of its share, so that work hides in the epilogue's slack.
#pragma once

#include "sm100.cuh"

namespace qsa {
namespace prefill {

constexpr int BM = 128;              // keys per tile (UMMA M)
constexpr int BT = 64;               // tokens per tile
constexpr int BN = BT * 4;           // UMMA N
constexpr int STAGES = 3;
constexpr int EPI_WARPS = 16;
constexpr int EPI_TOKENS = BT * 4 / EPI_WARPS;  // tokens of a tile per epilogue warp (16)
constexpr int NUM_THREADS = 64 + EPI_WARPS * 32;
constexpr int NUM_WARPS = NUM_THREADS / 32;
constexpr int KHALF_BYTES = BM * 128;
constexpr int K_STAGE_BYTES = 2 * KHALF_BYTES;
constexpr int QHALF_BYTES = BN * 128;
constexpr int Q_BYTES = 2 * QHALF_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int WARP_STAGE_BYTES = EPI_TOKENS * 32 * 4;   // one warp's 16 x 32 fp32 scores
constexpr int STAGING_BYTES = EPI_WARPS * WARP_STAGE_BYTES;
constexpr int MAX_TT = 2048;         // token tiles per launch
constexpr int64_t MAX_ROWS_PER_LAUNCH = (int64_t)MAX_TT * BT;
constexpr uint32_t IDESC = umma_idesc_bf16_f32(BM, BN);
constexpr uint32_t IDESC_F16 = umma_idesc_f16_f32(BM, BN);

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
  int32_t store_map;   // 1: tm_out describes out (W x T fp32, box 32 x 16)
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

constexpr size_t SMEM_BYTES = 1024 + Q_BYTES + STAGES * K_STAGE_BYTES + STAGING_BYTES + sizeof(SharedState);
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

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

// Widen [lo, hi) by the keys a row with interval (ks, ke) scores, if any.
__device__ __forceinline__ void row_span(const Params& p, int32_t ks, int32_t ke, int32_t& lo, int32_t& hi) {
  const int64_t l = ks > 0 ? ks : 0;
  int64_t h = ke < p.Nk ? (int64_t)ke : p.Nk;
  const int64_t wcut = (int64_t)ks + p.W;
  if (wcut < h) h = wcut;
  if (h > l) {
    lo = min(lo, (int32_t)l);
    hi = max(hi, (int32_t)h);
  }
}

// -inf into the columns of row t that no key of its interval covers.
__device__ __forceinline__ void fill_row(const Params& p, int64_t t, int lane) {
  int32_t ks, lo, hi;
  row_range(p, t, ks, lo, hi);
  const int64_t vlo = min((int64_t)lo - ks, (int64_t)p.W);
  const int64_t vhi = max((int64_t)hi - ks, vlo);
  float* row = p.out + t * p.out_stride;
  for (int64_t j = lane; j < vlo; j += 32) row[j] = -INFINITY;
  for (int64_t j = vhi + lane; j < p.W; j += 32) row[j] = -INFINITY;
}

__device__ __forceinline__ int tile_count(const SharedState& S, int tt) {
  return (int)(S.prefix[tt + 1] - S.prefix[tt]);
}

// Position in this CTA's run of (token tile, key tile) units.  Shared memory
// is read only when the token tile changes, so a step costs a few
// instructions on the issue paths.
struct Walk {
  int tt;    // token tile
  int i;     // key tile index within it
  int n;     // key tiles of tt
  int kt0;   // first key tile of tt

  // Normalise (tt, i) for a unit index that may lie past tt's tiles.
  __device__ __forceinline__ void settle(const SharedState& S, int ntt) {
    n = 0;
    while (tt < ntt) {
      n = tile_count(S, tt);
      if (i < n) break;
      i -= n;
      ++tt;
    }
    kt0 = tt < ntt ? S.kt_lo[tt] : 0;
  }
  // Step to the next unit; true when it starts a new token tile.
  __device__ __forceinline__ bool next(const SharedState& S, int ntt) {
    if (++i < n) return false;
    i = 0;
    ++tt;
    settle(S, ntt);
    return true;
  }
  __device__ __forceinline__ int kt() const { return kt0 + i; }
};

template <bool F16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_out, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_tile = smem;
  uint8_t* k_stages = smem + Q_BYTES;
  uint8_t* staging = k_stages + STAGES * K_STAGE_BYTES;
  SharedState& S = *reinterpret_cast<SharedState*>(staging + STAGING_BYTES);

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

  // Launched as a programmatic dependent (the mixed-batch path): wait for the
  // previous kernel's writes (ks, ke and the keys may come from it), then let
  // the next kernel begin launching.  A no-op for an ordinary launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- plan: key-tile range of every token tile.  16 threads share a token
  // tile, 4 rows each; every load of a pass is issued before any is used, so
  // a pass costs one memory round trip.
  {
    constexpr int GROUPS = NUM_THREADS / 16;   // token tiles per unroll step
    constexpr int UNROLL = 4;
    const bool vec = ((reinterpret_cast<uintptr_t>(p.ks) | reinterpret_cast<uintptr_t>(p.ke)) & 15) == 0;
    const int g16 = tid >> 4, l16 = tid & 15;
    for (int tt0 = 0; tt0 < ntt; tt0 += GROUPS * UNROLL) {
      int4 kv[UNROLL], ev[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int tt = tt0 + u * GROUPS + g16;
        const int64_t r = (int64_t)tt * BT + l16 * 4;
        kv[u] = make_int4(0, 0, 0, 0);   // rows past T read as ks = ke = 0: no keys
        ev[u] = kv[u];
        if (tt < ntt && r < p.T) {
          if (vec && r + 4 <= p.T) {
            kv[u] = __ldg(reinterpret_cast<const int4*>(p.ks + r));
            ev[u] = __ldg(reinterpret_cast<const int4*>(p.ke + r));
          } else {
            kv[u].x = __ldg(p.ks + r);
            ev[u].x = __ldg(p.ke + r);
            if (r + 1 < p.T) { kv[u].y = __ldg(p.ks + r + 1); ev[u].y = __ldg(p.ke + r + 1); }
            if (r + 2 < p.T) { kv[u].z = __ldg(p.ks + r + 2); ev[u].z = __ldg(p.ke + r + 2); }
            if (r + 3 < p.T) { kv[u].w = __ldg(p.ks + r + 3); ev[u].w = __ldg(p.ke + r + 3); }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const int tt = tt0 + u * GROUPS + g16;
        int32_t lo = INT32_MAX, hi = INT32_MIN;
        row_span(p, kv[u].x, ev[u].x, lo, hi);
        row_span(p, kv[u].y, ev[u].y, lo, hi);
        row_span(p, kv[u].z, ev[u].z, lo, hi);
        row_span(p, kv[u].w, ev[u].w, lo, hi);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (l16 == 0 && tt < ntt) {
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
  Walk start{ntt, 0, 0, 0};
  if (n_units > 0) {
    int lo = 0, hi = ntt - 1;  // last tt with prefix[tt] <= u_begin
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (S.prefix[mid] <= u_begin) lo = mid;
      else hi = mid - 1;
    }
    start.tt = lo;
    start.i = (int)(u_begin - S.prefix[lo]);
    start.settle(S, ntt);
  }

  if (warp == 0) {
    // =========================== TMA producer
    if (lane == 0) {
      Walk w = start;
      bool new_tt = true;
      uint32_t q_loads = 0;
      int s = 0;
      uint32_t ph = 0;   // fill count of stage s, mod 2
      for (uint32_t it = 0; it < n_units; ++it) {
        if (new_tt) {
          if (q_loads > 0 && !mbar_wait(&S.q_empty, (q_loads - 1) & 1, &S.abort)) {
            if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&S.q_full, Q_BYTES);
          tma_load_3d(q_tile, &S.q_full, &tm_q, 0, 0, p.q_row0 + w.tt * BT);
          tma_load_3d(q_tile + QHALF_BYTES, &S.q_full, &tm_q, 64, 0, p.q_row0 + w.tt * BT);
          ++q_loads;
        }
        if (!mbar_wait(&S.empty[s], ph ^ 1, &S.abort)) {
          if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          break;
        }
        const int kt = w.kt();
        mbar_arrive_expect_tx(&S.full[s], K_STAGE_BYTES);
        uint8_t* dst = k_stages + s * K_STAGE_BYTES;
        tma_load_2d(dst, &S.full[s], &tm_k, 0, kt * BM);
        tma_load_2d(dst + KHALF_BYTES, &S.full[s], &tm_k, 64, kt * BM);
        S.prod_issued = it + 1;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1;
        }
        new_tt = w.next(S, ntt);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // =========================== MMA issuer
    if (lane == 0) {
      Walk w = start;
      bool new_tt = true;
      uint32_t q_uses = 0;
      uint32_t last = 0xffffffffu;
      const uint64_t qdesc = umma_desc_sw128(smem_addr(q_tile));
      const uint64_t kdesc0 = umma_desc_sw128(smem_addr(k_stages));
      int s = 0;
      uint32_t ph = 0;   // fill count of stage s, mod 2
      for (uint32_t it = 0; it < n_units; ++it) {
        if (new_tt) {
          if (it > 0) umma_commit(&S.q_empty);  // old queries free once prior MMAs finish
          if (!mbar_wait(&S.q_full, q_uses & 1, &S.abort)) {
            if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
            break;
          }
          ++q_uses;
        }
        const int a = it & 1;
        if (!mbar_wait(&S.full[s], ph, &S.abort) || !mbar_wait(&S.acc_empty[a], ((it >> 1) & 1) ^ 1, &S.abort)) {
          if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          break;
        }
        tc_fence_after();
        umma_bf16_k128<KHALF_BYTES / 16, QHALF_BYTES / 16>(tmem_base + a * BN,
                                                           kdesc0 + (uint64_t)(s * (K_STAGE_BYTES / 16)), qdesc, F16 ? IDESC_F16 : IDESC);
        umma_commit(&S.empty[s]);
        umma_commit(&S.acc_full[a]);
        last = it;
        S.mma_consumed = it + 1;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1;
        }
        new_tt = w.next(S, ntt);
      }
      if (last != 0xffffffffu && !mbar_wait(&S.acc_full[last & 1], (last >> 1) & 1, nullptr))
        record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // =========================== epilogue (warps 2..17, four per TMEM lane quadrant)
    const int e = warp - 2;          // 0..15
    const int quad = warp & 3;       // TMEM lanes this warp may read
    const int part = e >> 2;         // which 16 tokens of the tile
    float* stage = reinterpret_cast<float*>(staging + e * WARP_STAGE_BYTES);
    // next row whose uncovered columns this warp fills (a launch has < 2^31 rows)
    int32_t fill_t = c * EPI_WARPS + e;
    const int32_t fill_step = G * EPI_WARPS;
    Walk w = start;
    bool new_tt = true;
    // this warp's 16 rows of the current token tile: lane l (and l + 16) holds row l
    int32_t r_ks = 0, r_lo = INT32_MAX, r_hi = INT32_MIN;
    bool any_row = false;     // at least one of the 16 rows exists
    bool uni = false;         // all existing rows share ks0
    bool all_rows = false;    // all 16 rows exist
    int32_t ks0 = 0, w_max_lo = 0, w_min_hi = 0;
    bool store_pending = false;
    for (uint32_t it = 0; it < n_units; ++it) {
      if (new_tt) {
        const int64_t t0 = (int64_t)w.tt * BT + part * EPI_TOKENS;
        const int64_t t = t0 + (lane & (EPI_TOKENS - 1));
        const bool valid = t < p.T;
        r_ks = 0;
        r_lo = INT32_MAX;
        r_hi = INT32_MIN;
        if (valid) row_range(p, t, r_ks, r_lo, r_hi);
        any_row = t0 < p.T;
        all_rows = t0 + EPI_TOKENS <= p.T;
        ks0 = __shfl_sync(0xffffffffu, r_ks, 0);
        uni = __all_sync(0xffffffffu, !valid || r_ks == ks0);
        w_max_lo = __reduce_max_sync(0xffffffffu, valid ? r_lo : INT32_MIN);
        w_min_hi = __reduce_min_sync(0xffffffffu, valid ? r_hi : INT32_MAX);
      }
      const int a = it & 1;
      // the TMEM loads below are warp-collective: leave together or not at all
      if (!__all_sync(0xffffffffu, mbar_wait(&S.acc_full[a], (it >> 1) & 1, &S.abort))) {
        if (lane == 0 && atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
        break;
      }
      tc_fence_after();
      float v[4 * EPI_TOKENS];
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + a * BN + part * 4 * EPI_TOKENS;
      tmem_ld32(taddr + 0, v);
      tmem_ld32(taddr + 32, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[a]);

      const int nb = w.kt() * BM + quad * 32;   // first key of this warp's block
      const int n = nb + lane;
      const int64_t t0 = (int64_t)w.tt * BT + part * EPI_TOKENS;
      const int64_t x = (int64_t)nb - ks0;                      // its column in the rows' output
      const bool unmasked = nb >= w_max_lo && nb + 32 <= w_min_hi;
      if (any_row && p.store_map && uni && x >= 0 && x < p.W && (x & 3) == 0) {
        // one TMA store of the 16 x 32 block; masked cells hold -inf, which
        // is their value, and cells past W or T are clipped by the map
        if (store_pending) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
        if (unmasked) {
#pragma unroll
          for (int i = 0; i < EPI_TOKENS; ++i)
            stage[i * 32 + lane] = head_sum_relu_x2(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], p.scale);
        } else {
#pragma unroll
          for (int i = 0; i < EPI_TOKENS; ++i) {
            const int32_t lo_i = __shfl_sync(0xffffffffu, r_lo, i);
            const int32_t hi_i = __shfl_sync(0xffffffffu, r_hi, i);
            const float sc = head_sum_relu_x2(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], p.scale);
            stage[i * 32 + lane] = (n >= lo_i && n < hi_i) ? sc : -INFINITY;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, stage, (int32_t)x, (int32_t)t0);
          bulk_commit_group();
        }
        store_pending = true;
      } else if (all_rows && uni && unmasked) {
        // every (row, key) of this warp's block is scored: no mask needed
        float* o = p.out + t0 * p.out_stride + (n - ks0);
#pragma unroll
        for (int i = 0; i < EPI_TOKENS; ++i)
          o[i * p.out_stride] = head_sum_relu_x2(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], p.scale);
      } else if (any_row) {
#pragma unroll
        for (int i = 0; i < EPI_TOKENS; ++i) {
          const int32_t ks_i = __shfl_sync(0xffffffffu, r_ks, i);
          const int32_t lo_i = __shfl_sync(0xffffffffu, r_lo, i);
          const int32_t hi_i = __shfl_sync(0xffffffffu, r_hi, i);
          if (n >= lo_i && n < hi_i)
            p.out[(t0 + i) * p.out_stride + (n - ks_i)] =
                head_sum_relu_x2(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], p.scale);
        }
      }
      new_tt = w.next(S, ntt);
      if (fill_t < p.T) {
        fill_row(p, fill_t, lane);
        fill_t += fill_step;
      }
    }
    if (!S.abort)
      for (; fill_t < p.T; fill_t += fill_step) fill_row(p, fill_t, lane);
    if (store_pending && lane == 0) bulk_wait_all();
    __syncwarp();
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
