// Decode / speculative-decode indexer scores over the paged compressed key
// cache (QSA docs, MATE, section "MQA score"; page addressing of vLLM
// qsa_cache.py, "_logical_to_physical_qsa_slots").
//
// Design (memory bound: 256 bytes of key per compressed key, a few bytes of
// score out):
//  * Work unit = (request b, 128 consecutive compressed keys).  Units are
//    numbered request by request; persistent CTA c takes the contiguous range
//    [c*U/G, (c+1)*U/G), so every CTA streams the same number of keys however
//    skewed the context lengths are.  No combine step is needed: every score
//    is independent, so the splits own disjoint output columns.
//  * Warp 0 (TMA producer) reads the page-table entries of 32 upcoming units
//    at once (one lane per unit) and streams each unit's pages into a ring of
//    shared-memory stages with 3-D tensor copies (128-byte swizzle), together
//    with the request's 4 query rows of 4 heads.
//  * Warp 1 issues tcgen05.mma (M = 128 keys, N = 16 = 4 tokens x 4 heads,
//    K = 128 in 8 steps) into one of four 16-column TMEM accumulators.
//  * Warps 2-5 read their 32 TMEM lanes (lane = key), apply ReLU, sum the 4
//    heads, scale, mask with each token's visible count and invalid pages,
//    and store coalesced fp32 rows.  Before the first unit they fill the
//    columns past each request's last unit with -inf.
#pragma once

#include "sm100.cuh"

namespace qsa {
namespace decode {

constexpr int UNIT = 128;                 // keys per work unit (= UMMA M)
constexpr int N_COLS = 16;                // UMMA N: 4 query tokens x 4 heads
constexpr int STAGES = 6;
constexpr int NACC = 4;                   // TMEM accumulators
constexpr int TMEM_COLS = 64;             // NACC * N_COLS
constexpr int NUM_THREADS = 192;          // 6 warps
constexpr int KHALF_BYTES = UNIT * 128;   // one 64-feature half of a unit's keys
constexpr int KEY_STAGE_BYTES = 2 * KHALF_BYTES;
constexpr int QHALF_BYTES = N_COLS * 128;
constexpr int Q_STAGE_BYTES = 2 * QHALF_BYTES;
constexpr int FILL_BLOCK = 1024;          // columns per tail-fill block
constexpr uint32_t IDESC = umma_idesc_bf16_f32(128, N_COLS);

struct Params {
  const int32_t* page_table;
  int64_t pt_stride;
  int32_t max_pages;
  const int32_t* seq_lens;
  int32_t B;
  int32_t Q;
  int32_t log2_ps;
  int64_t num_pages;
  float scale;
  float* out;
  int64_t out_sb;
  int64_t out_st;
  int32_t W;
  int32_t q_mode;   // 0: one 4-D box per K half; 1: one copy per (token, head) row
  int32_t q_bcast_b;
  int32_t q_bcast_t;
  int32_t q_bcast_h;
};

struct SharedState {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full[NACC];
  uint64_t acc_empty[NACC];
  uint32_t tmem_base;
  int abort;
  uint32_t red[NUM_THREADS / 32];
  int b_start;
  int j_start;
  uint32_t u_begin;
  uint32_t u_end;
  uint32_t prod_issued;
  uint32_t mma_consumed;
};

constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * (KEY_STAGE_BYTES + Q_STAGE_BYTES) +
                              sizeof(SharedState);

__device__ __forceinline__ int units_of(const Params& p, int b) {
  int L = max(__ldg(p.seq_lens + b), 0);
  int nk = min(L >> 2, p.W);
  return (nk + UNIT - 1) / UNIT;
}

// Visible compressed keys of query token i of request b (logical position
// seq_len - Q + i).
__device__ __forceinline__ int visible_of(int L, int Q, int i) {
  L = max(L, 0);
  int pos = L - Q + i;
  int v = min((pos + 1) >> 2, L >> 2);  // arithmetic shift == floor division
  return max(v, 0);
}

struct Walk {
  int b, j;
};

// Move w forward by `steps` units, skipping requests without units.
__device__ __forceinline__ void walk_advance(const Params& p, Walk& w, int steps) {
  w.j += steps;
  while (w.b < p.B) {
    int u = units_of(p, w.b);
    if (w.j < u) break;
    w.j -= u;
    ++w.b;
  }
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int w = 0; w < NUM_THREADS / 32; ++w) t += red[w];
  __syncthreads();
  return t;
}

// Inclusive scan over the block; *total receives the block sum.
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* red, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < NUM_THREADS / 32; ++w) {
    if (w < warp) before += red[w];
    all += red[w];
  }
  __syncthreads();
  *total = all;
  return x + before;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* key_stages = smem;
  uint8_t* q_stages = smem + STAGES * KEY_STAGE_BYTES;
  SharedState& S = *reinterpret_cast<SharedState*>(q_stages + STAGES * Q_STAGE_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < NACC; ++a) {
      mbar_init(&S.acc_full[a], 1);
      mbar_init(&S.acc_empty[a], 4);
    }
    S.abort = 0;
    S.prod_issued = 0;
    S.mma_consumed = 0;
    S.b_start = p.B;
    S.j_start = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_q);
  }
  if (p.q_mode == 1) {
    // Rows of query tokens >= Q are never written by the per-row copies:
    // make them zero once (the swizzle only permutes 16-byte chunks within a
    // 128-byte row, so whole rows can be cleared without it).
    for (int i = tid; i < STAGES * Q_STAGE_BYTES / 16; i += NUM_THREADS) {
      int off = i * 16;
      int row = (off % QHALF_BYTES) / 128;
      if (row >= 4 * p.Q) *reinterpret_cast<uint4*>(q_stages + off) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(&S.tmem_base, TMEM_COLS);

  // ---- this CTA's contiguous range of units
  uint32_t mine = 0;
  for (int b = tid; b < p.B; b += NUM_THREADS) mine += units_of(p, b);
  const uint32_t total = block_sum(mine, S.red);
  const uint32_t u_begin = static_cast<uint32_t>((uint64_t)c * total / G);
  const uint32_t u_end = static_cast<uint32_t>((uint64_t)(c + 1) * total / G);
  if (u_begin < u_end) {
    uint32_t carry = 0;
    for (int base = 0; base < p.B; base += NUM_THREADS) {
      int b = base + tid;
      uint32_t v = b < p.B ? (uint32_t)units_of(p, b) : 0u;
      uint32_t chunk_total;
      uint32_t incl = block_scan(v, S.red, &chunk_total) + carry;
      uint32_t excl = incl - v;
      if (v > 0 && u_begin >= excl && u_begin < incl) {
        S.b_start = b;
        S.j_start = (int)(u_begin - excl);
      }
      carry += chunk_total;
      if (carry > u_begin) break;  // uniform across the block
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;
  const Walk start{S.b_start, S.j_start};
  const uint32_t n_units = u_end - u_begin;

  if (warp == 0) {
    // =========================== TMA producer
    Walk w = start;
    uint32_t it = 0;
    const int ps = 1 << p.log2_ps;
    const int ppu = UNIT >> p.log2_ps;  // pages per unit (2..16)
    bool stop = false;
    for (uint32_t u0 = 0; u0 < n_units && !stop; u0 += 32) {
      Walk wl = w;
      walk_advance(p, wl, lane);
      const bool active = u0 + lane < n_units;
      int pages[16];
      int nvalid = 0;
      if (active) {
        const int L = max(__ldg(p.seq_lens + wl.b), 0);
        const int nk = min(L >> 2, p.W);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pages[i] = -1;
          if (i < ppu) {
            const int n_first = wl.j * UNIT + i * ps;
            const int logical = n_first >> p.log2_ps;
            if (n_first < nk && logical < p.max_pages) {
              int e = __ldg(p.page_table + (int64_t)wl.b * p.pt_stride + logical);
              if (e >= 0 && (int64_t)e < p.num_pages) {
                pages[i] = e;
                ++nvalid;
              }
            }
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) pages[i] = -1;
      }
      const int n_here = min(32u, n_units - u0);
      for (int l = 0; l < n_here; ++l) {
        const int b_l = __shfl_sync(0xffffffffu, wl.b, l);
        const int nv_l = __shfl_sync(0xffffffffu, nvalid, l);
        int pg[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pg[i] = __shfl_sync(0xffffffffu, pages[i], l);
        if (lane == 0) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S.empty[s], ph ^ 1, &S.abort)) {
            if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          } else {
            const int qrows = p.q_mode == 0 ? 16 : 4 * p.Q;
            const uint32_t bytes = (uint32_t)nv_l * ps * 256 + (uint32_t)qrows * 256;
            mbar_arrive_expect_tx(&S.full[s], bytes);
            uint8_t* kdst = key_stages + s * KEY_STAGE_BYTES;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (i < ppu && pg[i] >= 0) {
                tma_load_3d(kdst + i * ps * 128, &S.full[s], &tm_k, 0, 0, pg[i]);
                tma_load_3d(kdst + KHALF_BYTES + i * ps * 128, &S.full[s], &tm_k, 64, 0, pg[i]);
              }
            }
            uint8_t* qdst = q_stages + s * Q_STAGE_BYTES;
            const int qb = p.q_bcast_b ? 0 : b_l;
            if (p.q_mode == 0) {
              tma_load_4d(qdst, &S.full[s], &tm_q, 0, 0, 0, qb);
              tma_load_4d(qdst + QHALF_BYTES, &S.full[s], &tm_q, 64, 0, 0, qb);
            } else {
              for (int t = 0; t < p.Q; ++t)
                for (int h = 0; h < 4; ++h) {
                  const int ct = p.q_bcast_t ? 0 : t, ch = p.q_bcast_h ? 0 : h;
                  tma_load_4d(qdst + (t * 4 + h) * 128, &S.full[s], &tm_q, 0, ch, ct, qb);
                  tma_load_4d(qdst + QHALF_BYTES + (t * 4 + h) * 128, &S.full[s], &tm_q, 64, ch, ct, qb);
                }
            }
            S.prod_issued = it + 1;
          }
        }
        __syncwarp();
        if (__shfl_sync(0xffffffffu, *(volatile int*)&S.abort, 0)) {  // one decision for the warp
          stop = true;
          break;
        }
        ++it;
      }
      walk_advance(p, w, 32);
    }
  } else if (warp == 1) {
    // =========================== MMA issuer
    if (lane == 0) {
      uint32_t last_acc = 0xffffffffu;
      for (uint32_t it = 0; it < n_units; ++it) {
        const int s = it % STAGES, a = it % NACC;
        if (!mbar_wait(&S.full[s], (it / STAGES) & 1, &S.abort) ||
            !mbar_wait(&S.acc_empty[a], ((it / NACC) & 1) ^ 1, &S.abort)) {
          if (atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t kbase = smem_addr(key_stages + s * KEY_STAGE_BYTES);
        const uint32_t qbase = smem_addr(q_stages + s * Q_STAGE_BYTES);
        const uint32_t d = tmem_base + a * N_COLS;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t half = kk >> 2, within = (kk & 3) * 32;
          umma_bf16(d, umma_desc_sw128(kbase + half * KHALF_BYTES + within),
                    umma_desc_sw128(qbase + half * QHALF_BYTES + within), IDESC, kk > 0 ? 1u : 0u);
        }
        umma_commit(&S.empty[s]);
        umma_commit(&S.acc_full[a]);
        last_acc = it;
        S.mma_consumed = it + 1;
      }
      if (last_acc != 0xffffffffu) {
        // make sure the last MMAs have landed before TMEM is released
        if (!mbar_wait(&S.acc_full[last_acc % NACC], (last_acc / NACC) & 1, nullptr))
          record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // =========================== epilogue (warps 2..5)
    const int et = tid - 64;            // 0..127
    const int quad = warp & 3;          // TMEM lane quadrant this warp may read
    // Tail fill: columns past each request's last unit hold -inf.
    {
      const int blocks_per_row = (p.W + FILL_BLOCK - 1) / FILL_BLOCK;
      const int64_t nblocks = (int64_t)p.B * p.Q * blocks_per_row;
      for (int64_t f = c; f < nblocks; f += G) {
        const int64_t r = f / blocks_per_row;
        const int b = (int)(r / p.Q), t = (int)(r % p.Q);
        const int col0 = (int)(f % blocks_per_row) * FILL_BLOCK;
        const int cov = units_of(p, b) * UNIT;
        const int lo = max(cov, col0), hi = min(col0 + FILL_BLOCK, p.W);
        float* row = p.out + (int64_t)b * p.out_sb + (int64_t)t * p.out_st;
        for (int n = lo + et; n < hi; n += 128) row[n] = -INFINITY;
      }
    }
    // Per-unit metadata (request, first key, context length, valid-page
    // bits) is read 32 units at a time, lane l holding unit it0 + l, so no
    // global load sits between an accumulator and its stores.
    Walk w = start;
    const int ps = 1 << p.log2_ps;
    const int ppu = UNIT >> p.log2_ps;
    for (uint32_t it0 = 0; it0 < n_units; it0 += 32) {
      Walk wl = w;
      walk_advance(p, wl, lane);
      int m_len = 0;
      uint32_t m_valid = 0;
      if (it0 + lane < n_units) {
        m_len = __ldg(p.seq_lens + wl.b);
        const int nk = min(max(m_len, 0) >> 2, p.W);
        for (int i = 0; i < ppu; ++i) {
          const int n_first = wl.j * UNIT + i * ps;
          const int logical = n_first >> p.log2_ps;
          if (n_first < nk && logical < p.max_pages) {
            const int e = __ldg(p.page_table + (int64_t)wl.b * p.pt_stride + logical);
            if (e >= 0 && (int64_t)e < p.num_pages) m_valid |= 1u << i;
          }
        }
      }
      const int n_here = (int)min(32u, n_units - it0);
      bool stop = false;
      for (int l = 0; l < n_here; ++l) {
        const uint32_t it = it0 + l;
        const int a = it % NACC;
        // the TMEM load below is warp-collective: leave together or not at all
        if (!__all_sync(0xffffffffu, mbar_wait(&S.acc_full[a], (it / NACC) & 1, &S.abort))) {
          if (lane == 0 && atomicExch(&S.abort, 1) == 0) record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
          stop = true;
          break;
        }
        tc_fence_after();
        float v[16];
        tmem_ld16(tmem_base + ((uint32_t)(quad * 32) << 16) + a * N_COLS, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.acc_empty[a]);

        const int b = __shfl_sync(0xffffffffu, wl.b, l);
        const int j = __shfl_sync(0xffffffffu, wl.j, l);
        const int L = __shfl_sync(0xffffffffu, m_len, l);
        const uint32_t valid = __shfl_sync(0xffffffffu, m_valid, l);
        const int r = quad * 32 + lane;                 // key row within the unit
        const int n = j * UNIT + r;
        const bool page_ok = (valid >> (r >> p.log2_ps)) & 1u;
        if (n < p.W) {
          float* o = p.out + (int64_t)b * p.out_sb + n;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (t < p.Q) {
              const float sc = head_sum_relu(v[4 * t], v[4 * t + 1], v[4 * t + 2], v[4 * t + 3], p.scale);
              o[(int64_t)t * p.out_st] = (page_ok && n < visible_of(L, p.Q, t)) ? sc : -INFINITY;
            }
          }
        }
      }
      if (stop) break;
      walk_advance(p, w, 32);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (S.abort && tid == 0) {
    // let tensor copies that were issued but never consumed finish
    for (uint32_t it = S.mma_consumed; it < S.prod_issued; ++it)
      if (!mbar_wait(&S.full[it % STAGES], (it / STAGES) & 1, nullptr)) break;
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace decode
}  // namespace qsa
