// Decode / speculative-decode indexer scores over the paged compressed key
// cache (QSA docs, MATE, section "MQA score"; page addressing of vLLM
// qsa_cache.py, "_logical_to_physical_qsa_slots").
//
// Memory bound: 256 bytes of key per compressed key against a few bytes of
// score.  The design keeps as many key bytes in flight as the SM allows and
// touches no shared memory on the way:
//  * Work = the concatenation over requests of 8-key tiles (a tile never
//    straddles a page: page sizes are multiples of 8).  With more than one
//    request and at least twice as many warps as requests, each request is
//    cut into chunks of at most C tiles, C the smallest size for which all
//    chunks fit the grid, and each warp takes one chunk, so skewed context
//    lengths cost nothing extra and no warp pays a second query load;
//    otherwise warps take equal contiguous shares of the tile list.  No
//    combine step is needed (each score is independent).
//  * The kernel is latency-bound for short batches, so the dependent memory
//    round trips are kept to three (lengths, page entries with queries,
//    keys): the lengths load is the first instruction, the query and
//    page-entry loads are issued together, and with at most 32 requests each
//    warp plans its work in registers, with no block barrier.  The -inf
//    columns past each request's keys are stored where DRAM would otherwise
//    idle: by the warps without tiles when there are enough of them, else by
//    half of the warps before their first key loads.
//  * Each lane streams its part of the keys with 16-byte non-caching global
//    loads straight into registers (4 tiles = 256 bytes per lane in flight),
//    in the operand layout of mma.sync.m16n8k16 (B = 16 features x 8 keys).
//    Two loop forms (template PIPE): one batch of 4 tiles loaded, then
//    multiplied; or two half-batches alternating, the next one's loads issued
//    before the current one's math (the same bytes in flight, chosen at
//    launch: the fp8 cache always, bf16 / fp16 when warps get at most one
//    half-batch each).
//  * The request's query rows (4 tokens x 4 heads = M 16) stay in registers
//    as the A operand.  Features are visited in a permuted order, the same for
//    queries and keys, so that every load instruction reads whole 32-byte
//    sectors.
//  * Rows are ordered head-major (row = head * 4 + token), so a lane holds
//    heads h and h + 2 of one token; ReLU, one add, one shfl.xor 16 and the
//    scale give the score, which is masked with the token's visible count and
//    the page validity and stored.
// Tensor-core throughput is not the limit here (at most 4 of the 16 rows
// carry data for one token); the warp-level MMA is used because its operands
// come from registers, which lets the key loads bypass shared memory.
//
// fp8 E4M3 cache (vLLM qsa_cache.py, the state backend's fp8 cache dtypes;
// vLLM qsa_prepare.py, "_to_dst_dtype": stored = e4m3(bf16(k) / k_scale)):
// a lane reads 8 bytes per chunk instead of 16, with 6 tiles in flight as
// two halves of 3 (192 bytes per lane; 8 tiles spill registers and measured
// slower, 4 keep too few bytes in flight).  Every E4M3 value is exact in fp16,
// so keys are widened with one conversion per pair and the MMA runs on fp16.
// The query rows are made fp16 exactly: each row is multiplied by the power
// of two that puts its largest magnitude in [2^15, 2^16) (exact for every
// element within 29 binades of it), and the row's accumulators are multiplied
// back before the ReLU sum.  k_scale > 0 is folded into the score multiplier.
#pragma once

#include <cuda_fp16.h>

#include <type_traits>

#include "sm100.cuh"

namespace qsa {
namespace decode {

constexpr int TILE = 8;                 // keys per tile (mma.sync N)
constexpr int BATCH = 4;                // tiles in flight per warp (bf16 and fp16 keys)
constexpr int WARPS = 16;
constexpr int NUM_THREADS = WARPS * 32;
constexpr int MAX_B = 8192;             // requests per launch (prefix in shared memory)

struct Params {
  const uint16_t* q;        // bf16 bits
  int64_t q_sb, q_st, q_sh;
  const uint16_t* k_cache;  // bf16 bits (bf16 cache)
  const uint8_t* k8;        // E4M3 codes (fp8 cache)
  int64_t k_page_stride, k_row_stride;  // in elements
  int64_t num_pages;
  const int32_t* page_table;
  int64_t pt_stride;
  int32_t max_pages;
  const int32_t* seq_lens;
  int32_t B;
  int32_t Q;
  int32_t log2_ps;          // page size 2^log2_ps (power-of-two instance)
  uint32_t ps;              // page size (any-size instance): key n is in page n / ps, row n % ps
  uint32_t ps_magic;        // n / ps == (n * ps_magic) >> ps_shift for every key index n < 2^31
  int32_t ps_shift;
  float scale;              // fp8 cache: scale * k_scale
  float* out;
  int64_t out_sb;
  int64_t out_st;
  int32_t W;
};

constexpr size_t SMEM_BYTES = sizeof(int32_t) * (MAX_B + 1);

// Element format of q and the key cache: bf16 q and keys, fp16 q and keys,
// or bf16 q over an fp8 E4M3 cache.
enum class Fmt { BF16, F16, E4M3 };

// Keys of a request that can be visible in a column < W: the last query
// token sees seq_len / 4 of them.
__device__ __forceinline__ int scored_keys(const Params& p, int L) {
  return min(max(L, 0) >> 2, p.W);
}

// Visible compressed keys of query token i (logical position seq_len - Q + i).
__device__ __forceinline__ int visible_of(int L, int Q, int i) {
  L = max(L, 0);
  const int pos = L - Q + i;
  return max(min((pos + 1) >> 2, L >> 2), 0);  // arithmetic shift == floor division
}

__device__ __forceinline__ uint4 ld_stream16(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}

__device__ __forceinline__ uint2 ld_stream8(const void* ptr) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(ptr));
  return v;
}

__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four E4M3 codes (byte i = feature i) -> two fp16x2 words (features 0, 1
// and 2, 3), exact: one hardware conversion per pair.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t four, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(four));
}

// bf16x2 word -> fp16x2 word of the two values times dn (a power of two).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, float dn) {
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16) * dn, __uint_as_float(w & 0xffff0000u) * dn);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Power-of-two factors for a query row whose largest bf16 magnitude (bits
// without the sign) is m: dn = 2^(142 - E) with E its exponent field, so the
// row times dn has its largest magnitude in [2^15, 2^16), and up = 1 / dn.
// E is held at >= 16 so that both factors are normal floats.
__device__ __forceinline__ void row_factors(uint32_t m, float& dn, float& up) {
  const int e = max((int)(m >> 7), 16);
  dn = __uint_as_float((uint32_t)(269 - e) << 23);
  up = __uint_as_float((uint32_t)(e - 15) << 23);
}

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane (g, c) = (lane >> 2, lane & 3) reads, for every key and query row it
// serves, the four 16-byte chunks c, c + 4, c + 8, c + 12 of the 128
// features (chunk m = features 8m .. 8m + 7).  Word w (0..15) of those 64
// bytes holds features 8 * (c + 4 * (w >> 2)) + 2 * (w & 3) + {0, 1}.  In
// k-step s the MMA takes words 2s and 2s + 1 as its k = 2c + {0,1} and
// k = 2c + 8 + {0,1} entries, for the queries and the keys alike; over the
// eight k-steps and four lanes every feature is used exactly once.

// Query fragments of request b: A = 16 rows (row = head * 4 + token) x 128.
// fp8 cache: fp16 fragments of the scaled rows, and in up0 / up1 the factors
// that undo the scaling of rows g and g + 8.
template <Fmt F>
__device__ __forceinline__ void load_queries(const Params& p, int b, int lane, uint32_t (&a)[8][4], float& up0,
                                             float& up1) {
  const int g = lane >> 2, c = lane & 3;
  const int t = g & 3, h = g >> 2;  // rows g and g + 8: heads h and h + 2 of token t
  // Rows of tokens t >= Q read token Q - 1 instead (no branch, so the loads
  // stay in flight); their scores are never stored.
  uint32_t w0[16], w1[16];
  const uint16_t* r0 = p.q + b * p.q_sb + min(t, p.Q - 1) * p.q_st + h * p.q_sh;
  const uint16_t* r1 = r0 + 2 * p.q_sh;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(r0 + 8 * (c + 4 * i)));
    const uint4 y = __ldg(reinterpret_cast<const uint4*>(r1 + 8 * (c + 4 * i)));
    w0[4 * i] = x.x; w0[4 * i + 1] = x.y; w0[4 * i + 2] = x.z; w0[4 * i + 3] = x.w;
    w1[4 * i] = y.x; w1[4 * i + 1] = y.y; w1[4 * i + 2] = y.z; w1[4 * i + 3] = y.w;
  }
  if constexpr (F == Fmt::E4M3) {
    uint32_t m0 = 0, m1 = 0;  // largest magnitude bits of rows g and g + 8 (this lane's 32 features)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      m0 = max(m0, max(w0[i] & 0x7fffu, (w0[i] >> 16) & 0x7fffu));
      m1 = max(m1, max(w1[i] & 0x7fffu, (w1[i] >> 16) & 0x7fffu));
    }
    // the row's four lanes c = 0..3 differ in the low two lane bits
    m0 = max(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
    m1 = max(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
    m0 = max(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
    m1 = max(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
    float dn0, dn1;
    row_factors(m0, dn0, up0);
    row_factors(m1, dn1, up1);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      w0[i] = bf16x2_to_f16x2(w0[i], dn0);
      w1[i] = bf16x2_to_f16x2(w1[i], dn1);
    }
  }
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    a[s][0] = w0[2 * s];      // row g,     k = 2c + {0,1}
    a[s][1] = w1[2 * s];      // row g + 8, k = 2c + {0,1}
    a[s][2] = w0[2 * s + 1];  // row g,     k = 2c + 8 + {0,1}
    a[s][3] = w1[2 * s + 1];  // row g + 8, k = 2c + 8 + {0,1}
  }
}

// Logical page of key n and its row in that page.
template <bool GEN>
__device__ __forceinline__ void page_of(const Params& p, int n, int& lp, int& row) {
  if constexpr (GEN) {
    lp = (int)(((uint64_t)(uint32_t)n * p.ps_magic) >> p.ps_shift);
    row = n - lp * (int)p.ps;
  } else {
    lp = n >> p.log2_ps;
    row = n & ((1 << p.log2_ps) - 1);
  }
}

template <Fmt F, bool GEN, bool PIPE>
__global__ void __launch_bounds__(NUM_THREADS, 1) decode_kernel(const Params p) {
  constexpr bool FP8 = F == Fmt::E4M3;
  constexpr int NB = FP8 ? 6 : BATCH;  // tiles in flight per warp (fp8: two halves of 3)
  extern __shared__ int32_t prefix[];  // prefix[b]: tiles before request b
  __shared__ uint32_t red[WARPS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gw = blockIdx.x * WARPS + warp;
  const int nw = gridDim.x * WARPS;

  // Launched as a programmatic dependent (the mixed-batch path): wait for the
  // previous kernel's writes, then let the next kernel begin launching.  A
  // no-op for an ordinary launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- the lengths load goes out first.  With at most 32 requests every
  // warp builds the request plan in its own registers (lane b: request b), so
  // no warp waits for another; otherwise one block-wide scan in shared memory.
  const bool warp_plan = p.B <= 32;
  const int len0 = warp_plan ? (lane < p.B ? __ldg(p.seq_lens + lane) : 0) : (tid < p.B ? __ldg(p.seq_lens + tid) : 0);
  uint32_t total = 0, lp = 0;   // warp plan: lp = tiles before request `lane` (all tiles for lanes >= B)
  if (warp_plan) {
    const uint32_t v = lane < p.B ? (uint32_t)((scored_keys(p, len0) + TILE - 1) / TILE) : 0u;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    lp = x - v;
    total = __shfl_sync(0xffffffffu, x, 31);
  }
  // tiles before request b (b <= B); every lane of the warp calls it
  auto pfx = [&](int b) -> uint32_t {
    if (warp_plan) {
      const uint32_t s = __shfl_sync(0xffffffffu, lp, b & 31);
      return b < 32 ? s : total;
    }
    return (uint32_t)prefix[b];
  };

  // ---- tiles per request and their exclusive prefix (block-wide chunks)
  uint32_t carry = 0;
  if (!warp_plan) {
  for (int base = 0; base < p.B; base += NUM_THREADS) {
    const int b = base + tid;
    uint32_t v = 0;
    if (b < p.B) v = (uint32_t)((scored_keys(p, base == 0 ? len0 : __ldg(p.seq_lens + b)) + TILE - 1) / TILE);
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) red[warp] = x;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      before += w < warp ? red[w] : 0u;
      all += red[w];
    }
    if (b < p.B) prefix[b] = (int32_t)(carry + before + x - v);
    carry += all;
    __syncthreads();
  }
  if (tid == 0) prefix[p.B] = (int32_t)carry;
  __syncthreads();
  total = carry;
  }

  // ---- -inf for the columns past each request's last tile.  With fewer
  // rows than warps, a row's uncovered columns are striped over nw / rows
  // warps in 32-column steps; otherwise each warp takes whole rows.
  auto fill_tail = [&](int fw, int fn) {  // this warp is fw of the fn warps sharing the fill
    const int64_t rows = (int64_t)p.B * p.Q;
    if (rows <= fn) {
      const int r = fw % (int)rows, k0 = fw / (int)rows, ks = fn / (int)rows;
      if (k0 < ks) {
        const int b = r / p.Q, t = r - b * p.Q;
        const int cov = (int)(pfx(b + 1) - pfx(b)) * TILE;
        float* row = p.out + (int64_t)b * p.out_sb + (int64_t)t * p.out_st;
        for (int n = cov + k0 * 32 + lane; n < p.W; n += ks * 32) row[n] = -INFINITY;
      }
    } else {
      for (int64_t r = fw; r < rows; r += fn) {
        const int b = (int)(r / p.Q), t = (int)(r % p.Q);
        const int cov = (int)(pfx(b + 1) - pfx(b)) * TILE;
        float* row = p.out + (int64_t)b * p.out_sb + (int64_t)t * p.out_st;
        for (int n = cov + lane; n < p.W; n += 32) row[n] = -INFINITY;
      }
    }
  };

  // ---- this warp's share of the tiles
  uint32_t t_begin = 0, t_end = 0;
  int b = 0;
  uint32_t used;  // warps that get tiles (the first `used` warps of the grid)
  if (p.B > 1 && 2 * p.B <= nw) {
    // chunks of at most C tiles that never cross a request: C is the least
    // size with sum_b ceil(n_b / C) <= nw; ceil(total / (nw - B)) always fits
    // and is within one of it.
    uint32_t C = max((total + (uint32_t)(nw - p.B) - 1) / (uint32_t)(nw - p.B), 1u);
    // warp index -> (request, chunk): walk the requests with one lane each
    // and a running chunk count (requests are few when this branch runs)
    int found = -1;
    uint32_t chunk0 = 0, w_before = 0;
    for (int base = 0; base < p.B && found < 0; base += 32) {
      const int rb = base + lane;
      // every lane calls pfx (a shuffle in the warp plan); rb + 1 <= B + 31
      // stays inside the shared table, as this branch has 2B <= nw
      const uint32_t p1 = pfx(rb + 1), p0 = pfx(rb);
      const uint32_t nb = rb < p.B ? p1 - p0 : 0u;
      const uint32_t wb = (nb + C - 1) / C;
      uint32_t x = wb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const uint32_t excl = w_before + x - wb;
      const bool mine = rb < p.B && (uint32_t)gw >= excl && (uint32_t)gw < excl + wb;
      const unsigned m = __ballot_sync(0xffffffffu, mine);
      if (m) {
        const int src = __ffs(m) - 1;
        found = base + src;
        chunk0 = (uint32_t)gw - __shfl_sync(0xffffffffu, excl, src);
      }
      w_before += __shfl_sync(0xffffffffu, x, 31);
    }
    used = w_before;  // one chunk per warp
    if (found >= 0) {
      b = found;
      const uint32_t pb = pfx(b), nb = pfx(b + 1) - pb;
      t_begin = pb + chunk0 * C;
      t_end = pb + min((chunk0 + 1) * C, nb);
    }
  } else {
    const uint32_t per = total / (uint32_t)nw, rem = total % (uint32_t)nw;
    used = min(total, (uint32_t)nw);
    t_begin = (uint32_t)gw * per + min((uint32_t)gw, rem);
    t_end = t_begin + per + ((uint32_t)gw < rem ? 1u : 0u);
    if (t_begin < t_end) {
      int lo = 0, hi = p.B - 1;  // last request with prefix[b] <= t_begin
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pfx(mid) <= t_begin) lo = mid;
        else hi = mid - 1;
      }
      b = lo;
      while (pfx(b + 1) <= t_begin) ++b;  // skip requests without tiles
    }
  }
  // The -inf tail goes where DRAM would otherwise idle.  When at least an
  // eighth of the warps get no tiles, those warps write all of it while the
  // others stream keys; otherwise the upper half of each CTA's warps write it
  // now, before the page-entry and query round trips that precede their
  // first key loads, while the lower half go straight to theirs (measured on
  // B200: 16 single-token rows 6.5 -> 6.05 us with idle warps filling; 16 x 4
  // rows of long contexts 14.3 us filling after the keys, 14.0 with every
  // warp filling here, 13.2 with half of them).
  const bool idle_fill = ((uint32_t)nw - used) * 8u >= (uint32_t)nw;
  constexpr int FILL_WARPS = WARPS / 2;
  if (!idle_fill && warp >= WARPS - FILL_WARPS)
    fill_tail(blockIdx.x * FILL_WARPS + warp - (WARPS - FILL_WARPS), gridDim.x * FILL_WARPS);
  if (t_begin >= t_end) {
    if (idle_fill) fill_tail(gw - (int)used, nw - (int)used);
    return;
  }
  int j = (int)(t_begin - pfx(b));
  uint32_t left = t_end - t_begin;
  int ob = b;

  const int g = lane >> 2, c = lane & 3;
  const int t = g & 3;                  // token of this lane's rows
  const int key = 2 * c + (lane >> 4);  // key of a tile this lane stores
  uint32_t qa[8][4];
  float up0 = 1.f, up1 = 1.f;
  load_queries<F>(p, b, lane, qa, up0, up1);
  int L = __ldg(p.seq_lens + b);
  int nt_b = (int)(pfx(b + 1) - pfx(b));
  // Page entries of the current request, read 32 tiles ahead so that no
  // page-table load sits between two batches of key loads.  Power-of-two
  // pages: lane l holds the page of tile j0 + l (a tile never straddles a
  // page).  Any page size >= 8: lane l holds logical page lp0 + l, where lp0
  // is the page of tile j0's first key; 32 pages of >= 8 rows cover the 32
  // tiles j0 .. j0 + 31.
  int j0 = j;
  int entry = -1;
  int lp0 = 0;
  // The raw entry stays a pending load until a batch reads it; the range
  // check happens there.
  auto fetch_entries = [&]() {
    int logical;
    if constexpr (GEN) {
      int row0;
      page_of<true>(p, j0 * TILE, lp0, row0);
      logical = min(lp0 + lane, p.max_pages - 1);
    } else {
      const int tile = min(j0 + lane, nt_b - 1);
      logical = min((tile * TILE) >> p.log2_ps, p.max_pages - 1);
    }
    entry = p.max_pages > 0 ? __ldg(p.page_table + (int64_t)b * p.pt_stride + logical) : -1;
  };
  fetch_entries();

  if constexpr (PIPE) {
    // Two half-batches alternate: the loads of the next one go out before the
    // math of the current one, so a warp always has keys in flight while it
    // multiplies.  A batch never leaves its request; at a request boundary the
    // pipeline drains, the next request's queries load, and it restarts.
    constexpr int HB = NB / 2;  // tiles per half-batch
    using KV = typename std::conditional<FP8, uint2, uint4>::type;
    auto issue = [&](KV (&kv)[HB][4], int& jb, int& cnt, uint32_t& valid) {
      cnt = (int)min((uint32_t)min(min(HB, nt_b - j), 32 - (j - j0)), left);
      jb = j;
      valid = 0;
  #pragma unroll
      for (int u = 0; u < HB; ++u) {
        int lp, row;
        page_of<GEN>(p, (j + u) * TILE + g, lp, row);
        const int src = GEN ? (lp - lp0) & 31 : (j - j0 + u) & 31;
        const int ent = __shfl_sync(0xffffffffu, entry, src);
        const bool ok = lp < p.max_pages && ent >= 0 && (int64_t)ent < p.num_pages;
        valid |= ok ? 1u << u : 0u;
        const int64_t off = (int64_t)ent * p.k_page_stride + (int64_t)row * p.k_row_stride;
        if constexpr (FP8) {
          if (u < cnt && ok) {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv[u][i] = ld_stream8(p.k8 + off + 8 * (c + 4 * i));
          } else {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv[u][i] = make_uint2(0, 0);
          }
        } else {
          if (u < cnt && ok) {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv[u][i] = ld_stream16(p.k_cache + off + 8 * (c + 4 * i));
          } else {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv[u][i] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      j += cnt;
      left -= (uint32_t)cnt;
      if (left > 0) {
        if (j == nt_b) {
          do {
            ++b;
          } while (pfx(b + 1) == pfx(b));
          j = 0;
          j0 = 0;
          nt_b = (int)(pfx(b + 1) - pfx(b));
          fetch_entries();
        } else if (j - j0 == 32) {
          j0 = j;
          fetch_entries();
        }
      }
    };
    auto compute = [&](const KV (&kv)[HB][4], int jb, int cnt, uint32_t valid) {
      const uint32_t vst = GEN ? __shfl_sync(0xffffffffu, valid, key << 2) : valid;
      const int vis = t < p.Q ? visible_of(L, p.Q, t) : 0;
      float d[HB][4];
  #pragma unroll
      for (int v = 0; v < HB; ++v) d[v][0] = d[v][1] = d[v][2] = d[v][3] = 0.f;
  #pragma unroll
      for (int s = 0; s < 8; ++s) {
  #pragma unroll
        for (int v = 0; v < HB; ++v) {
          if constexpr (FP8) {
            const uint32_t four = (s & 1) ? kv[v][s >> 1].y : kv[v][s >> 1].x;
            uint32_t b0, b1;
            e4m3x4_to_f16x2x2(four, b0, b1);
            mma_f16_16816(d[v], qa[s], b0, b1);
          } else if constexpr (F == Fmt::F16) {
            const uint32_t* w = reinterpret_cast<const uint32_t*>(kv[v]);
            mma_f16_16816(d[v], qa[s], w[2 * s], w[2 * s + 1]);
          } else {
            const uint32_t* w = reinterpret_cast<const uint32_t*>(kv[v]);
            mma_bf16_16816(d[v], qa[s], w[2 * s], w[2 * s + 1]);
          }
        }
      }
  #pragma unroll
      for (int v = 0; v < HB; ++v) {
        if (v < cnt) {
          float s0, s1;
          if constexpr (FP8) {
            s0 = fmaxf(d[v][0], 0.f) * up0 + fmaxf(d[v][2], 0.f) * up1;
            s1 = fmaxf(d[v][1], 0.f) * up0 + fmaxf(d[v][3], 0.f) * up1;
          } else {
            s0 = fmaxf(d[v][0], 0.f) + fmaxf(d[v][2], 0.f);
            s1 = fmaxf(d[v][1], 0.f) + fmaxf(d[v][3], 0.f);
          }
          s0 += __shfl_xor_sync(0xffffffffu, s0, 16);  // the other two heads
          s1 += __shfl_xor_sync(0xffffffffu, s1, 16);
          const int n = (jb + v) * TILE + key;
          if (t < p.Q && n < p.W) {
            const float sc = p.scale * ((lane >> 4) ? s1 : s0);
            p.out[(int64_t)ob * p.out_sb + (int64_t)t * p.out_st + n] = ((vst >> v) & 1u) && n < vis ? sc : -INFINITY;
          }
        }
      }
    };
    KV kvA[HB][4], kvB[HB][4];
    int jA = 0, cA = 0, jB = 0, cB = 0;
    uint32_t vA = 0, vB = 0;
    issue(kvA, jA, cA, vA);
    while (true) {
      bool more = left > 0 && b == ob;
      if (more) issue(kvB, jB, cB, vB);
      compute(kvA, jA, cA, vA);
      if (more) {
        more = left > 0 && b == ob;
        if (more) issue(kvA, jA, cA, vA);
        compute(kvB, jB, cB, vB);
        if (more) continue;
      }
      if (left == 0) break;
      // the next request: its queries, then a fresh pipeline
      ob = b;
      L = __ldg(p.seq_lens + b);
      load_queries<F>(p, b, lane, qa, up0, up1);
      issue(kvA, jA, cA, vA);
    }
  } else {
    while (left > 0) {
      const int cnt = (int)min((uint32_t)min(min(NB, nt_b - j), 32 - (j - j0)), left);
      uint4 kv[FP8 ? 1 : NB][4];   // bf16: chunk i = 16 bytes
      uint2 kv8[FP8 ? NB : 1][4];  // fp8: chunk i = 8 bytes
      uint32_t valid = 0;  // bit u: the page of key g of tile u (this lane's loads) is valid
  #pragma unroll
      for (int u = 0; u < NB; ++u) {
        // keys past the request's pages (logical page >= max_pages) and
        // entries outside the pool are invalid
        int lp, row;
        page_of<GEN>(p, (j + u) * TILE + g, lp, row);
        const int src = GEN ? (lp - lp0) & 31 : (j - j0 + u) & 31;
        const int ent = __shfl_sync(0xffffffffu, entry, src);
        const bool ok = lp < p.max_pages && ent >= 0 && (int64_t)ent < p.num_pages;
        valid |= ok ? 1u << u : 0u;
        const int64_t off = (int64_t)ent * p.k_page_stride + (int64_t)row * p.k_row_stride;
        if constexpr (FP8) {
          if (u < cnt && ok) {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv8[u][i] = ld_stream8(p.k8 + off + 8 * (c + 4 * i));
          } else {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv8[u][i] = make_uint2(0, 0);
          }
        } else {
          if (u < cnt && ok) {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv[u][i] = ld_stream16(p.k_cache + off + 8 * (c + 4 * i));
          } else {
  #pragma unroll
            for (int i = 0; i < 4; ++i) kv[u][i] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      // validity of the key this lane stores (key 2c + lane / 16), held by the
      // lanes that loaded it (4 * key .. 4 * key + 3); uniform over a tile
      // when pages hold whole tiles
      const uint32_t vst = GEN ? __shfl_sync(0xffffffffu, valid, key << 2) : valid;
      const int vis = t < p.Q ? visible_of(L, p.Q, t) : 0;
      const int jb = j;
      j += cnt;
      left -= (uint32_t)cnt;
      // next request or next 32 tiles: issue those loads before the math
      if (left > 0) {
        if (j == nt_b) {
          do {
            ++b;
          } while (pfx(b + 1) == pfx(b));
          j = 0;
          j0 = 0;
          nt_b = (int)(pfx(b + 1) - pfx(b));
          fetch_entries();
        } else if (j - j0 == 32) {
          j0 = j;
          fetch_entries();
        }
      }
      // the MMA chains of four tiles interleaved by k-step: four independent
      // accumulators keep the tensor pipe busy instead of waiting on one chain
  #pragma unroll
      for (int u0 = 0; u0 < NB; u0 += BATCH) {
        float d[BATCH][4];
  #pragma unroll
        for (int v = 0; v < BATCH; ++v) d[v][0] = d[v][1] = d[v][2] = d[v][3] = 0.f;
  #pragma unroll
        for (int s = 0; s < 8; ++s) {
  #pragma unroll
          for (int v = 0; v < BATCH; ++v) {
            if constexpr (FP8) {
              // words 2s, 2s + 1 = bytes 0-3 (s even) or 4-7 (s odd) of chunk s / 2
              const uint32_t four = (s & 1) ? kv8[u0 + v][s >> 1].y : kv8[u0 + v][s >> 1].x;
              uint32_t b0, b1;
              e4m3x4_to_f16x2x2(four, b0, b1);
              mma_f16_16816(d[v], qa[s], b0, b1);
            } else if constexpr (F == Fmt::F16) {
              const uint32_t* w = reinterpret_cast<const uint32_t*>(kv[u0 + v]);
              mma_f16_16816(d[v], qa[s], w[2 * s], w[2 * s + 1]);
            } else {
              const uint32_t* w = reinterpret_cast<const uint32_t*>(kv[u0 + v]);
              mma_bf16_16816(d[v], qa[s], w[2 * s], w[2 * s + 1]);
            }
          }
        }
  #pragma unroll
        for (int v = 0; v < BATCH; ++v) {
          const int u = u0 + v;
          if (u < cnt) {
            // d0/d1: head h, keys 2c and 2c+1; d2/d3: head h + 2
            float s0, s1;
            if constexpr (FP8) {
              s0 = fmaxf(d[v][0], 0.f) * up0 + fmaxf(d[v][2], 0.f) * up1;
              s1 = fmaxf(d[v][1], 0.f) * up0 + fmaxf(d[v][3], 0.f) * up1;
            } else {
              s0 = fmaxf(d[v][0], 0.f) + fmaxf(d[v][2], 0.f);
              s1 = fmaxf(d[v][1], 0.f) + fmaxf(d[v][3], 0.f);
            }
            s0 += __shfl_xor_sync(0xffffffffu, s0, 16);  // the other two heads
            s1 += __shfl_xor_sync(0xffffffffu, s1, 16);
            const int n = (jb + u) * TILE + key;
            if (t < p.Q && n < p.W) {
              const float sc = p.scale * ((lane >> 4) ? s1 : s0);
              p.out[(int64_t)ob * p.out_sb + (int64_t)t * p.out_st + n] = ((vst >> u) & 1u) && n < vis ? sc : -INFINITY;
            }
          }
        }
      }
      if (ob != b) {
        ob = b;
        L = __ldg(p.seq_lens + b);
        load_queries<F>(p, b, lane, qa, up0, up1);
      }
    }
  }
}

}  // namespace decode
}  // namespace qsa
