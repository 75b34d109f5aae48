// Core attention after the indexer (QSA docs, MATE, section "Core
// Attention"): the caller keeps the top-scoring compressed blocks, expands
// them to token indices, and attention runs over those tokens only.
//
//  * expand_kernel: block indices [T, k] -> token indices [T, 4k + 3], one
//    warp per row: the four tokens of each kept block, then the row's open
//    group (the tokens after its last complete 4-token group, which no
//    compressed key covers yet), then -1.
//  * attn_kernel: split-KV sparse attention.  One CTA per (row, KV head,
//    split of the row's token list).  The row's query heads of one KV head
//    (up to 16; 12 for the canonical 24 / 2 geometry) are the M = 16 side of
//    mma.sync.m16n8k16, read from shared memory for every chunk (so three
//    CTAs fit an SM).  Each 32-entry chunk of the token list is gathered row
//    by row (512-byte K and V rows found through the page table) with
//    16-byte cp.async copies into a 2-stage shared-memory ring per CTA
//    (XOR-swizzled 16-byte units, so ldmatrix reads are conflict-free;
//    masked entries are zero-filled).  Warp w scores the chunk's tokens
//    8w .. 8w + 7 against all heads, the chunk maximum is exchanged through
//    shared memory, and the probabilities (bf16) are written to shared memory
//    where warp w multiplies them into its 64 output features.  The
//    running maximum, sum and unnormalised output of the split go to a
//    workspace.
//  * combine_kernel: one warp per (row, query head) merges the splits (each
//    weighted by 2^(m_s - M)), applies the sigmoid gate, writes the bf16
//    output and the natural-log LSE (zeros and -inf for a row with no
//    visible token).
// The gather is memory bound (1 KB of K and V per token and KV head against
// 4 * 12 * 256 FLOP), so the warp-level tensor-core MMA is enough; its
// operands come from shared memory the copies land in.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace qsa {
namespace attn {

constexpr int D = 256;            // head dimension
constexpr int CHUNK = 32;         // token-list entries per pipeline stage
constexpr int STAGES = 2;
constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int MAX_GROUP = 16;     // query heads per KV head (the MMA's M)
constexpr int ROW_BYTES = D * 2;  // one K or V row
constexpr int KV_STAGE_BYTES = CHUNK * ROW_BYTES;          // 16 KB for K, 16 KB for V
constexpr int P_STRIDE = CHUNK + 8;                        // bf16 elements per probability row (padded)
constexpr int Q_BYTES = MAX_GROUP * ROW_BYTES;             // 8 KB

struct Params {
  const uint16_t* q;          // bf16 [T, Hq, 256]
  int64_t q_st, q_sh;
  int32_t Hq, Hkv, group;
  const uint16_t* k;          // bf16 [pages, page_size, Hkv, 256]
  const uint16_t* v;
  int64_t num_pages;
  int32_t page_size;
  int64_t kv_page_stride, kv_row_stride, kv_head_stride;   // elements
  const int32_t* page_table;
  int64_t pt_stride;
  int32_t max_pages;
  const int32_t* cu;          // int32 [R + 1]: query rows of request r are cu[r] .. cu[r+1]-1
  const int32_t* seq_lens;    // int32 [R]: tokens of request r (its query rows included)
  int32_t R;
  const int32_t* tok;         // int32 [T, width], request-local token indices, -1 pads
  int64_t tok_stride;
  int32_t width;
  int64_t T;
  int32_t splits;             // splits per (row, KV head)
  int32_t chunks_per_split;
  float scale_log2;           // scale * log2(e)
  float* part_o;              // [T, Hkv, splits, group, 256] unnormalised outputs
  float* part_ml;             // [T, Hkv, splits, group, 2]: running max (log2 units), sum
  // combine
  const float* gate;          // [T, Hq] or null
  uint16_t* out;              // bf16 [T, Hq, 256], row stride out_st, head stride 256
  int64_t out_st;
  float* lse;                 // [T, Hq] or null
};

constexpr size_t SMEM_BYTES = Q_BYTES + STAGES * 2 * KV_STAGE_BYTES + 16 * P_STRIDE * 2 + 1024;

// Request of query row t and the row's logical position (vLLM qsa_cache.py,
// "_logical_positions": seq_len - query_len + i).  Whole warp: the last r
// with cu[r] <= t is found 32 candidates per memory round trip (each step
// samples 32 evenly spaced entries of the remaining range).
__device__ __forceinline__ void row_request(const int32_t* __restrict__ cu, const int32_t* __restrict__ seq_lens,
                                            int R, int64_t t, int lane, int& r, int& pos, int& L) {
  int lo = 0, n = R;  // the answer lies in [lo, lo + n)
  while (n > 1) {
    const int step = (n + 31) >> 5;
    const int idx = lo + lane * step;
    const bool le = idx < lo + n && (int64_t)__ldg(cu + idx) <= t;
    const unsigned m = __ballot_sync(0xffffffffu, le);   // a prefix of the lanes (cu is non-decreasing)
    const int k = 31 - __clz(m);                          // last sample at or before t (lane 0 always is)
    lo += k * step;
    n = min(step, n - k * step);
  }
  r = lo;
  const int first = __ldg(cu + lo);
  const int qlen = __ldg(cu + lo + 1) - first;
  L = __ldg(seq_lens + lo);
  pos = L - qlen + (int)(t - first);
}

// ---------------------------------------------------------------- expansion

constexpr int EXPAND_MAX_K = 512;   // block-hint width limit (QSA docs, "Core Attention")

struct ExpandParams {
  const int32_t* blk;   // [T, k]
  int64_t blk_stride;
  int32_t k;
  const int32_t* cu;
  const int32_t* seq_lens;
  int32_t R;
  int64_t T;
  int32_t* tok;         // [T, 4k + 3]
  int64_t tok_stride;
};

__global__ void __launch_bounds__(256) expand_kernel(const ExpandParams p) {
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (t >= p.T) return;
  int r, pos, L;
  row_request(p.cu, p.seq_lens, p.R, t, lane, r, pos, L);
  const int32_t* src = p.blk + t * p.blk_stride;
  int32_t* dst = p.tok + t * p.tok_stride;
  const int width = 4 * p.k + 3;
  // every block entry of the row (k <= 512: 16 per lane) in one round trip
  int bv[EXPAND_MAX_K / 32];
#pragma unroll
  for (int u = 0; u < EXPAND_MAX_K / 32; ++u) {
    const int i = u * 32 + lane;
    bv[u] = i < p.k ? __ldg(src + i) : -1;
  }
  int n = 0;  // tokens written so far (warp-uniform)
#pragma unroll
  for (int u = 0; u < EXPAND_MAX_K / 32; ++u) {
    const int b = bv[u];
    const unsigned keep = __ballot_sync(0xffffffffu, b >= 0);
    if (b >= 0) {
      const int at = n + 4 * __popc(keep & ((1u << lane) - 1u));
      const int4 four = make_int4(4 * b, 4 * b + 1, 4 * b + 2, 4 * b + 3);
      dst[at] = four.x;
      dst[at + 1] = four.y;
      dst[at + 2] = four.z;
      dst[at + 3] = four.w;
    }
    n += 4 * __popc(keep);
  }
  // the open group: positions 4 * visible .. pos, visible = max(0, min((pos+1)/4, L/4))
  if (pos >= 0) {
    const int vis = max(0, min((pos + 1) >> 2, L >> 2));
    const int open = pos + 1 - 4 * vis;
    if (lane < open && n + lane < width) dst[n + lane] = 4 * vis + lane;
    n += max(open, 0);
  }
  for (int j = n + lane; j < width; j += 32) dst[j] = -1;
}

// ---------------------------------------------------------------- attention

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte unit u (0..31) of row n in a 512-byte-row matrix
// whose units are XOR-swizzled by the row's low 3 bits: the 8 rows an
// ldmatrix phase reads land in 8 different bank groups.
__device__ __forceinline__ uint32_t swz(int n, int u) { return (uint32_t)(n * ROW_BYTES + ((u ^ (n & 7)) << 4)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(THREADS, 3) attn_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* q_s = smem;
  uint8_t* kv_s = smem + Q_BYTES;                                   // stage s: K at 2s, V at 2s + 1
  uint16_t* p_s = reinterpret_cast<uint16_t*>(kv_s + STAGES * 2 * KV_STAGE_BYTES);
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(p_s) + 16 * P_STRIDE * 2);  // [WARPS][16]
  uint8_t* valid_s = reinterpret_cast<uint8_t*>(red + WARPS * 16 * 2);  // [STAGES][CHUNK]: entry visible

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t cta = blockIdx.x;
  const int split = (int)(cta % p.splits);
  const int g = (int)((cta / p.splits) % p.Hkv);
  const int64_t t = cta / ((int64_t)p.splits * p.Hkv);

  int r, pos, L;
  row_request(p.cu, p.seq_lens, p.R, t, lane, r, pos, L);

  // ---- queries of KV head g: rows h < group, zero rows above
  {
    const uint16_t* qrow = p.q + t * p.q_st + (int64_t)g * p.group * p.q_sh;
#pragma unroll
    for (int i = 0; i < (MAX_GROUP * 32) / THREADS; ++i) {
      const int unit = tid + i * THREADS;  // 16 rows x 32 units
      const int h = unit >> 5, u = unit & 31;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (h < p.group) v = __ldg(reinterpret_cast<const uint4*>(qrow + h * p.q_sh + u * 8));
      *reinterpret_cast<uint4*>(q_s + swz(h, u)) = v;
    }
  }

  // ---- this split's entries of the row's token list
  const int e_begin = split * p.chunks_per_split * CHUNK;
  const int e_end = min(p.width, e_begin + p.chunks_per_split * CHUNK);
  const int nchunks = e_end > e_begin ? (e_end - e_begin + CHUNK - 1) / CHUNK : 0;
  const int32_t* tok_row = p.tok + t * p.tok_stride;
  const int32_t* pt_row = p.page_table + (int64_t)r * p.pt_stride;

  // Warp w gathers token slots n = w + 4i (i < 8) of every chunk, one K row
  // and one V row per slot (32 lanes x 16 bytes each).  Their row offsets
  // are found four chunks (a window) at a time: lane l resolves slot
  // w + 4 (l & 7) of chunk 4 win + (l >> 3), list entry first, then page
  // entry, and the loads shuffle them out.  The two dependent loads of a
  // window run a window ahead: its list entries are loaded when the previous
  // window starts and its page entries two chunks later, so no chunk waits
  // on them.
  auto tok_of = [&](int win) -> int {
    const int c = 4 * win + (lane >> 3);
    const int e = e_begin + c * CHUNK + warp + WARPS * (lane & 7);
    return e < e_end ? __ldg(tok_row + e) : -1;
  };
  auto page_of = [&](int j) -> int {
    if (j < 0 || j > pos || j >= L) return -1;
    const int lp = j / p.page_size;
    return lp < p.max_pages ? __ldg(pt_row + lp) : -1;
  };
  auto offset_of = [&](int j, int page) -> int64_t {
    if (j < 0 || j > pos || j >= L || page < 0 || (int64_t)page >= p.num_pages) return -1;
    const int lp = j / p.page_size;
    return (int64_t)page * p.kv_page_stride + (int64_t)(j - lp * p.page_size) * p.kv_row_stride +
           (int64_t)g * p.kv_head_stride;
  };
  int64_t win_off = -1;                          // this window's offsets (-1: masked)
  int tok_nx = tok_of(0), page_nx = -1;          // the next window's entries as they arrive
  page_nx = page_of(tok_nx);
  win_off = offset_of(tok_nx, page_nx);
  tok_nx = tok_of(1);
  // Gather chunk c into stage s (chunks are loaded in order 0, 1, 2, ...).
  auto load_chunk = [&](int c, int s) {
    if ((c & 3) == 0 && c > 0) {                 // window c / 4 begins: its pages were looked up
      win_off = offset_of(tok_nx, page_nx);
      tok_nx = tok_of((c >> 2) + 1);
    } else if ((c & 3) == 2) {
      page_nx = page_of(tok_nx);                 // page entries of the next window
    }
    const uint32_t kbase = smem_addr(kv_s + (2 * s) * KV_STAGE_BYTES);
    const uint32_t vbase = smem_addr(kv_s + (2 * s + 1) * KV_STAGE_BYTES);
    const int u = lane;
#pragma unroll
    for (int i = 0; i < CHUNK / WARPS; ++i) {
      const int n = warp + WARPS * i;  // token slot in the chunk
      const int64_t off = __shfl_sync(0xffffffffu, win_off, (c & 3) * 8 + i);
      const bool ok = off >= 0;
      const uint16_t* ksrc = ok ? p.k + off + u * 8 : p.k;
      const uint16_t* vsrc = ok ? p.v + off + u * 8 : p.v;
      cp_async16(kbase + swz(n, u), ksrc, ok);
      cp_async16(vbase + swz(n, u), vsrc, ok);
      if (lane == 0) valid_s[s * CHUNK + n] = ok ? 1 : 0;
    }
  };

  // ---- prologue: the first STAGES - 1 chunks
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < nchunks) load_chunk(s, s);
    cp_async_commit();
  }

  // query fragments (A, 16 x 256) are read from shared memory for every
  // chunk rather than held in registers (64 fewer registers: three CTAs per
  // SM).  ldmatrix x4: matrices (rows 0-7, k 0-7), (rows 8-15, k 0-7),
  // (rows 0-7, k 8-15), (rows 8-15, k 8-15).
  const uint32_t qb = smem_addr(q_s);
  const int q_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int q_khalf = lane >> 4;

  const int g8 = lane >> 2, c4 = lane & 3;
  float m_run[2] = {-INFINITY, -INFINITY};  // rows g8, g8 + 8 (log2 units)
  float l_run[2] = {0.f, 0.f};              // this thread's share of the row sums
  float o[8][4];                            // rows g8 / g8 + 8, features 64 * warp + 8 * nt + 2 * c4 + {0, 1}
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

  for (int c = 0; c < nchunks; ++c) {
    const int s = c % STAGES;
    cp_async_wait<STAGES - 2>();
    __syncthreads();  // stage s landed for every thread; stage (c - 1) % STAGES is free
    {
      const int cn = c + STAGES - 1;
      if (cn < nchunks) load_chunk(cn, cn % STAGES);
      cp_async_commit();
    }
    const uint32_t kb = smem_addr(kv_s + (2 * s) * KV_STAGE_BYTES);
    const uint32_t vb = smem_addr(kv_s + (2 * s + 1) * KV_STAGE_BYTES);

    // ---- scores of tokens 8 * warp .. 8 * warp + 7 (one n-tile), all heads
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    {
      // ldmatrix x4 over K rows (tokens): matrices = features 16s..+7, +8..+15, +16..+23, +24..+31
      const int n = 8 * warp + (lane & 7);
      const int q4 = lane >> 3;
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2) {
        uint32_t b0, b1, b2, b3, a0, a1, a2, a3, a4, a5, a6, a7;
        ldsm_x4(kb + swz(n, 4 * s2 + q4), b0, b1, b2, b3);
        ldsm_x4(qb + swz(q_row, 4 * s2 + q_khalf), a0, a1, a2, a3);
        ldsm_x4(qb + swz(q_row, 4 * s2 + 2 + q_khalf), a4, a5, a6, a7);
        mma_bf16(sc, a0, a1, a2, a3, b0, b1);
        mma_bf16(sc, a4, a5, a6, a7, b2, b3);
      }
    }
    // sc[0], sc[1]: row g8, tokens 8w + 2c4 + {0,1}; sc[2], sc[3]: row g8 + 8
    const int n0 = 8 * warp + 2 * c4;
    const bool v0 = valid_s[s * CHUNK + n0] != 0, v1 = valid_s[s * CHUNK + n0 + 1] != 0;
    float x[4];
    x[0] = v0 ? sc[0] * p.scale_log2 : -INFINITY;
    x[1] = v1 ? sc[1] * p.scale_log2 : -INFINITY;
    x[2] = v0 ? sc[2] * p.scale_log2 : -INFINITY;
    x[3] = v1 ? sc[3] * p.scale_log2 : -INFINITY;
    float mx0 = fmaxf(x[0], x[1]), mx1 = fmaxf(x[2], x[3]);
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    float* red_c = red + (c & 1) * WARPS * 16;  // two buffers: no barrier needed before reuse
    if (c4 == 0) {
      red_c[warp * 16 + g8] = mx0;
      red_c[warp * 16 + g8 + 8] = mx1;
    }
    __syncthreads();
    float cm0 = red_c[g8], cm1 = red_c[g8 + 8];
#pragma unroll
    for (int w = 1; w < WARPS; ++w) {
      cm0 = fmaxf(cm0, red_c[w * 16 + g8]);
      cm1 = fmaxf(cm1, red_c[w * 16 + g8 + 8]);
    }
    const float mn0 = fmaxf(m_run[0], cm0), mn1 = fmaxf(m_run[1], cm1);
    // rows with nothing visible yet keep max -inf: their probabilities are 0
    const float a0 = mn0 == -INFINITY ? 1.f : exp2f(m_run[0] - mn0);
    const float a1 = mn1 == -INFINITY ? 1.f : exp2f(m_run[1] - mn1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    const float p0 = mn0 == -INFINITY ? 0.f : exp2f(x[0] - mn0);
    const float p1 = mn0 == -INFINITY ? 0.f : exp2f(x[1] - mn0);
    const float p2 = mn1 == -INFINITY ? 0.f : exp2f(x[2] - mn1);
    const float p3 = mn1 == -INFINITY ? 0.f : exp2f(x[3] - mn1);
    l_run[0] = l_run[0] * a0 + p0 + p1;
    l_run[1] = l_run[1] * a1 + p2 + p3;
    // probabilities as bf16 into the shared P tile [16 rows][32 tokens]
    *reinterpret_cast<uint32_t*>(p_s + g8 * P_STRIDE + n0) = pack_bf16(p0, p1);
    *reinterpret_cast<uint32_t*>(p_s + (g8 + 8) * P_STRIDE + n0) = pack_bf16(p2, p3);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      o[nt][0] *= a0;
      o[nt][1] *= a0;
      o[nt][2] *= a1;
      o[nt][3] *= a1;
    }
    __syncthreads();
    // ---- O[:, 64w .. 64w + 63] += P (16 x 32) . V (32 x 64)
    {
      const uint32_t pb = smem_addr(p_s);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        {
          const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = 16 * ks + (lane >> 4) * 8;
          ldsm_x4(pb + (uint32_t)(row * P_STRIDE + col) * 2, a[0], a[1], a[2], a[3]);
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          // V rows (tokens) 16ks .. 16ks + 15, features 64w + 16np .. + 15, transposed:
          // matrices (tok 0-7, f 0-7), (tok 8-15, f 0-7), (tok 0-7, f 8-15), (tok 8-15, f 8-15)
          const int n = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int u = 8 * warp + 2 * np + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + swz(n, u), b0, b1, b2, b3);
          mma_bf16(o[2 * np], a[0], a[1], a[2], a[3], b0, b1);
          mma_bf16(o[2 * np + 1], a[0], a[1], a[2], a[3], b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();

  // ---- the split's running max, sum and unnormalised output
  float l0 = l_run[0], l1 = l_run[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();
  if (c4 == 0) {
    red[warp * 16 + g8] = l0;
    red[warp * 16 + g8 + 8] = l1;
  }
  __syncthreads();
  const int64_t base = (t * p.Hkv + g) * p.splits + split;  // (row, KV head, split)
  float* po = p.part_o + base * p.group * D;
  float* pml = p.part_ml + base * p.group * 2;
  if (warp == 0 && c4 == 0) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      s0 += red[w * 16 + g8];
      s1 += red[w * 16 + g8 + 8];
    }
    if (g8 < p.group) {
      pml[g8 * 2] = m_run[0];
      pml[g8 * 2 + 1] = s0;
    }
    if (g8 + 8 < p.group) {
      pml[(g8 + 8) * 2] = m_run[1];
      pml[(g8 + 8) * 2 + 1] = s1;
    }
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int f = 64 * warp + 8 * nt + 2 * c4;
    if (g8 < p.group) *reinterpret_cast<float2*>(po + g8 * D + f) = make_float2(o[nt][0], o[nt][1]);
    if (g8 + 8 < p.group) *reinterpret_cast<float2*>(po + (g8 + 8) * D + f) = make_float2(o[nt][2], o[nt][3]);
  }
}

// One warp per (row, query head): merge the splits.
__global__ void __launch_bounds__(256) combine_kernel(const Params p) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= p.T * p.Hq) return;
  const int64_t t = wid / p.Hq;
  const int h = (int)(wid % p.Hq);
  const int g = h / p.group, hh = h % p.group;
  const int64_t base = (t * p.Hkv + g) * p.splits;
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, p.part_ml[((base + s) * p.group + hh) * 2]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float Lsum = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float ms = p.part_ml[((base + s) * p.group + hh) * 2];
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      Lsum += w * p.part_ml[((base + s) * p.group + hh) * 2 + 1];
      const float* po = p.part_o + ((base + s) * p.group + hh) * D + lane * 8;
      const float4 x = *reinterpret_cast<const float4*>(po);
      const float4 y = *reinterpret_cast<const float4*>(po + 4);
      acc[0] += w * x.x; acc[1] += w * x.y; acc[2] += w * x.z; acc[3] += w * x.w;
      acc[4] += w * y.x; acc[5] += w * y.y; acc[6] += w * y.z; acc[7] += w * y.w;
    }
  }
  float mul = Lsum > 0.f ? 1.f / Lsum : 0.f;
  if (p.gate) mul *= 1.f / (1.f + expf(-p.gate[t * p.Hq + h]));
  uint4 packed;
  packed.x = pack_bf16(acc[0] * mul, acc[1] * mul);
  packed.y = pack_bf16(acc[2] * mul, acc[3] * mul);
  packed.z = pack_bf16(acc[4] * mul, acc[5] * mul);
  packed.w = pack_bf16(acc[6] * mul, acc[7] * mul);
  *reinterpret_cast<uint4*>(p.out + t * p.out_st + (int64_t)h * D + lane * 8) = packed;
  if (p.lse && lane == 0) p.lse[t * p.Hq + h] = Lsum > 0.f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace attn
}  // namespace qsa
