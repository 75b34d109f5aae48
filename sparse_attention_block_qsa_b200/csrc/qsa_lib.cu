// C ABI of the QSA MQA indexer score (declared in include/qsa.h): host-side
// validation, TMA tensor-map encoding and kernel launches.  One translation
// unit, so the kernels and the device error word share one module.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "qsa.h"
#include "decode.cuh"
#include "prefill.cuh"
#include "topk.cuh"
#include "attention.cuh"
#include "paged_batch.cuh"

namespace {

thread_local char g_detail[512] = "";

qsa_status_t fail(qsa_status_t s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return s;
}

qsa_status_t ok() {
  g_detail[0] = '\0';
  return QSA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// [begin, end) byte range touched by a strided 3-D view (non-negative strides).
struct Range {
  uintptr_t lo, hi;
};

Range span(const void* base, int64_t elem, int64_t n0, int64_t s0, int64_t n1, int64_t s1, int64_t n2, int64_t s2,
           int64_t inner) {
  uintptr_t b = reinterpret_cast<uintptr_t>(base);
  int64_t last = (n0 > 0 ? (n0 - 1) * s0 : 0) + (n1 > 0 ? (n1 - 1) * s1 : 0) + (n2 > 0 ? (n2 - 1) * s2 : 0);
  return Range{b, b + static_cast<uintptr_t>((last + inner) * elem)};
}

bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// ---------------------------------------------------------------- driver entry
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

qsa_status_t encode_bf16_map(CUtensorMap* map, int rank, void* base, const cuuint64_t* dims,
                             const cuuint64_t* strides_bytes, const cuuint32_t* box, const char* what,
                             bool f16 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(QSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides_bytes, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QSA_ERR_ALIGNMENT, "tensor map for %s rejected by the driver (CUresult %d)", what, (int)r);
  return QSA_OK;
}

// Store map of a W x rows fp32 matrix with the given row stride (elements),
// box 32 x 16.  Returns false when TMA cannot address it (the caller then
// stores element by element): the base and the row pitch must be multiples
// of 16 bytes.
bool encode_f32_store_map(CUtensorMap* map, float* base, int64_t W, int64_t rows, int64_t stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || !aligned(base, 16) || W <= 0 || rows <= 0 || W > UINT32_MAX || rows > UINT32_MAX) return false;
  const int64_t pitch = rows > 1 ? stride * 4 : ((W * 4 + 15) / 16) * 16;
  if (pitch % 16 != 0 || pitch < W * 4 || pitch >= (int64_t(1) << 40)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)W, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)pitch};
  cuuint32_t box[2] = {32, (cuuint32_t)qsa::prefill::EPI_TOKENS};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  int sms = 0;
  bool attrs_set = false;
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

qsa_status_t device_info(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(QSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.attrs_set) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(QSA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200); device %d is sm_%d%d", dev, major,
                  minor);
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    struct {
      const void* fn;
      size_t bytes;
    } kernels[] = {
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::BF16, false, false>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::BF16, true, false>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::BF16, false, true>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::BF16, true, true>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::F16, false, false>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::F16, true, false>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::F16, false, true>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::F16, true, true>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::E4M3, false, true>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::decode::decode_kernel<qsa::decode::Fmt::E4M3, true, true>), qsa::decode::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::prefill::prefill_kernel<false>), qsa::prefill::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::prefill::prefill_kernel<true>), qsa::prefill::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::attn::attn_kernel), qsa::attn::SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::topk::topk_rows_kernel), qsa::topk::ROWS_SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::topk::topk_pipe_kernel), qsa::topk::PIPE_SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::topk::topk_filter_kernel), qsa::topk::TP_SMEM_BYTES},
        {reinterpret_cast<const void*>(qsa::topk::topk_list_kernel),
         qsa::topk::TP_LIST_WARPS * qsa::topk::tp_list_warp_bytes(qsa::topk::MAX_W)},
    };
    for (auto& k : kernels) {
      e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)k.bytes);
      if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    d.attrs_set = true;
  }
  *sms = d.sms;
  return QSA_OK;
}

qsa_status_t launch_status(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
  return ok();
}

// Launch with programmatic stream serialization (the kernel may begin
// launching while the previous kernel on the stream finishes; every kernel of
// this library waits with griddepcontrol.wait before its first global read).
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------- intervals
__global__ void prefill_intervals_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ seq_lens,
                                         const int32_t* __restrict__ key_offsets, int32_t S, int64_t T,
                                         int32_t* __restrict__ ks, int32_t* __restrict__ ke) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int lo = 0, hi = S - 1;  // last sequence whose first row is <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)__ldg(cu + mid) <= t) lo = mid;
    else hi = mid - 1;
  }
  const int32_t first = __ldg(cu + lo);
  const int32_t qlen = __ldg(cu + lo + 1) - first;
  const int32_t L = __ldg(seq_lens + lo);
  const int32_t pos = L - qlen + (int32_t)(t - first);  // logical position of the row
  const int32_t vis = max(0, min((pos + 1) >> 2, L >> 2));
  const int32_t off = __ldg(key_offsets + lo);
  ks[t] = off;
  ke[t] = off + vis;
}

// ---------------------------------------------------------------- prefill core
struct PrefillArgs {
  const void* q;
  int64_t q_stride_t, q_stride_h;
  const void* k;
  int64_t k_stride, Nk;
  const int32_t* ks;
  const int32_t* ke;
  int64_t T;
  float scale;
  float* out;
  int64_t out_stride;
  int32_t W;
  bool f16 = false;  // q and k hold fp16 instead of bf16
};

qsa_status_t validate_prefill(const PrefillArgs& a) {
  if (a.T < 0 || a.Nk < 0 || a.W < 0) return fail(QSA_ERR_INVALID_ARG, "T, Nk and W must be non-negative");
  if (a.T > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "T = %lld rows exceeds 2^31 - 1", (long long)a.T);
  if (a.Nk > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "Nk = %lld keys exceeds 2^31 - 1", (long long)a.Nk);
  if (!std::isfinite(a.scale)) return fail(QSA_ERR_INVALID_ARG, "scale must be finite");
  if (a.T == 0 || a.W == 0) return QSA_OK;
  if (!a.q || !a.ks || !a.ke || !a.out || (a.Nk > 0 && !a.k))
    return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(a.q, 16) || (a.Nk > 0 && !aligned(a.k, 16)))
    return fail(QSA_ERR_ALIGNMENT, "q and k must start on a 16-byte boundary");
  if (!aligned(a.out, 4) || !aligned(a.ks, 4) || !aligned(a.ke, 4))
    return fail(QSA_ERR_ALIGNMENT, "out, ks and ke must be 4-byte aligned");
  if (a.q_stride_h <= 0 || a.q_stride_h % 8 != 0)
    return fail(QSA_ERR_ALIGNMENT, "q_stride_h = %lld must be a positive multiple of 8", (long long)a.q_stride_h);
  if (a.T > 1 && (a.q_stride_t <= 0 || a.q_stride_t % 8 != 0))
    return fail(QSA_ERR_ALIGNMENT, "q_stride_t = %lld must be a positive multiple of 8", (long long)a.q_stride_t);
  if (a.Nk > 1 && (a.k_stride < 128 || a.k_stride % 8 != 0))
    return fail(QSA_ERR_ALIGNMENT, "k_stride = %lld must be a multiple of 8 and >= 128", (long long)a.k_stride);
  if (a.T > 1 && a.out_stride < a.W)
    return fail(QSA_ERR_INVALID_ARG, "out_stride = %lld is below W = %d", (long long)a.out_stride, a.W);
  const Range ro = span(a.out, 4, a.T, a.out_stride, 1, 0, 1, 0, a.W);
  const Range rq = span(a.q, 2, a.T, a.q_stride_t, 4, a.q_stride_h, 1, 0, 128);
  const Range rks = span(a.ks, 4, a.T, 1, 1, 0, 1, 0, 1), rke = span(a.ke, 4, a.T, 1, 1, 0, 1, 0, 1);
  if (overlaps(ro, rq) || overlaps(ro, rks) || overlaps(ro, rke) ||
      (a.Nk > 0 && overlaps(ro, span(a.k, 2, a.Nk, a.k_stride, 1, 0, 1, 0, 128))))
    return fail(QSA_ERR_INVALID_ARG, "out overlaps an input");
  return QSA_OK;
}

qsa_status_t launch_prefill(const PrefillArgs& a, cudaStream_t stream, bool pdl = false) {
  int sms = 0;
  qsa_status_t st = device_info(&sms);
  if (st != QSA_OK) return st;
  CUtensorMap tm_q, tm_k;
  memset(&tm_k, 0, sizeof tm_k);
  {
    const int64_t st_t = a.T > 1 ? a.q_stride_t : 4 * a.q_stride_h;
    cuuint64_t dims[3] = {128, 4, (cuuint64_t)a.T};
    cuuint64_t strides[2] = {(cuuint64_t)a.q_stride_h * 2, (cuuint64_t)st_t * 2};
    cuuint32_t box[3] = {64, 4, (cuuint32_t)qsa::prefill::BT};
    st = encode_bf16_map(&tm_q, 3, const_cast<void*>(a.q), dims, strides, box, "q", a.f16);
    if (st != QSA_OK) return st;
  }
  if (a.Nk > 0) {
    cuuint64_t dims[2] = {128, (cuuint64_t)a.Nk};
    cuuint64_t strides[1] = {(cuuint64_t)(a.Nk > 1 ? a.k_stride : 128) * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)qsa::prefill::BM};
    st = encode_bf16_map(&tm_k, 2, const_cast<void*>(a.k), dims, strides, box, "k", a.f16);
    if (st != QSA_OK) return st;
  }
  for (int64_t r0 = 0; r0 < a.T; r0 += qsa::prefill::MAX_ROWS_PER_LAUNCH) {
    qsa::prefill::Params p;
    p.ks = a.ks + r0;
    p.ke = a.ke + r0;
    p.q_row0 = (int32_t)r0;
    p.T = std::min<int64_t>(a.T - r0, qsa::prefill::MAX_ROWS_PER_LAUNCH);
    p.Nk = a.Nk;
    p.scale = a.scale;
    p.out = a.out + r0 * a.out_stride;
    p.out_stride = a.out_stride;
    p.W = a.W;
    CUtensorMap tm_out;
    memset(&tm_out, 0, sizeof tm_out);
    p.store_map = encode_f32_store_map(&tm_out, p.out, a.W, p.T, a.out_stride) ? 1 : 0;
    if (pdl)
      launch_pdl(a.f16 ? qsa::prefill::prefill_kernel<true> : qsa::prefill::prefill_kernel<false>, dim3(sms),
                 dim3(qsa::prefill::NUM_THREADS), qsa::prefill::SMEM_BYTES, stream, tm_q, tm_k, tm_out, p);
    else if (a.f16)
      qsa::prefill::prefill_kernel<true><<<sms, qsa::prefill::NUM_THREADS, qsa::prefill::SMEM_BYTES, stream>>>(
          tm_q, tm_k, tm_out, p);
    else
      qsa::prefill::prefill_kernel<false><<<sms, qsa::prefill::NUM_THREADS, qsa::prefill::SMEM_BYTES, stream>>>(
          tm_q, tm_k, tm_out, p);
    st = launch_status("prefill kernel");
    if (st != QSA_OK) return st;
  }
  return ok();
}

// ---------------------------------------------------------------- top-k core
struct TopkArgs {
  const float* scores;
  int64_t score_stride;
  const int32_t* lengths;
  int64_t rows;
  int32_t W, k;
  int32_t* idx;
  int64_t idx_stride;
};

qsa_status_t validate_topk(const TopkArgs& a) {
  if (a.rows < 0) return fail(QSA_ERR_INVALID_ARG, "rows must be non-negative");
  if (a.rows > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "rows = %lld exceeds 2^31 - 1", (long long)a.rows);
  if (a.k < 1 || a.k > 2048) return fail(QSA_ERR_UNSUPPORTED, "k = %d must be in [1, 2048]", a.k);
  if (a.W < 1 || a.W > 65536) return fail(QSA_ERR_UNSUPPORTED, "W = %d must be in [1, 65536]", a.W);
  if (a.rows == 0) return QSA_OK;
  if (!a.scores || !a.idx) return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(a.scores, 4) || !aligned(a.idx, 4) || (a.lengths && !aligned(a.lengths, 4)))
    return fail(QSA_ERR_ALIGNMENT, "scores, lengths and idx must be 4-byte aligned");
  if (a.rows > 1 && a.score_stride < a.W)
    return fail(QSA_ERR_INVALID_ARG, "score_stride = %lld is below W = %d", (long long)a.score_stride, a.W);
  if (a.rows > 1 && a.idx_stride < a.k)
    return fail(QSA_ERR_INVALID_ARG, "idx_stride = %lld is below k = %d", (long long)a.idx_stride, a.k);
  const Range ri = span(a.idx, 4, a.rows, a.idx_stride, 1, 0, 1, 0, a.k);
  if (overlaps(ri, span(a.scores, 4, a.rows, a.score_stride, 1, 0, 1, 0, a.W)) ||
      (a.lengths && overlaps(ri, span(a.lengths, 4, a.rows, 1, 1, 0, 1, 0, 1))))
    return fail(QSA_ERR_INVALID_ARG, "idx overlaps an input");
  return QSA_OK;
}

// Bytes at the end of a fused prefill + top-k workspace that carry the top-k
// kernel's per-CTA threshold predictions from one chunk to the next.
constexpr size_t kPredBytes = 4096;
constexpr int64_t kPredFloats = kPredBytes / sizeof(float);

qsa_status_t launch_topk(const TopkArgs& a, cudaStream_t stream, float* pred_state = nullptr,
                         uint8_t* ws = nullptr) {
  int sms = 0;
  qsa_status_t st = device_info(&sms);
  if (st != QSA_OK) return st;
  qsa::topk::Params p;
  p.scores = a.scores;
  p.stride = a.rows > 1 ? a.score_stride : a.W;
  p.lengths = a.lengths;
  p.W = a.W;
  p.k = a.k;
  p.idx = a.idx;
  p.idx_stride = a.idx_stride;
  p.vec4 = aligned(a.scores, 16) && (p.stride % 4 == 0);
  p.rows = a.rows;
  p.pred_state = pred_state;
  p.row_list = nullptr;
  p.row_count = nullptr;
  p.ws = ws;
  // the predictions carried between chunks hold one float per CTA
  const int64_t max_grid = pred_state ? kPredFloats : INT32_MAX;
  if (ws != nullptr && p.vec4 && a.W % 4 == 0) {
    // with a workspace: filter pass, list selection, exact pass over the rows that missed
    using namespace qsa::topk;
    const TpLayout L = tp_layout(a.rows);
    const int64_t grid_f = std::min<int64_t>(std::min<int64_t>(a.rows, (int64_t)sms * TP_CTAS_PER_SM), TP_PRED_FLOATS);
    Params f = p;
    f.pred_state = reinterpret_cast<float*>(ws + L.pred);  // carried between calls through the workspace
    topk_filter_kernel<<<(unsigned)grid_f, TP_THREADS, TP_SMEM_BYTES, stream>>>(f);
    st = launch_status("top-k filter kernel");
    if (st != QSA_OK) return st;
    const int64_t grid_l = std::min<int64_t>((a.rows + TP_LIST_WARPS - 1) / TP_LIST_WARPS,
                                             (int64_t)sms * TP_LIST_CTAS_PER_SM);
    topk_list_kernel<<<(unsigned)grid_l, TP_LIST_WARPS * 32, TP_LIST_WARPS * tp_list_warp_bytes(a.W), stream>>>(p);
    st = launch_status("top-k list kernel");
    if (st != QSA_OK) return st;
    Params q = p;
    q.pred_state = nullptr;
    q.row_list = reinterpret_cast<const int32_t*>(ws + L.list);
    q.row_count = reinterpret_cast<const uint32_t*>(ws + L.count);
    topk_rows_kernel<<<(unsigned)std::min<int64_t>(a.rows, (int64_t)sms * ROWS_CTAS_PER_SM), THREADS, ROWS_SMEM_BYTES,
                       stream>>>(q);
  } else if (p.vec4 && a.W % 4 == 0) {
    // rows start on 16-byte boundaries: stream them with bulk copies
    const int64_t grid = std::min<int64_t>(std::min<int64_t>(a.rows, (int64_t)sms * qsa::topk::PIPE_CTAS_PER_SM), max_grid);
    qsa::topk::topk_pipe_kernel<<<(unsigned)grid, qsa::topk::PIPE_THREADS, qsa::topk::PIPE_SMEM_BYTES, stream>>>(p);
  } else {
    const int64_t grid = std::min<int64_t>(std::min<int64_t>(a.rows, (int64_t)sms * qsa::topk::ROWS_CTAS_PER_SM), max_grid);
    qsa::topk::topk_rows_kernel<<<(unsigned)grid, qsa::topk::THREADS, qsa::topk::ROWS_SMEM_BYTES, stream>>>(p);
  }
  return launch_status("top-k kernel");
}

// One thread waits on an mbarrier that nothing arrives on (unless `arrive`),
// with the kernels' bounded wait and the given limit.
__global__ void selftest_wait_kernel(uint64_t timeout_ns, int32_t arrive) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    qsa::mbar_init(&bar, 1);
    qsa::fence_mbar_init();
    if (arrive) qsa::mbar_arrive(&bar);
    if (!qsa::mbar_wait_for(&bar, 0, nullptr, timeout_ns)) qsa::record_device_error(QSA_DEVERR_WAIT_TIMEOUT);
  }
}

// Scratch of qsa_mqa_prefill_topk_noalloc: a fixed array that every GPU
// loading this library holds until the process exits.  Host code must not
// hand the symbol itself to a kernel (on the host it only stands in for the
// device array); its device address is fetched once per device below.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Split-KV plan of the sparse attention: a row's token list is cut into
// `splits` runs of `cps` 32-entry chunks, so that rows x KV heads x splits
// gives the grid at most about 9 CTAs per SM of a 148-SM part (three waves
// of three resident CTAs; rounded down so that the last wave is full; device
// independent, so the workspace size depends on the shapes only).
void attn_splits(int64_t T, int32_t Hkv, int32_t width, int32_t* splits, int32_t* cps) {
  const int64_t chunks = std::max<int64_t>(1, ((int64_t)width + qsa::attn::CHUNK - 1) / qsa::attn::CHUNK);
  const int64_t pairs = std::max<int64_t>(1, T * Hkv);
  int64_t sp = std::min<int64_t>(chunks, std::max<int64_t>(1, 1332 / pairs));
  const int64_t per = (chunks + sp - 1) / sp;
  sp = (chunks + per - 1) / per;
  *splits = (int32_t)sp;
  *cps = (int32_t)per;
}

}  // namespace

// ================================================================ C ABI
extern "C" {

const char* qsa_status_string(qsa_status_t s) {
  switch (s) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG: a size, count, pointer or value is out of range";
    case QSA_ERR_ALIGNMENT: return "QSA_ERR_ALIGNMENT: a base address or stride breaks the layout rules";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED: configuration not implemented";
    case QSA_ERR_WORKSPACE: return "QSA_ERR_WORKSPACE: workspace too small";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA: CUDA call or launch failed";
  }
  return "unknown qsa_status_t";
}

const char* qsa_last_error_detail(void) { return g_detail; }

qsa_status_t qsa_device_error(uint32_t* bits) {
  if (!bits) return fail(QSA_ERR_INVALID_ARG, "bits must not be null");
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, qsa::g_device_error, sizeof v);
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(qsa::g_device_error, &zero, sizeof zero);
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
  *bits = v;
  return ok();
}

qsa_status_t qsa_selftest_bounded_wait(uint64_t timeout_ns, int32_t arrive, void* stream) {
  if (timeout_ns > 10000000000ull) return fail(QSA_ERR_INVALID_ARG, "timeout_ns above 10 s");
  int sms = 0;
  qsa_status_t st = device_info(&sms);
  if (st != QSA_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns, arrive);
  return launch_status("self-test kernel");
}

// Every format: E4M3 keys take 1 byte per element (strides multiples of 16)
// and are scaled by k_scale; bf16 and fp16 keys take 2 (k_scale == 1).
extern "C++" {
template <qsa::decode::Fmt F, bool GEN, bool PIPE>
static void launch_decode(int sms, const qsa::decode::Params& p, cudaStream_t stream, bool pdl) {
  if (pdl)
    launch_pdl(qsa::decode::decode_kernel<F, GEN, PIPE>, dim3(sms), dim3(qsa::decode::NUM_THREADS),
               qsa::decode::SMEM_BYTES, stream, p);
  else
    qsa::decode::decode_kernel<F, GEN, PIPE><<<sms, qsa::decode::NUM_THREADS, qsa::decode::SMEM_BYTES, stream>>>(p);
}

// The two-half-batch loop: always for the fp8 cache (its widening is the
// longest step between batches); for bf16 / fp16 keys when no warp gets more
// than one half-batch (measured on B200: fp8 16 x 4 long contexts 15.4 ->
// 12.8 us, 16 x 1 8.2 -> 6.3 us; bf16 1 x 1 4.0 -> 3.5 us, but bf16 16 x 4
// 13.2 -> 14.3 us).
template <qsa::decode::Fmt F>
static void launch_decode_fmt(int sms, const qsa::decode::Params& p, cudaStream_t stream, bool pdl, bool pow2,
                              bool pipe) {
  if constexpr (F == qsa::decode::Fmt::E4M3) {
    pow2 ? launch_decode<F, false, true>(sms, p, stream, pdl) : launch_decode<F, true, true>(sms, p, stream, pdl);
  } else {
    if (pipe)
      pow2 ? launch_decode<F, false, true>(sms, p, stream, pdl) : launch_decode<F, true, true>(sms, p, stream, pdl);
    else
      pow2 ? launch_decode<F, false, false>(sms, p, stream, pdl) : launch_decode<F, true, false>(sms, p, stream, pdl);
  }
}
}

static qsa_status_t decode_common(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                                  const void* k_cache, qsa::decode::Fmt fmt, float k_scale, int64_t num_pages,
                                  int32_t page_size,
                                  int64_t k_page_stride, int64_t k_row_stride, const int32_t* page_table,
                                  int64_t pt_stride, int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t Q,
                                  float scale, float* out, int64_t out_stride_b, int64_t out_stride_t, int32_t W,
                                  void* stream, bool pdl = false) {
  if (B < 0 || W < 0) return fail(QSA_ERR_INVALID_ARG, "B and W must be non-negative");
  if (Q < 1 || Q > 4) return fail(QSA_ERR_UNSUPPORTED, "Q = %d query tokens per request; 1..4 supported", Q);
  if (page_size < 8 || page_size > 1024)
    return fail(QSA_ERR_UNSUPPORTED, "page_size = %d; supported page sizes are 8 .. 1024", page_size);
  const bool fp8 = fmt == qsa::decode::Fmt::E4M3;
  if (!std::isfinite(scale)) return fail(QSA_ERR_INVALID_ARG, "scale must be finite");
  if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(scale * k_scale)))
    return fail(QSA_ERR_INVALID_ARG, "k_scale must be finite and positive, and scale * k_scale finite");
  if (max_pages < 0) return fail(QSA_ERR_INVALID_ARG, "max_pages must be non-negative");
  if (num_pages < 1 || num_pages > INT32_MAX)
    return fail(QSA_ERR_INVALID_ARG, "num_pages = %lld must be in [1, 2^31 - 1]", (long long)num_pages);
  if (B == 0 || W == 0) return ok();
  if (!q || !k_cache || !seq_lens || !out || (max_pages > 0 && !page_table))
    return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k_cache, 16))
    return fail(QSA_ERR_ALIGNMENT, "q and k_cache must be 16-byte aligned");
  if (!aligned(out, 4) || !aligned(seq_lens, 4) || (page_table && !aligned(page_table, 4)))
    return fail(QSA_ERR_ALIGNMENT, "out, seq_lens and page_table must be 4-byte aligned");
  const int64_t qs[3] = {B > 1 ? q_stride_b : 0, Q > 1 ? q_stride_t : 0, q_stride_h};
  for (int i = 0; i < 3; ++i)
    if (qs[i] < 0 || qs[i] % 8 != 0)
      return fail(QSA_ERR_ALIGNMENT, "q strides must be non-negative multiples of 8 (got %lld)", (long long)qs[i]);
  const int kb = fp8 ? 1 : 2;  // bytes per key element
  const int64_t kmul = 16 / kb;
  if (k_row_stride < 128 || k_row_stride % kmul != 0)
    return fail(QSA_ERR_ALIGNMENT, "k_row_stride = %lld must be a multiple of %lld and >= 128",
                (long long)k_row_stride, (long long)kmul);
  if (num_pages > 1 && (k_page_stride <= 0 || k_page_stride % kmul != 0))
    return fail(QSA_ERR_ALIGNMENT, "k_page_stride = %lld must be a positive multiple of %lld",
                (long long)k_page_stride, (long long)kmul);
  if (max_pages > 0 && B > 1 && pt_stride < max_pages)
    return fail(QSA_ERR_INVALID_ARG, "pt_stride = %lld is below max_pages = %d", (long long)pt_stride, max_pages);
  if (Q > 1 && out_stride_t < W) return fail(QSA_ERR_INVALID_ARG, "out_stride_t is below W");
  if (B > 1 && out_stride_b < (int64_t)(Q - 1) * (Q > 1 ? out_stride_t : 0) + W)
    return fail(QSA_ERR_INVALID_ARG, "out_stride_b is too small: rows of different requests overlap");
  {
    const Range ro = span(out, 4, B, B > 1 ? out_stride_b : 0, Q, Q > 1 ? out_stride_t : 0, 1, 0, W);
    const Range rq = span(q, 2, B, qs[0], Q, qs[1], 4, qs[2], 128);
    const Range rk = span(k_cache, kb, num_pages, num_pages > 1 ? k_page_stride : 0, page_size, k_row_stride, 1, 0, 128);
    const Range rs = span(seq_lens, 4, B, 1, 1, 0, 1, 0, 1);
    bool bad = overlaps(ro, rq) || overlaps(ro, rk) || overlaps(ro, rs);
    if (max_pages > 0) bad = bad || overlaps(ro, span(page_table, 4, B, B > 1 ? pt_stride : 0, 1, 0, 1, 0, max_pages));
    if (bad) return fail(QSA_ERR_INVALID_ARG, "out overlaps an input");
  }

  int sms = 0;
  qsa_status_t st = device_info(&sms);
  if (st != QSA_OK) return st;

  qsa::decode::Params p;
  p.q_sb = B > 1 ? q_stride_b : 0;
  p.q_st = Q > 1 ? q_stride_t : 0;
  p.q_sh = q_stride_h;
  p.k_cache = fp8 ? nullptr : static_cast<const uint16_t*>(k_cache);
  p.k8 = fp8 ? static_cast<const uint8_t*>(k_cache) : nullptr;
  p.k_page_stride = num_pages > 1 ? k_page_stride : 0;
  p.k_row_stride = k_row_stride;
  p.num_pages = num_pages;
  p.pt_stride = pt_stride;
  p.max_pages = max_pages;
  p.Q = Q;
  const bool pow2 = (page_size & (page_size - 1)) == 0;
  int log2_ps = 0;
  while ((1 << (log2_ps + 1)) <= page_size) ++log2_ps;
  p.log2_ps = log2_ps;
  // Key n lies in logical page n / ps = (n * m) >> s for 0 <= n < 2^30, with
  // s = 31 + floor(log2 ps) and m = ceil(2^s / ps) < 2^32 (ps >= 8).  Write
  // m * ps = 2^s + e with 0 <= e < ps: then n * m / 2^s = n / ps +
  // n * e / (ps * 2^s), and n * e < 2^30 * 2^(floor(log2 ps) + 1) = 2^s, so the
  // extra term stays below 1 / ps and never lifts the floor past n / ps.
  // (A request holds fewer than 2^29 keys: seq_len is an int32 of tokens.)
  p.ps = (uint32_t)page_size;
  p.ps_shift = 31 + log2_ps;
  p.ps_magic = (uint32_t)(((1ull << p.ps_shift) + (uint64_t)page_size - 1) / (uint64_t)page_size);
  p.scale = fp8 ? scale * k_scale : scale;
  p.out_sb = out_stride_b;
  p.out_st = out_stride_t;
  p.W = W;
  // Requests are independent: launch them in groups that fit the kernel's
  // prefix table and whose 8-key tile count, at most ceil(W / 8) per request,
  // fits the kernel's 32-bit tile indices.
  const int64_t tiles_per_req = ((int64_t)W + qsa::decode::TILE - 1) / qsa::decode::TILE;
  const int32_t group = (int32_t)std::min<int64_t>(qsa::decode::MAX_B, (int64_t)UINT32_MAX / tiles_per_req);
  for (int32_t b0 = 0; b0 < B; b0 += group) {
    p.B = std::min(B - b0, group);
    p.q = static_cast<const uint16_t*>(q) + (int64_t)b0 * p.q_sb;
    p.page_table = max_pages > 0 ? page_table + (int64_t)b0 * pt_stride : page_table;
    p.seq_lens = seq_lens + b0;
    p.out = out + (int64_t)b0 * out_stride_b;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    using qsa::decode::Fmt;
    const bool pipe = (int64_t)p.B * tiles_per_req <=
                      (int64_t)sms * qsa::decode::WARPS * (qsa::decode::BATCH / 2);  // at most one half-batch a warp
    if (fmt == Fmt::E4M3)
      launch_decode_fmt<Fmt::E4M3>(sms, p, s, pdl, pow2, pipe);
    else if (fmt == Fmt::F16)
      launch_decode_fmt<Fmt::F16>(sms, p, s, pdl, pow2, pipe);
    else
      launch_decode_fmt<Fmt::BF16>(sms, p, s, pdl, pow2, pipe);
    st = launch_status("decode kernel");
    if (st != QSA_OK) return st;
  }
  return ok();
}

qsa_status_t qsa_mqa_decode(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                            const void* k_cache, int64_t num_pages, int32_t page_size, int64_t k_page_stride,
                            int64_t k_row_stride, const int32_t* page_table, int64_t pt_stride, int32_t max_pages,
                            const int32_t* seq_lens, int32_t B, int32_t Q, float scale, float* out,
                            int64_t out_stride_b, int64_t out_stride_t, int32_t W, void* stream) {
  return decode_common(q, q_stride_b, q_stride_t, q_stride_h, k_cache, qsa::decode::Fmt::BF16, 1.f, num_pages,
                       page_size, k_page_stride, k_row_stride, page_table, pt_stride, max_pages, seq_lens, B, Q, scale,
                       out, out_stride_b, out_stride_t, W, stream);
}

qsa_status_t qsa_mqa_decode_f16(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                                const void* k_cache, int64_t num_pages, int32_t page_size, int64_t k_page_stride,
                                int64_t k_row_stride, const int32_t* page_table, int64_t pt_stride, int32_t max_pages,
                                const int32_t* seq_lens, int32_t B, int32_t Q, float scale, float* out,
                                int64_t out_stride_b, int64_t out_stride_t, int32_t W, void* stream) {
  return decode_common(q, q_stride_b, q_stride_t, q_stride_h, k_cache, qsa::decode::Fmt::F16, 1.f, num_pages,
                       page_size, k_page_stride, k_row_stride, page_table, pt_stride, max_pages, seq_lens, B, Q, scale,
                       out, out_stride_b, out_stride_t, W, stream);
}

qsa_status_t qsa_mqa_decode_fp8(const void* q, int64_t q_stride_b, int64_t q_stride_t, int64_t q_stride_h,
                                const void* k_cache, float k_scale, int64_t num_pages, int32_t page_size,
                                int64_t k_page_stride, int64_t k_row_stride, const int32_t* page_table,
                                int64_t pt_stride, int32_t max_pages, const int32_t* seq_lens, int32_t B, int32_t Q,
                                float scale, float* out, int64_t out_stride_b, int64_t out_stride_t, int32_t W,
                                void* stream) {
  return decode_common(q, q_stride_b, q_stride_t, q_stride_h, k_cache, qsa::decode::Fmt::E4M3, k_scale, num_pages,
                       page_size, k_page_stride, k_row_stride, page_table, pt_stride, max_pages, seq_lens, B, Q, scale,
                       out, out_stride_b, out_stride_t, W, stream);
}

qsa_status_t qsa_mqa_prefill(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k, int64_t k_stride,
                             int64_t Nk, const int32_t* ks, const int32_t* ke, int64_t T, float scale, float* out,
                             int64_t out_stride, int32_t W, void* stream) {
  PrefillArgs a{q, q_stride_t, q_stride_h, k, k_stride, Nk, ks, ke, T, scale, out, out_stride, W};
  qsa_status_t st = validate_prefill(a);
  if (st != QSA_OK) return st;
  if (T == 0 || W == 0) return ok();
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

qsa_status_t qsa_mqa_prefill_f16(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                                 int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke, int64_t T,
                                 float scale, float* out, int64_t out_stride, int32_t W, void* stream) {
  PrefillArgs a{q, q_stride_t, q_stride_h, k, k_stride, Nk, ks, ke, T, scale, out, out_stride, W, true};
  qsa_status_t st = validate_prefill(a);
  if (st != QSA_OK) return st;
  if (T == 0 || W == 0) return ok();
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

qsa_status_t qsa_prefill_intervals(const int32_t* cu_seqlens_q, const int32_t* seq_lens, const int32_t* key_offsets,
                                   int32_t S, int64_t T, int32_t* ks, int32_t* ke, void* stream) {
  if (S < 0 || T < 0) return fail(QSA_ERR_INVALID_ARG, "S and T must be non-negative");
  if (T == 0) return ok();
  if (S == 0) return fail(QSA_ERR_INVALID_ARG, "T > 0 rows need at least one sequence");
  if (!cu_seqlens_q || !seq_lens || !key_offsets || !ks || !ke)
    return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  const int threads = 256;
  const int64_t blocks = (T + threads - 1) / threads;
  if (blocks > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "T too large");
  prefill_intervals_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      cu_seqlens_q, seq_lens, key_offsets, S, T, ks, ke);
  return launch_status("prefill interval kernel");
}

qsa_status_t qsa_topk(const float* scores, int64_t score_stride, const int32_t* lengths, int64_t rows, int32_t W,
                      int32_t k, int32_t* idx, int64_t idx_stride, void* stream) {
  TopkArgs a{scores, score_stride, lengths, rows, W, k, idx, idx_stride};
  qsa_status_t st = validate_topk(a);
  if (st != QSA_OK) return st;
  if (rows == 0) return ok();
  return launch_topk(a, static_cast<cudaStream_t>(stream));
}

size_t qsa_topk_workspace_size(int64_t rows, int32_t W, int32_t k) {
  (void)W;
  (void)k;
  return rows > 0 ? qsa::topk::tp_layout(rows).total : 0;
}

qsa_status_t qsa_topk_ws(const float* scores, int64_t score_stride, const int32_t* lengths, int64_t rows, int32_t W,
                         int32_t k, int32_t* idx, int64_t idx_stride, void* workspace, size_t workspace_bytes,
                         void* stream) {
  TopkArgs a{scores, score_stride, lengths, rows, W, k, idx, idx_stride};
  qsa_status_t st = validate_topk(a);
  if (st != QSA_OK) return st;
  if (rows == 0) return ok();
  const size_t need = qsa_topk_workspace_size(rows, W, k);
  if (!workspace) return fail(QSA_ERR_INVALID_ARG, "null workspace");
  if (!aligned(workspace, 256)) return fail(QSA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  if (workspace_bytes < need)
    return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes; %zu needed for %lld rows", workspace_bytes, need,
                (long long)rows);
  const Range rw{reinterpret_cast<uintptr_t>(workspace), reinterpret_cast<uintptr_t>(workspace) + need};
  if (overlaps(rw, span(scores, 4, rows, rows > 1 ? score_stride : W, 1, 0, 1, 0, W)) ||
      overlaps(rw, span(idx, 4, rows, rows > 1 ? idx_stride : k, 1, 0, 1, 0, k)) ||
      (lengths && overlaps(rw, span(lengths, 4, rows, 1, 1, 0, 1, 0, 1))))
    return fail(QSA_ERR_INVALID_ARG, "workspace overlaps an argument");
  return launch_topk(a, static_cast<cudaStream_t>(stream), nullptr, static_cast<uint8_t*>(workspace));
}

qsa_status_t qsa_mqa_prefill_topk_noalloc(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                                          int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke,
                                          int64_t T, float scale, int32_t W, int32_t topk_k, int32_t* idx,
                                          int64_t idx_stride, void* stream) {
  if (T < 0 || W < 1) return fail(QSA_ERR_INVALID_ARG, "T must be non-negative and W positive");
  // one chunk of min(T, 64) rows of scores plus the selection state must fit
  const int64_t rows = std::min<int64_t>(T, 64);
  if ((size_t)rows * (size_t)W * sizeof(float) + kPredBytes > kNoAllocScratchBytes)
    return fail(QSA_ERR_WORKSPACE,
                "W = %d needs %lld bytes of scratch for one chunk of %lld rows; the static scratch holds %zu", W,
                (long long)((size_t)rows * (size_t)W * sizeof(float) + kPredBytes), (long long)rows,
                kNoAllocScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(QSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      // first call on this device (with it current): the device address of the array
      e = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
      if (e != cudaSuccess) {
        g_noalloc_ptr[dev] = nullptr;
        return fail(QSA_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
      }
    }
    scratch = g_noalloc_ptr[dev];
  }
  return qsa_mqa_prefill_topk(q, q_stride_t, q_stride_h, k, k_stride, Nk, ks, ke, T, scale, W, topk_k, idx,
                              idx_stride, scratch, kNoAllocScratchBytes, stream);
}

size_t qsa_prefill_topk_workspace_size(int64_t T, int32_t W) {
  if (T <= 0 || W <= 0) return 0;
  return (size_t)T * (size_t)W * sizeof(float) + kPredBytes;
}

qsa_status_t qsa_mqa_prefill_topk(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k,
                                  int64_t k_stride, int64_t Nk, const int32_t* ks, const int32_t* ke, int64_t T,
                                  float scale, int32_t W, int32_t topk_k, int32_t* idx, int64_t idx_stride,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (W < 1) return fail(QSA_ERR_UNSUPPORTED, "W = %d must be in [1, 65536]", W);
  float* ws = static_cast<float*>(workspace);
  PrefillArgs pa{q, q_stride_t, q_stride_h, k, k_stride, Nk, ks, ke, T, scale, ws, (int64_t)W, W};
  TopkArgs ta{ws, (int64_t)W, nullptr, T, W, topk_k, idx, idx_stride};
  {
    // k, W and alignment; the workspace holds one chunk of rows, not T, so
    // its overlaps are checked below against the chunk actually used
    TopkArgs one = ta;
    one.rows = std::min<int64_t>(T, 1);
    one.idx_stride = topk_k;
    qsa_status_t st = validate_topk(one);
    if (st != QSA_OK) return st;
  }
  if (T > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "rows = %lld exceeds 2^31 - 1", (long long)T);
  if (T > 1 && idx_stride < topk_k)
    return fail(QSA_ERR_INVALID_ARG, "idx_stride = %lld is below k = %d", (long long)idx_stride, topk_k);
  qsa_status_t st;
  if (T < 0 || Nk < 0) return fail(QSA_ERR_INVALID_ARG, "T and Nk must be non-negative");
  if (T == 0) return ok();
  if (!workspace) return fail(QSA_ERR_WORKSPACE, "workspace is null");
  if (!aligned(workspace, 16)) return fail(QSA_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  // the workspace ends with the top-k kernel's per-CTA predictions, carried
  // from one chunk to the next
  if (workspace_bytes < kPredBytes)
    return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes is too small", workspace_bytes);
  const size_t score_bytes = (workspace_bytes - kPredBytes) & ~size_t(15);
  float* pred_state = reinterpret_cast<float*>(static_cast<char*>(workspace) + score_bytes);
  const int64_t row_bytes = (int64_t)W * 4;
  int64_t chunk = (int64_t)(score_bytes / (size_t)row_bytes);
  const int64_t min_rows = std::min<int64_t>(T, qsa::prefill::BT);
  if (chunk < min_rows)
    return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes holds %lld rows of W = %d floats; at least %lld needed",
                workspace_bytes, (long long)chunk, W, (long long)min_rows);
  if (chunk >= T) chunk = T;
  else chunk = chunk / qsa::prefill::BT * qsa::prefill::BT;
  {
    // the workspace must not overlap anything the calls read or write
    const Range rw = span(ws, 4, chunk, W, 1, 0, 1, 0, W);
    const Range rq = span(q, 2, T, q_stride_t, 4, q_stride_h, 1, 0, 128);
    const Range ri = span(idx, 4, T, idx_stride, 1, 0, 1, 0, topk_k);
    bool bad = overlaps(rw, rq) || overlaps(rw, ri) || overlaps(rw, span(ks, 4, T, 1, 1, 0, 1, 0, 1)) ||
               overlaps(rw, span(ke, 4, T, 1, 1, 0, 1, 0, 1));
    if (Nk > 0) bad = bad || overlaps(rw, span(k, 2, Nk, k_stride, 1, 0, 1, 0, 128));
    if (bad) return fail(QSA_ERR_INVALID_ARG, "workspace overlaps an input or idx");
  }
  {
    cudaError_t e = cudaMemsetAsync(pred_state, 0, kPredBytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  }
  for (int64_t r0 = 0; r0 < T; r0 += chunk) {
    const int64_t n = std::min(chunk, T - r0);
    PrefillArgs c = pa;
    c.q = static_cast<const uint16_t*>(q) + r0 * q_stride_t;
    c.ks = ks + r0;
    c.ke = ke + r0;
    c.T = n;
    st = validate_prefill(c);
    if (st != QSA_OK) return st;
    st = launch_prefill(c, static_cast<cudaStream_t>(stream));
    if (st != QSA_OK) return st;
    TopkArgs t = ta;
    t.rows = n;
    t.idx = idx + r0 * idx_stride;
    st = launch_topk(t, static_cast<cudaStream_t>(stream), pred_state);
    if (st != QSA_OK) return st;
  }
  return ok();
}

qsa_status_t qsa_expand_block_indices(const int32_t* blocks, int64_t blk_stride, int32_t k, const int32_t* cu_seqlens_q,
                                      const int32_t* seq_lens, int32_t R, int64_t T, int32_t* token_idx,
                                      int64_t tok_stride, void* stream) {
  if (T < 0 || R < 0) return fail(QSA_ERR_INVALID_ARG, "T and R must be non-negative");
  if (k < 1 || k > 512) return fail(QSA_ERR_UNSUPPORTED, "k = %d blocks per row; 1..512 supported", k);
  if (T == 0) return ok();
  if (R == 0) return fail(QSA_ERR_INVALID_ARG, "T > 0 rows need at least one request");
  if (T > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "T = %lld rows exceeds 2^31 - 1", (long long)T);
  if (!blocks || !cu_seqlens_q || !seq_lens || !token_idx) return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(blocks, 4) || !aligned(token_idx, 4) || !aligned(cu_seqlens_q, 4) || !aligned(seq_lens, 4))
    return fail(QSA_ERR_ALIGNMENT, "index arrays must be 4-byte aligned");
  const int64_t width = 4 * (int64_t)k + 3;
  if (T > 1 && (blk_stride < k || tok_stride < width))
    return fail(QSA_ERR_INVALID_ARG, "blk_stride must be >= k and tok_stride >= 4k + 3");
  if (overlaps(span(token_idx, 4, T, tok_stride, 1, 0, 1, 0, width), span(blocks, 4, T, blk_stride, 1, 0, 1, 0, k)))
    return fail(QSA_ERR_INVALID_ARG, "token_idx overlaps blocks");
  int sms = 0;
  qsa_status_t st = device_info(&sms);
  if (st != QSA_OK) return st;
  qsa::attn::ExpandParams p{blocks, T > 1 ? blk_stride : k, k, cu_seqlens_q, seq_lens, R, T, token_idx,
                            T > 1 ? tok_stride : width};
  const int64_t blocks_n = (T * 32 + 255) / 256;
  qsa::attn::expand_kernel<<<(unsigned)blocks_n, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status("index expansion kernel");
}

size_t qsa_sparse_attention_workspace_size(int64_t T, int32_t Hq, int32_t Hkv, int32_t width) {
  if (T <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || width <= 0) return 0;
  int32_t splits = 0, cps = 0;
  attn_splits(T, Hkv, width, &splits, &cps);
  const size_t group = (size_t)(Hq / Hkv);
  return (size_t)T * (size_t)Hkv * (size_t)splits * group * (qsa::attn::D + 2) * sizeof(float);
}

qsa_status_t qsa_sparse_attention(const void* q, int64_t q_stride_t, int64_t q_stride_h, int32_t Hq, const void* k_cache,
                                  const void* v_cache, int64_t num_pages, int32_t page_size, int64_t kv_page_stride,
                                  int64_t kv_row_stride, int64_t kv_head_stride, int32_t Hkv,
                                  const int32_t* page_table, int64_t pt_stride, int32_t max_pages,
                                  const int32_t* cu_seqlens_q, const int32_t* seq_lens, int32_t R,
                                  const int32_t* token_idx, int64_t tok_stride, int32_t width, int64_t T,
                                  const float* gate, float scale, void* out, int64_t out_stride_t, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  using qsa::attn::D;
  if (T < 0 || R < 0 || width < 0 || max_pages < 0) return fail(QSA_ERR_INVALID_ARG, "negative size argument");
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Hq / Hkv > qsa::attn::MAX_GROUP)
    return fail(QSA_ERR_UNSUPPORTED, "Hq = %d, Hkv = %d: Hq must be a multiple of Hkv with at most %d query heads per KV head",
                Hq, Hkv, qsa::attn::MAX_GROUP);
  if (page_size < 1) return fail(QSA_ERR_INVALID_ARG, "page_size must be positive");
  if (num_pages < 1 || num_pages > INT32_MAX) return fail(QSA_ERR_INVALID_ARG, "num_pages out of range");
  if (!std::isfinite(scale)) return fail(QSA_ERR_INVALID_ARG, "scale must be finite");
  if (T == 0) return ok();
  if (T > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "T = %lld rows exceeds 2^31 - 1", (long long)T);
  if (R == 0) return fail(QSA_ERR_INVALID_ARG, "T > 0 rows need at least one request");
  if (!q || !k_cache || !v_cache || !cu_seqlens_q || !seq_lens || !out || (width > 0 && !token_idx) ||
      (max_pages > 0 && !page_table))
    return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
    return fail(QSA_ERR_ALIGNMENT, "q, k_cache, v_cache and out must be 16-byte aligned");
  if ((gate && !aligned(gate, 4)) || (lse && !aligned(lse, 4)) || (token_idx && !aligned(token_idx, 4)) ||
      (page_table && !aligned(page_table, 4)))
    return fail(QSA_ERR_ALIGNMENT, "gate, lse, token_idx and page_table must be 4-byte aligned");
  const int64_t strides[6] = {T > 1 ? q_stride_t : 8, Hq > 1 ? q_stride_h : 8, num_pages > 1 ? kv_page_stride : 8,
                              page_size > 1 ? kv_row_stride : 8, Hkv > 1 ? kv_head_stride : 8,
                              T > 1 ? out_stride_t : 8};
  for (int i = 0; i < 6; ++i)
    if (strides[i] <= 0 || strides[i] % 8 != 0)
      return fail(QSA_ERR_ALIGNMENT, "strides must be positive multiples of 8 elements (got %lld)", (long long)strides[i]);
  if (Hq > 1 && q_stride_h < D) return fail(QSA_ERR_INVALID_ARG, "q_stride_h below the head dimension 256");
  if (Hkv > 1 && kv_head_stride < D) return fail(QSA_ERR_INVALID_ARG, "kv_head_stride below 256");
  if (page_size > 1 && kv_row_stride < (int64_t)Hkv * (Hkv > 1 ? kv_head_stride : D))
    return fail(QSA_ERR_INVALID_ARG, "kv_row_stride too small for Hkv heads");
  if (T > 1 && out_stride_t < (int64_t)Hq * D) return fail(QSA_ERR_INVALID_ARG, "out_stride_t below Hq * 256");
  if (T > 1 && width > 0 && tok_stride < width) return fail(QSA_ERR_INVALID_ARG, "tok_stride below width");
  if (max_pages > 0 && R > 1 && pt_stride < max_pages) return fail(QSA_ERR_INVALID_ARG, "pt_stride below max_pages");
  {
    const Range ro = span(out, 2, T, T > 1 ? out_stride_t : 0, Hq, D, 1, 0, D);
    bool bad = overlaps(ro, span(q, 2, T, T > 1 ? q_stride_t : 0, Hq, Hq > 1 ? q_stride_h : 0, 1, 0, D));
    const Range rk = span(k_cache, 2, num_pages, num_pages > 1 ? kv_page_stride : 0, page_size,
                          page_size > 1 ? kv_row_stride : 0, Hkv, Hkv > 1 ? kv_head_stride : 0, D);
    const Range rv = span(v_cache, 2, num_pages, num_pages > 1 ? kv_page_stride : 0, page_size,
                          page_size > 1 ? kv_row_stride : 0, Hkv, Hkv > 1 ? kv_head_stride : 0, D);
    bad = bad || overlaps(ro, rk) || overlaps(ro, rv);
    if (lse) bad = bad || overlaps(span(lse, 4, T, Hq, 1, 0, 1, 0, Hq), ro);
    if (bad) return fail(QSA_ERR_INVALID_ARG, "out overlaps an input (or lse)");
  }
  int32_t splits = 1, cps = 1;
  attn_splits(T, Hkv, width, &splits, &cps);
  const size_t need = qsa_sparse_attention_workspace_size(T, Hq, Hkv, width > 0 ? width : 1);
  if (!workspace || workspace_bytes < need)
    return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes; %zu needed", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(QSA_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  int sms = 0;
  qsa_status_t st = device_info(&sms);
  if (st != QSA_OK) return st;
  qsa::attn::Params p;
  p.q = static_cast<const uint16_t*>(q);
  p.q_st = q_stride_t;
  p.q_sh = q_stride_h;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.k = static_cast<const uint16_t*>(k_cache);
  p.v = static_cast<const uint16_t*>(v_cache);
  p.num_pages = num_pages;
  p.page_size = page_size;
  p.kv_page_stride = kv_page_stride;
  p.kv_row_stride = kv_row_stride;
  p.kv_head_stride = kv_head_stride;
  p.page_table = page_table;
  p.pt_stride = pt_stride;
  p.max_pages = max_pages;
  p.cu = cu_seqlens_q;
  p.seq_lens = seq_lens;
  p.R = R;
  p.tok = token_idx;
  p.tok_stride = T > 1 ? tok_stride : width;
  p.width = width;
  p.T = T;
  p.splits = splits;
  p.chunks_per_split = cps;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634);
  float* ws = static_cast<float*>(workspace);
  p.part_o = ws;
  p.part_ml = ws + (size_t)T * Hkv * splits * p.group * D;
  p.gate = gate;
  p.out = static_cast<uint16_t*>(out);
  p.out_st = T > 1 ? out_stride_t : (int64_t)Hq * D;
  p.lse = lse;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t ctas = T * Hkv * splits;
  if (ctas > INT32_MAX) return fail(QSA_ERR_UNSUPPORTED, "too many rows for one launch");
  qsa::attn::attn_kernel<<<(unsigned)ctas, qsa::attn::THREADS, qsa::attn::SMEM_BYTES, s>>>(p);
  st = launch_status("sparse attention kernel");
  if (st != QSA_OK) return st;
  const int64_t warps = T * Hq;
  qsa::attn::combine_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>(p);
  return launch_status("sparse attention combine kernel");
}

// Workspace of qsa_mqa_paged_batch: the prefill keys packed (at most W per
// prefill request, 256 bytes each), then ks and ke of the prefill rows.
static size_t paged_batch_layout(int32_t R, int32_t D, int64_t prefill_rows, int32_t W, size_t* ks_off,
                                 size_t* ke_off) {
  const size_t keys = (size_t)(R - D) * (size_t)W * 256;
  const size_t iv = ((size_t)prefill_rows * 4 + 15) & ~size_t(15);
  *ks_off = keys;
  *ke_off = keys + iv;
  return keys + 2 * iv;
}

size_t qsa_mqa_paged_batch_workspace_size(int32_t R, int32_t num_decodes, int32_t decode_query_len, int64_t T,
                                          int32_t W) {
  if (R <= 0 || num_decodes < 0 || num_decodes > R || W <= 0 || T < 0) return 0;
  const int64_t rows = T - (int64_t)num_decodes * (num_decodes > 0 ? decode_query_len : 0);
  if (rows <= 0 || num_decodes == R) return 0;
  size_t a, b;
  return paged_batch_layout(R, num_decodes, rows, W, &a, &b);
}

qsa_status_t qsa_mqa_paged_batch(const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k_cache,
                                 int64_t num_pages, int32_t page_size, int64_t k_page_stride, int64_t k_row_stride,
                                 const int32_t* page_table, int64_t pt_stride, int32_t max_pages,
                                 const int32_t* cu_seqlens_q, const int32_t* seq_lens, int32_t R, int32_t num_decodes,
                                 int32_t decode_query_len, int64_t T, float scale, float* out, int64_t out_stride,
                                 int32_t W, void* workspace, size_t workspace_bytes, void* stream) {
  const int32_t D = num_decodes;
  if (R < 0 || D < 0 || D > R || T < 0 || W < 0) return fail(QSA_ERR_INVALID_ARG, "negative or inconsistent counts");
  if (D > 0 && (decode_query_len < 1 || decode_query_len > 4))
    return fail(QSA_ERR_UNSUPPORTED, "decode_query_len = %d; 1..4 supported", decode_query_len);
  const int64_t row0 = (int64_t)D * (D > 0 ? decode_query_len : 0);
  if (row0 > T) return fail(QSA_ERR_INVALID_ARG, "T = %lld rows is below the decode rows %lld", (long long)T,
                            (long long)row0);
  if (T > row0 && D == R) return fail(QSA_ERR_INVALID_ARG, "rows past the decode requests need prefill requests");
  if (R - D > qsa::batch::MAX_PREFILL)
    return fail(QSA_ERR_UNSUPPORTED, "%d prefill requests; at most %d per call", R - D, qsa::batch::MAX_PREFILL);
  if ((int64_t)(R - D) * W > INT32_MAX)
    return fail(QSA_ERR_UNSUPPORTED, "prefill requests x W = %lld keys exceeds 2^31 - 1", (long long)(R - D) * W);
  if (page_size < 8 || page_size > 1024)
    return fail(QSA_ERR_UNSUPPORTED, "page_size = %d; supported page sizes are 8 .. 1024", page_size);
  if (T == 0 || W == 0) return ok();
  if (!q || !k_cache || !cu_seqlens_q || !seq_lens || !out || (max_pages > 0 && !page_table))
    return fail(QSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(cu_seqlens_q, 4) || !aligned(seq_lens, 4)) return fail(QSA_ERR_ALIGNMENT, "index arrays must be 4-byte aligned");
  if (T > 1 && out_stride < W) return fail(QSA_ERR_INVALID_ARG, "out_stride below W");
  if (T > 1 && (q_stride_t <= 0 || q_stride_t % 8 != 0))
    return fail(QSA_ERR_ALIGNMENT, "q_stride_t must be a positive multiple of 8");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t ostride = T > 1 ? out_stride : W;
  const int64_t qst = T > 1 ? q_stride_t : 4 * q_stride_h;
  qsa_status_t st;
  // every check that can fail runs before the first launch
  qsa::batch::Params bp;
  PrefillArgs pa{};
  const bool has_prefill = T > row0;
  if (has_prefill) {
    size_t ks_off = 0, ke_off = 0;
    const size_t need = paged_batch_layout(R, D, T - row0, W, &ks_off, &ke_off);
    if (!workspace || workspace_bytes < need)
      return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes; %zu needed", workspace_bytes, need);
    if (!aligned(workspace, 16)) return fail(QSA_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    if (num_pages < 1 || num_pages > INT32_MAX) return fail(QSA_ERR_INVALID_ARG, "num_pages out of range");
    if (!aligned(k_cache, 16) || k_row_stride < 128 || k_row_stride % 8 != 0 ||
        (num_pages > 1 && (k_page_stride <= 0 || k_page_stride % 8 != 0)))
      return fail(QSA_ERR_ALIGNMENT, "k_cache must be 16-byte aligned with strides that are multiples of 8");
    if (max_pages > 0 && R > 1 && pt_stride < max_pages)
      return fail(QSA_ERR_INVALID_ARG, "pt_stride = %lld is below max_pages = %d", (long long)pt_stride, max_pages);
    char* ws = static_cast<char*>(workspace);
    bp.cu = cu_seqlens_q;
    bp.seq_lens = seq_lens;
    bp.R = R;
    bp.D = D;
    bp.row0 = row0;
    bp.T = T;
    bp.k_cache = static_cast<const uint16_t*>(k_cache);
    bp.num_pages = num_pages;
    bp.page_size = page_size;
    bp.k_page_stride = num_pages > 1 ? k_page_stride : 0;
    bp.k_row_stride = k_row_stride;
    bp.page_table = page_table;
    bp.pt_stride = pt_stride;
    bp.max_pages = max_pages;
    bp.W = W;
    bp.packed = reinterpret_cast<uint16_t*>(ws);
    bp.ks = reinterpret_cast<int32_t*>(ws + ks_off);
    bp.ke = reinterpret_cast<int32_t*>(ws + ke_off);
    bp.out = out;
    bp.out_stride = ostride;
    const int64_t cap = (int64_t)(R - D) * W;
    pa = PrefillArgs{static_cast<const uint16_t*>(q) + row0 * qst, qst, q_stride_h, bp.packed, 128, cap,
                     bp.ks, bp.ke, T - row0, scale, out + row0 * ostride, ostride, W};
    st = validate_prefill(pa);
    if (st != QSA_OK) return st;
    const Range rw = span(workspace, 1, 1, 0, 1, 0, 1, 0, (int64_t)need);
    if (overlaps(rw, span(out, 4, T, ostride, 1, 0, 1, 0, W)) || overlaps(rw, span(q, 2, T, qst, 4, q_stride_h, 1, 0, 128)))
      return fail(QSA_ERR_INVALID_ARG, "workspace overlaps q or out");
  }
  // 1. decode rows: requests 0 .. D-1, decode_query_len rows each (validated, then launched)
  if (D > 0) {
    const int32_t Q = decode_query_len;
    st = decode_common(q, Q * qst, qst, q_stride_h, k_cache, qsa::decode::Fmt::BF16, 1.f, num_pages, page_size,
                       k_page_stride, k_row_stride, page_table, pt_stride, max_pages, seq_lens, D, Q, scale, out,
                       Q * ostride, ostride, W, stream, /*pdl=*/true);
    if (st != QSA_OK) return st;
  }
  if (!has_prefill) return ok();
  int sms = 0;
  st = device_info(&sms);
  if (st != QSA_OK) return st;
  // 2. the metadata step for the prefill requests: intervals and packed keys
  launch_pdl(qsa::batch::gather_kernel, dim3(sms * 4), dim3(qsa::batch::THREADS), qsa::batch::SMEM_BYTES, s, bp);
  st = launch_status("paged-batch metadata kernel");
  if (st != QSA_OK) return st;
  // 3. prefill rows over the packed keys
  st = launch_prefill(pa, s, /*pdl=*/true);
  if (st != QSA_OK) return st;
  // 4. keys whose page is missing
  launch_pdl(qsa::batch::fixup_kernel, dim3(R - D), dim3(qsa::batch::THREADS), 0, s, bp);
  return launch_status("paged-batch fix-up kernel");
}

}  // extern "C"
