// C-ABI entry points of the indexer top-k library: argument validation,
// error reporting, the device error record and TMA tensor-map encoding.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "si_internal.h"

namespace si {
namespace {

thread_local char g_last_error[512] = "";

// Error record written by the kernels of this library (per device).
__device__ int g_device_error[4];

// Test hook: the next g_fail_allocs scratch allocations of the library fail.
std::atomic<int> g_fail_allocs{0};

// The library's stream-ordered memory pool per device.  Scratch that calls
// allocate and free on their stream comes from it; it keeps up to
// kPoolKeepBytes of freed memory between calls (the default pool would give
// it back at every synchronisation and make the next call map it anew).
constexpr int kMaxDevices = 64;
constexpr uint64_t kPoolKeepBytes = 1ull << 30;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kMaxDevices] = {};

cudaError_t library_pool(int dev, bool renew, cudaMemPool_t* out) {
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (renew && g_pool[dev]) g_pool[dev] = nullptr;  // a device reset destroyed it: make another
  if (!g_pool[dev]) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof props);
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = kPoolKeepBytes;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return e;
    }
    g_pool[dev] = pool;
  }
  *out = g_pool[dev];
  return cudaSuccess;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s per bounded wait

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

si_status fail(si_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return st;
}

si_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SI_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// The record's address in the current context, asked for on every call (no
// cache that a device reset or another context could make stale).
si_status device_error_record(int** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_device_error);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error record)");
  *out = static_cast<int*>(p);
  return SI_OK;
}

si_status error_word(const si_options* opt, int** out) {
  if (opt && opt->device_status) {
    if (reinterpret_cast<uintptr_t>(opt->device_status) % 8 != 0)
      return fail(SI_ERR_INVALID_ARGUMENT, "device_status must be 8-byte aligned");
    *out = opt->device_status;
    return SI_OK;
  }
  return device_error_record(out);
}

si_status scratch_alloc(void** p, size_t bytes, cudaStream_t stream, const char* what) {
  *p = nullptr;
  int left = g_fail_allocs.load();
  while (left > 0 && !g_fail_allocs.compare_exchange_weak(left, left - 1)) {
  }
  if (left > 0)
    return fail(SI_ERR_OUT_OF_MEMORY, "allocating %zu bytes for %s: failed by the allocation-failure test hook",
                bytes, what);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SI_ERR_UNSUPPORTED, "device index %d", dev);
  for (int attempt = 0; attempt < 2; ++attempt) {
    cudaMemPool_t pool = nullptr;
    e = library_pool(dev, attempt > 0, &pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(p, bytes, pool, stream);
    if (e == cudaSuccess) return SI_OK;
    cudaGetLastError();
    *p = nullptr;
    if (e == cudaErrorMemoryAllocation) break;
  }
  return fail(SI_ERR_OUT_OF_MEMORY, "cudaMallocFromPoolAsync(%zu) for %s: %s", bytes, what, cudaGetErrorString(e));
}

si_status encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                         uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                         uint32_t box_outer) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return fail(SI_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(g_encode_err));
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SI_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return SI_OK;
}

bool try_encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                        const uint64_t stride_bytes[2], const uint32_t box[3]) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return false;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {stride_bytes[0], stride_bytes[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

si_status check_common(const void* q, const void* kc, const float* w, int B, int S, int T, int H,
                       int D, int m, int k, const int32_t* out_idx, const float* out_score) {
  if (!q || !kc || !w || !out_idx)
    return fail(SI_ERR_INVALID_ARGUMENT, "q, kc, w and out_idx must be non-null device pointers");
  if (B < 1 || S < 1 || T < 1 || H < 1 || D < 1 || m < 1 || k < 1)
    return fail(SI_ERR_INVALID_ARGUMENT, "B, S, T, H_I, D, m, k must be >= 1 (got %d %d %d %d %d %d %d)",
                B, S, T, H, D, m, k);
  if (!aligned(q, 16) || !aligned(kc, 16) || !aligned(w, 16) || !aligned(out_idx, 4) ||
      (out_score && !aligned(out_score, 4)))
    return fail(SI_ERR_INVALID_ARGUMENT, "q, kc, w must be 16-byte aligned; outputs 4-byte aligned");
  return SI_OK;
}

}  // namespace si

namespace si {

// Scratch for MXFP4 keys decoded to bf16: [B, T, D] bf16 plus alignment slack.
size_t mxfp4_key_bytes(int B, int T, int D) {
  return static_cast<size_t>(B) * T * D * 2 + 256;
}

// The streaming top-k over rows row0 .. row0+S-1 of every sequence (S rows
// held in q, w and the outputs); row0 = 0, S = sequence length is the
// whole-sequence call.
si_status stream_topk_rows(const void* q, const void* kc, const float* w, int B, int row0, int S,
                           int T, int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                           void* stream, const si_options* opt) {
  si_status st = check_common(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score);
  if (st != SI_OK) return st;
  if (row0 < 0) return fail(SI_ERR_INVALID_ARGUMENT, "row0 must be >= 0 (got %d)", row0);
  if (static_cast<long long>(row0) + S > 0x7FFFFFFFll)
    return fail(SI_ERR_UNSUPPORTED, "row0 + rows must fit in 31 bits");
  si_options o;
  std::memset(&o, 0, sizeof o);
  if (opt) o = *opt;
  if (o.dtype != SI_DTYPE_BF16 && o.dtype != SI_DTYPE_FP8_E4M3 && o.dtype != SI_DTYPE_MXFP4_KEYS)
    return fail(SI_ERR_INVALID_ARGUMENT, "unknown dtype %d", static_cast<int>(o.dtype));
  if (o.dtype == SI_DTYPE_FP8_E4M3 && (!o.q_scale || !o.kc_scale))
    return fail(SI_ERR_INVALID_ARGUMENT, "fp8 inputs need q_scale and kc_scale");
  const bool mx = o.dtype == SI_DTYPE_MXFP4_KEYS;
  if (mx && !o.kc_mx_scale) return fail(SI_ERR_INVALID_ARGUMENT, "MXFP4 keys need kc_mx_scale");
  if (mx && o.workspace && (o.workspace_bytes < mxfp4_key_bytes(B, T, D)))
    return fail(SI_ERR_INVALID_ARGUMENT, "workspace of %zu bytes < %zu needed for the decoded keys",
                o.workspace_bytes, mxfp4_key_bytes(B, T, D));
  // default partition: 512 keys, halved while the pool for this k does not
  // fit in shared memory (an explicit key_tile is taken as given)
  int key_tile = o.key_tile;
  if (key_tile == 0) {
    const int fp8 = o.dtype == SI_DTYPE_FP8_E4M3;
    int ns = 0, cap = 0;
    size_t bytes = 0;
    key_tile = 512;
    while (key_tile > 64 && !stream_smem_plan(k, key_tile, fp8, &ns, &cap, &bytes)) key_tile >>= 1;
  }
  if (!(key_tile == 64 || (key_tile % 128 == 0 && key_tile >= 128 && key_tile <= 1024)))
    return fail(SI_ERR_INVALID_ARGUMENT, "key_tile must be 64 or a multiple of 128 up to 1024 (got %d)", key_tile);
  if (o.query_chunk < 0 || (o.query_chunk % 4) != 0)
    return fail(SI_ERR_INVALID_ARGUMENT, "query_chunk must be 0 or a positive multiple of 4 (got %d)", o.query_chunk);
  if (D != 128 || H_I != 64)
    return fail(SI_ERR_UNSUPPORTED, "streaming path implements D=128, H_I=64 (got D=%d, H_I=%d)", D, H_I);
  if (k > 2048) return fail(SI_ERR_UNSUPPORTED, "k <= 2048 (got %d)", k);
  if (static_cast<long long>(B) * S * H_I > 0x7FFFFFFFll || static_cast<long long>(B) * T > 0x7FFFFFFFll)
    return fail(SI_ERR_UNSUPPORTED, "B*S*H_I and B*T must fit in 31 bits");
  StreamConfig cfg;
  cfg.query_chunk = o.query_chunk;
  cfg.key_tile = key_tile;
  cfg.fp8 = o.dtype == SI_DTYPE_FP8_E4M3;
  cfg.q_scale = o.q_scale;
  cfg.kc_scale = o.kc_scale;
  cfg.wait_limit_ns = kDefaultWaitLimitNs;
  cfg.test_withhold = 0;
  cfg.unsorted = o.unsorted != 0;
  cfg.row0 = row0;
  st = error_word(&o, &cfg.err);
  if (st != SI_OK) return st;
  bool sorted_by_merge = false;
  cfg.out_sorted = &sorted_by_merge;
  // the caller's workspace: the decoded MXFP4 keys first, then the split-key partials
  if (o.workspace) {
    const size_t used = mx ? mxfp4_key_bytes(B, T, D) : 0;
    if (o.workspace_bytes > used) {
      cfg.split_ws = static_cast<uint8_t*>(o.workspace) + used;
      cfg.split_ws_bytes = o.workspace_bytes - used;
    }
  }
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // MXFP4 keys: decode them to bf16 scratch first (exact), then score as bf16
  void* kraw = nullptr;  // the allocation, when the library made it
  if (mx) {
    const size_t need = mxfp4_key_bytes(B, T, D);
    void* base = o.workspace;
    if (!base) {
      st = scratch_alloc(&kraw, need, cs, "the decoded MXFP4 keys");
      if (st != SI_OK) return st;
      base = kraw;
    }
    void* kdec = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(base) + 255) & ~static_cast<uintptr_t>(255));
    st = launch_mxfp4_to_bf16(kc, o.kc_mx_scale, static_cast<long long>(B) * T, D, kdec, cs);
    kc = kdec;
  }
  if (st == SI_OK) st = launch_stream_topk(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score, cs, cfg);
  // the kernel leaves each row's k results in pool order: sort them now
  // (rows that went through the split-key merge are sorted already)
  if (st == SI_OK && !cfg.unsorted && out_score && !sorted_by_merge)
    st = launch_row_sort(out_idx, out_score, static_cast<long long>(B) * S, k, cs);
  if (kraw) {
    const cudaError_t e = cudaFreeAsync(kraw, cs);
    if (e != cudaSuccess && st == SI_OK) st = cuda_fail(e, "cudaFreeAsync");
  }
  return st;
}

}  // namespace si

using namespace si;

extern "C" {

si_status si_indexer_topk_ex(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                             void* stream, const si_options* opt) {
  return stream_topk_rows(q, kc, w, B, 0, S, T, H_I, D, m, k, out_idx, out_score, stream, opt);
}

si_status si_indexer_topk_rows(const void* q, const void* kc, const float* w, int B, int row0, int R,
                               int T, int H_I, int D, int m, int k, int32_t* out_idx,
                               float* out_score, void* stream, const si_options* opt) {
  return stream_topk_rows(q, kc, w, B, row0, R, T, H_I, D, m, k, out_idx, out_score, stream, opt);
}

si_status si_sort_topk_rows(int32_t* idx, float* score, int64_t rows, int k, void* stream) {
  if (rows < 0) return fail(SI_ERR_INVALID_ARGUMENT, "rows must be >= 0 (got %lld)", static_cast<long long>(rows));
  if (k < 1 || k > 2048) return fail(SI_ERR_INVALID_ARGUMENT, "1 <= k <= 2048 (got %d)", k);
  if (rows == 0) return SI_OK;
  if (!idx || !score) return fail(SI_ERR_INVALID_ARGUMENT, "idx and score must be non-null");
  if (!aligned(idx, 4) || !aligned(score, 4))
    return fail(SI_ERR_INVALID_ARGUMENT, "idx and score must be 4-byte aligned");
  return launch_row_sort(idx, score, rows, k, static_cast<cudaStream_t>(stream));
}

si_status si_indexer_topk(const void* q, const void* kc, const float* w, int B, int S, int T,
                          int H_I, int D, int m, int k, int32_t* out_idx, float* out_score,
                          void* stream) {
  return si_indexer_topk_ex(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score, stream, nullptr);
}

// Test entry point (not declared in the public header): runs the streaming
// kernel with a short wait limit and one key tile withheld, so that its
// bounded waits run out and it exits with SI_ERR_TIMEOUT recorded.
si_status si_test_stream_timeout(const void* q, const void* kc, const float* w, int B, int S, int T,
                                 int m, int k, int32_t* out_idx, void* stream,
                                 unsigned long long wait_limit_ns, int32_t* device_status) {
  si_status st = check_common(q, kc, w, B, S, T, 64, 128, m, k, out_idx, nullptr);
  if (st != SI_OK) return st;
  StreamConfig cfg;
  cfg.query_chunk = 0;
  cfg.key_tile = 256;
  cfg.fp8 = 0;
  cfg.q_scale = nullptr;
  cfg.kc_scale = nullptr;
  cfg.wait_limit_ns = wait_limit_ns;
  cfg.test_withhold = 1;
  cfg.unsorted = false;
  si_options o;
  std::memset(&o, 0, sizeof o);
  o.device_status = device_status;
  st = error_word(&o, &cfg.err);
  if (st != SI_OK) return st;
  return launch_stream_topk(q, kc, w, B, S, T, 64, 128, m, k, out_idx, nullptr,
                            static_cast<cudaStream_t>(stream), cfg);
}

si_status si_indexer_materialize(const void* q, const void* kc, const float* w, int B, int S,
                                 int T, int H_I, int D, int m, int k, int32_t* out_idx,
                                 float* out_score, void* stream, const si_options* opt) {
  si_status st = check_common(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score);
  if (st != SI_OK) return st;
  if (opt && opt->dtype != SI_DTYPE_BF16)
    return fail(SI_ERR_UNSUPPORTED, "materialize path takes bf16 inputs");
  if (T > 16384) return fail(SI_ERR_UNSUPPORTED, "materialize path sorts rows of T <= 16384 (got %d)", T);
  return launch_materialize(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score,
                            static_cast<cudaStream_t>(stream), opt ? opt->workspace : nullptr,
                            opt ? opt->workspace_bytes : 0);
}

size_t si_indexer_workspace_size(int B, int S, int T, int H_I, int D, int m, int k, int materialize,
                                 const si_options* opt) {
  (void)m;
  if (B < 1 || S < 1 || T < 1 || H_I < 1 || D < 1 || k < 1) return 0;
  if (materialize) return materialize_workspace_bytes(B, S, T, H_I);
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    n_sm = 1024;  // no device to ask: a bound for any GPU
  }
  const size_t mxb = opt && opt->dtype == SI_DTYPE_MXFP4_KEYS ? mxfp4_key_bytes(B, T, D) : 0;
  return mxb + stream_split_bytes_bound(B, S, k, opt ? opt->query_chunk : 0, n_sm);
}

size_t si_two_stage_workspace_size(int B, int S, int T, int block, int n_keep, int query_chunk) {
  if (B < 1 || S < 1 || T < 1 || block < 1 || n_keep < 1 || query_chunk < 0) return 0;
  return two_stage_workspace_bytes(B, S, T, block, n_keep, query_chunk ? query_chunk : 16384);
}

si_status si_indexer_topk_two_stage(const void* q, const void* kc, const float* w, int B, int S, int T,
                                    int H_I, int D, int m, int k, int block, int n_keep, int32_t* out_idx,
                                    float* out_score, void* stream, const si_options* opt) {
  si_status st = check_common(q, kc, w, B, S, T, H_I, D, m, k, out_idx, out_score);
  if (st != SI_OK) return st;
  if (!out_score) return fail(SI_ERR_INVALID_ARGUMENT, "the two-stage path needs out_score");
  if (opt && opt->dtype != SI_DTYPE_BF16) return fail(SI_ERR_UNSUPPORTED, "the two-stage path takes bf16 inputs");
  if (block < 1 || block > 64 || n_keep < 1 || n_keep > 2048)
    return fail(SI_ERR_INVALID_ARGUMENT, "1 <= block <= 64 and 1 <= n_keep <= 2048 (got %d, %d)", block, n_keep);
  if (D != 128 || H_I != 64)
    return fail(SI_ERR_UNSUPPORTED, "two-stage path implements D=128, H_I=64 (got D=%d, H_I=%d)", D, H_I);
  if (k > 2048) return fail(SI_ERR_UNSUPPORTED, "k <= 2048 (got %d)", k);
  if (static_cast<long long>(m) * block > 0x7FFFFFFFll || static_cast<long long>(B) * S * H_I > 0x7FFFFFFFll)
    return fail(SI_ERR_UNSUPPORTED, "m*block and B*S*H_I must fit in 31 bits");
  const int chunk = opt && opt->query_chunk > 0 ? opt->query_chunk : 16384;
  int* err = nullptr;
  st = error_word(opt, &err);
  if (st != SI_OK) return st;
  return launch_two_stage(q, kc, w, B, S, T, m, k, block, n_keep, chunk, out_idx, out_score,
                          opt ? opt->workspace : nullptr, opt ? opt->workspace_bytes : 0, kDefaultWaitLimitNs,
                          err, static_cast<cudaStream_t>(stream));
}

si_status si_sparse_attention(const void* q, const void* kv, const int32_t* idx, int B, int S, int T, int H,
                              int Dk, int Dv, int k, float scale, void* out, float* lse, void* stream,
                              const si_options* opt) {
  if (!q || !kv || !idx || !out || !lse)
    return fail(SI_ERR_INVALID_ARGUMENT, "q, kv, idx, out and lse must be non-null device pointers");
  if (B < 1 || S < 1 || T < 1 || H < 1 || Dk < 1 || Dv < 1 || k < 1)
    return fail(SI_ERR_INVALID_ARGUMENT, "B, S, T, H, Dk, Dv, k must be >= 1");
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(idx, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return fail(SI_ERR_INVALID_ARGUMENT, "q, kv, idx, out must be 16-byte aligned; lse 4-byte aligned");
  if (!(scale >= 0.f) || scale != scale)
    return fail(SI_ERR_INVALID_ARGUMENT, "scale must be >= 0 (0 = 1/sqrt(Dk))");
  if (H != 64 || Dk != 576 || Dv != 512)
    return fail(SI_ERR_UNSUPPORTED, "sparse attention implements H=64, Dk=576, Dv=512 (got %d, %d, %d)", H, Dk, Dv);
  if (k % 128 != 0 || k > 512) return fail(SI_ERR_UNSUPPORTED, "k must be 128, 256, 384 or 512 (got %d)", k);
  if (static_cast<long long>(B) * S * H > 0x7FFFFFFFll || static_cast<long long>(B) * T > 0x7FFFFFFFll)
    return fail(SI_ERR_UNSUPPORTED, "B*S*H and B*T must fit in 31 bits");
  int* err = nullptr;
  si_status st = error_word(opt, &err);
  if (st != SI_OK) return st;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf(static_cast<float>(Dk));
  return launch_sparse_attention(q, kv, idx, B, S, T, k, sc, out, lse, err, kDefaultWaitLimitNs,
                                 static_cast<cudaStream_t>(stream));
}

si_status si_mxfp4_to_bf16(const void* codes, const void* scales, int64_t rows, int D, void* out,
                           void* stream) {
  if (rows < 0) return fail(SI_ERR_INVALID_ARGUMENT, "rows must be >= 0 (got %lld)", static_cast<long long>(rows));
  if (D < 32 || D % 32 != 0) return fail(SI_ERR_INVALID_ARGUMENT, "D must be a positive multiple of 32 (got %d)", D);
  if (rows == 0) return SI_OK;
  if (!codes || !scales || !out) return fail(SI_ERR_INVALID_ARGUMENT, "codes, scales and out must be non-null");
  if (!aligned(codes, 16) || !aligned(out, 16))
    return fail(SI_ERR_INVALID_ARGUMENT, "codes and out must be 16-byte aligned");
  return launch_mxfp4_to_bf16(codes, scales, static_cast<long long>(rows), D, out,
                              static_cast<cudaStream_t>(stream));
}

si_status si_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int* rec = nullptr;
  si_status st = device_error_record(&rec);
  if (st != SI_OK) return st;
  int h[4] = {0, 0, 0, 0};
  e = cudaMemcpy(h, rec, sizeof h, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error record");
  if (h[0] != 0) {
    e = cudaMemset(rec, 0, sizeof h);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error record");
    return fail(static_cast<si_status>(h[0]), "a kernel's bounded wait ran out (site %d)", h[1]);
  }
  return SI_OK;
}

const char* si_status_string(si_status s) {
  switch (s) {
    case SI_OK: return "SI_OK";
    case SI_ERR_INVALID_ARGUMENT: return "SI_ERR_INVALID_ARGUMENT";
    case SI_ERR_UNSUPPORTED: return "SI_ERR_UNSUPPORTED";
    case SI_ERR_OUT_OF_MEMORY: return "SI_ERR_OUT_OF_MEMORY";
    case SI_ERR_CUDA: return "SI_ERR_CUDA";
    case SI_ERR_TIMEOUT: return "SI_ERR_TIMEOUT";
  }
  return "SI_ERR_UNKNOWN";
}

const char* si_last_error(void) { return g_last_error; }

void si_test_fail_allocations(int n) { g_fail_allocs.store(n > 0 ? n : 0); }

int si_version(void) { return 300; }

}  // extern "C"
