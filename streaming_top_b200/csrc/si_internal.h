// Host-side declarations shared by the translation units of the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/streaming_top.h"
#include "../../include/streaming_top_test.h"

namespace si {

// Records `msg` as the calling thread's last error and returns `st`.
si_status fail(si_status st, const char* fmt, ...);
// Converts a CUDA runtime error into SI_ERR_CUDA with context.
si_status cuda_fail(cudaError_t e, const char* what);
// Host-side checks shared by every entry point: non-null pointers, sizes
// >= 1, 16-byte aligned inputs, 4-byte aligned outputs.
si_status check_common(const void* q, const void* kc, const float* w, int B, int S, int T, int H,
                       int D, int m, int k, const int32_t* out_idx, const float* out_score);

// Device-resident error record of this library on the current device:
// int[4] = {code, where, detail, spare}.  code 0 = none, SI_ERR_TIMEOUT =
// a bounded wait gave up.  Written by kernels with atomicCAS (first wins).
si_status device_error_record(int** out);
// The error word of a call: opt->device_status when given, else the
// device record above.
si_status error_word(const si_options* opt, int** out);

// Stream-ordered allocation of library scratch on `stream` from the
// library's memory pool of the current device (freed with cudaFreeAsync);
// SI_ERR_OUT_OF_MEMORY (with a message naming `what`) when it fails or when
// the allocation-failure test hook says so.
si_status scratch_alloc(void** p, size_t bytes, cudaStream_t stream, const char* what);

// TMA tensor-map encoder (driver entry point, resolved once).
si_status encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                         uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                         uint32_t box_outer);
// 3-D tiled tensor map (128-byte swizzle): dims[0] contiguous, strides (in
// bytes) of dims 1 and 2 in any order.  Returns false, recording no error,
// when the driver refuses the layout (the caller then uses 2-D boxes).
bool try_encode_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, const uint64_t dims[3],
                        const uint64_t stride_bytes[2], const uint32_t box[3]);

struct StreamConfig {
  int query_chunk;  // queries per launch (multiple of 4), or S
  int key_tile;     // partition length in keys: 64 or multiple of 128
  int fp8;          // 0 bf16, 1 e4m3
  const float* q_scale;
  const float* kc_scale;
  uint64_t wait_limit_ns;
  int test_withhold;  // test hook: withhold one key-tile load (timeout path)
  bool unsorted;      // leave rows in pool order (no in-kernel sort either)
  int row0 = 0;       // absolute position of the first query row held (row ranges)
  int* err = nullptr; // device error word the kernels write (int[2]: code, site)
  bool allow_split = true;     // split the keys of too few units over CTAs (then merge)
  void* split_ws = nullptr;    // optional scratch for the split partials
  size_t split_ws_bytes = 0;
  bool* out_sorted = nullptr;  // set when every row left the call sorted (split + merge)
};

// Merges split-key partial top-ks [rows][n_split][k] (index, score; -1 / -inf
// padded) into the exact top-k of each row, sorted, into out [rows][k].
si_status launch_merge_splits(const int32_t* part_idx, const float* part_score, long long rows, int n_split, int k,
                              int32_t* out_idx, float* out_score, cudaStream_t stream);
// Key partitions per unit (1 = no split) and an upper bound of the partials'
// bytes for a streaming call.
int stream_split_count(long long n_units, int max_kt, int n_sm, int k);
size_t stream_split_bytes_bound(int B, int S, int k, int query_chunk, int n_sm);

// The streaming top-k over rows row0 .. row0+S-1 of every sequence (q, w
// and the outputs hold S rows; device pointers): argument checks, the MXFP4
// key decode, the streaming kernel and the row sort.  The body of
// si_indexer_topk_ex / si_indexer_topk_rows.
si_status stream_topk_rows(const void* q, const void* kc, const float* w, int B, int row0, int S, int T,
                           int H_I, int D, int m, int k, int32_t* out_idx, float* out_score, void* stream,
                           const si_options* opt);
// Bytes of the bf16 copy of MXFP4 keys [B, T, D] (plus alignment slack).
size_t mxfp4_key_bytes(int B, int T, int D);

// Sparse attention over selected latents (H = 64, Dk = 576, Dv = 512, k a
// multiple of 128 up to 512).
si_status launch_sparse_attention(const void* q, const void* kv, const int32_t* idx, int B, int S, int T, int k,
                                  float scale, void* out, float* lse, int* err, uint64_t wait_limit_ns,
                                  cudaStream_t stream);

// Decodes MXFP4 rows (codes [rows, D/2], E8M0 scales [rows, D/32]) to bf16 [rows, D].
si_status launch_mxfp4_to_bf16(const void* codes, const void* scales, long long rows, int D, void* out,
                               cudaStream_t stream);

// Two-stage indexer (blocks of G keys scored by their pooled key, the best
// n_keep kept, then the top-k of their keys): scratch bytes and driver.
size_t two_stage_workspace_bytes(int B, int S, int T, int G, int n_keep, int chunk);
si_status launch_two_stage(const void* q, const void* kc, const float* w, int B, int S, int T, int m, int k,
                           int G, int n_keep, int chunk, int32_t* out_idx, float* out_score, void* workspace,
                           size_t workspace_bytes, uint64_t wait_limit_ns, int* err, cudaStream_t stream);

// Sorts rows [rows, k] of (idx, score) in place by (score desc, index asc).
si_status launch_row_sort(int32_t* idx, float* score, long long rows, int k, cudaStream_t stream);

// Shared-memory plan of the streaming kernel for (k, key_tile, fp8); returns
// false when it cannot fit.
bool stream_smem_plan(int k, int key_tile, int fp8, int* n_stages, int* pool_cap, size_t* bytes);

si_status launch_stream_topk(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H, int D, int m, int k, int32_t* out_idx, float* out_score,
                             cudaStream_t stream, const StreamConfig& cfg);

si_status launch_materialize(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H, int D, int m, int k, int32_t* out_idx, float* out_score,
                             cudaStream_t stream, void* workspace, size_t workspace_bytes);

size_t materialize_workspace_bytes(int B, int S, int T, int H);

}  // namespace si
