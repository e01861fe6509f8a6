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

// TMA tensor-map encoder (driver entry point, resolved once).
si_status encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                         uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                         uint32_t box_outer);

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
};

// Decodes MXFP4 rows (codes [rows, D/2], E8M0 scales [rows, D/32]) to bf16 [rows, D].
si_status launch_mxfp4_to_bf16(const void* codes, const void* scales, long long rows, int D, void* out,
                               cudaStream_t stream);

// Two-stage indexer (blocks of G keys scored by their pooled key, the best
// n_keep kept, then the top-k of their keys): scratch bytes and driver.
size_t two_stage_workspace_bytes(int B, int S, int T, int G, int n_keep, int chunk);
si_status launch_two_stage(const void* q, const void* kc, const float* w, int B, int S, int T, int m, int k,
                           int G, int n_keep, int chunk, int32_t* out_idx, float* out_score, void* workspace,
                           size_t workspace_bytes, uint64_t wait_limit_ns, cudaStream_t stream);

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
