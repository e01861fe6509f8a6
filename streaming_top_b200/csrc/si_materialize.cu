// Materialize path: the method StreamIndex contrasts with (abstract: public
// CSA implementations build the [B, S, H_I, T] fp32 score tensor before the
// top-k reduction).  Kept in the library as ground truth for small S:
//   1. logits  L[b,t,h,s] = sum_d q[b,t,h,d] * kc[b,s,d]      (all t, h, s)
//   2. reduce  I[b,t,s]   = sum_h w[b,t,h] * ReLU(L[b,t,h,s])  (visible s)
//   3. select  per row: full bitonic sort of the visible keys, first k kept.
// Plain CUDA-core kernels; every sum runs in index order with one fp32
// rounding per fused multiply-add.
#include <cuda_runtime.h>

#include <cstdint>

#include "si_internal.h"

namespace si {
namespace {

constexpr int TILE = 64;   // output tile edge of the logits kernel
constexpr int KC = 32;     // d-chunk staged in shared memory

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// L[(b*S*H + r)*T + s] for r = t*H + h: q rows x keys, one 64x64 tile per CTA.
__global__ void __launch_bounds__(256) logits_kernel(const uint16_t* __restrict__ q,
                                                     const uint16_t* __restrict__ kc,
                                                     float* __restrict__ L, int S, int T, int H,
                                                     int D) {
  __shared__ float As[KC][TILE + 1];
  __shared__ float Bs[KC][TILE + 1];
  const int b = blockIdx.z;
  const long long rows = static_cast<long long>(S) * H;
  const long long r0 = static_cast<long long>(blockIdx.x) * TILE;
  const int s0 = blockIdx.y * TILE;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const uint16_t* qb = q + static_cast<size_t>(b) * rows * D;
  const uint16_t* kb = kc + static_cast<size_t>(b) * T * D;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int d0 = 0; d0 < D; d0 += KC) {
    for (int e = threadIdx.x; e < TILE * KC; e += 256) {
      const int r = e / KC, dd = e % KC, d = d0 + dd;
      const long long row = r0 + r;
      As[dd][r] = (row < rows && d < D) ? bf16_to_f32(qb[static_cast<size_t>(row) * D + d]) : 0.f;
      const int s = s0 + r;
      Bs[dd][r] = (s < T && d < D) ? bf16_to_f32(kb[static_cast<size_t>(s) * D + d]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int dd = 0; dd < KC; ++dd) {
      float a[4], c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[dd][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) c[j] = Bs[dd][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], c[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long row = r0 + ty * 4 + i;
    if (row >= rows) continue;
    float* out = L + (static_cast<size_t>(b) * rows + row) * T;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int s = s0 + tx * 4 + j;
      if (s < T) out[s] = acc[i][j];
    }
  }
}

// I[(b*S + t)*T + s] = sum_h w * ReLU(L) for visible s; -inf otherwise.
__global__ void reduce_kernel(const float* __restrict__ L, const float* __restrict__ w,
                              float* __restrict__ I, int S, int T, int H, int m) {
  const long long row = blockIdx.x;  // b*S + t
  const int t = static_cast<int>(row % S);
  const int s = blockIdx.y * blockDim.x + threadIdx.x;
  if (s >= T) return;
  const int nv = (t + 1) / m < T ? (t + 1) / m : T;
  float acc = 0.f;
  if (s < nv) {
    const float* lr = L + static_cast<size_t>(row) * H * T + s;
    const float* wr = w + static_cast<size_t>(row) * H;
    for (int h = 0; h < H; ++h) acc = fmaf(wr[h], fmaxf(lr[static_cast<size_t>(h) * T], 0.f), acc);
  } else {
    acc = -__int_as_float(0x7f800000);
  }
  I[static_cast<size_t>(row) * T + s] = acc;
}

__device__ __forceinline__ uint32_t ord32(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord32(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// One CTA per row: sort the visible keys by (score desc, index asc).
__global__ void __launch_bounds__(1024) select_kernel(const float* __restrict__ I, int S, int T,
                                                      int m, int k, int32_t* __restrict__ out_idx,
                                                      float* __restrict__ out_score) {
  extern __shared__ uint64_t keys[];
  const long long row = blockIdx.x;
  const int t = static_cast<int>(row % S);
  const int n = (t + 1) / m < T ? (t + 1) / m : T;
  int np = 1;
  while (np < n) np <<= 1;
  const float* ir = I + static_cast<size_t>(row) * T;
  for (int s = threadIdx.x; s < np; s += blockDim.x)
    keys[s] = s < n ? ((static_cast<uint64_t>(ord32(ir[s])) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(s))) : 0ull;
  __syncthreads();
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (np >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t x = keys[lo], y = keys[hi];
        if ((x < y) == desc) {
          keys[lo] = y;
          keys[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  const size_t ob = static_cast<size_t>(row) * k;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    int32_t id = -1;
    float sc = -__int_as_float(0x7f800000);
    if (j < n) {
      id = static_cast<int32_t>(~static_cast<uint32_t>(keys[j]));
      sc = unord32(static_cast<uint32_t>(keys[j] >> 32));
    }
    out_idx[ob + j] = id;
    if (out_score) out_score[ob + j] = sc;
  }
}

}  // namespace

size_t materialize_workspace_bytes(int B, int S, int T, int H) {
  const size_t rows = static_cast<size_t>(B) * S;
  return rows * H * T * sizeof(float) + rows * T * sizeof(float) + 256;
}

si_status launch_materialize(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H, int D, int m, int k, int32_t* out_idx, float* out_score,
                             cudaStream_t stream, void* workspace, size_t workspace_bytes) {
  const size_t need = materialize_workspace_bytes(B, S, T, H);
  void* ws = workspace;
  bool owned = false;
  cudaError_t e;
  if (ws) {
    if (workspace_bytes < need)
      return fail(SI_ERR_INVALID_ARGUMENT, "workspace of %zu bytes < %zu needed", workspace_bytes, need);
  } else {
    size_t free_b = 0, total_b = 0;
    e = cudaMemGetInfo(&free_b, &total_b);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemGetInfo");
    if (need > free_b)
      return fail(SI_ERR_OUT_OF_MEMORY,
                  "materialize needs %zu bytes for the [B,S,H_I,T] logits and [B,S,T] scores; %zu free",
                  need, free_b);
    const si_status sa = scratch_alloc(&ws, need, stream, "the materialized logits and scores");
    if (sa != SI_OK) return sa;
    owned = true;
  }
  float* L = static_cast<float*>(ws);
  float* I = L + static_cast<size_t>(B) * S * H * T;
  const long long rows = static_cast<long long>(S) * H;
  si_status st = SI_OK;
  {
    dim3 grid(static_cast<unsigned>((rows + TILE - 1) / TILE), (T + TILE - 1) / TILE, B);
    logits_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(q),
                                            static_cast<const uint16_t*>(kc), L, S, T, H, D);
    e = cudaGetLastError();
    if (e != cudaSuccess) st = cuda_fail(e, "logits_kernel launch");
  }
  if (st == SI_OK) {
    dim3 grid(static_cast<unsigned>(static_cast<long long>(B) * S), (T + 255) / 256);
    reduce_kernel<<<grid, 256, 0, stream>>>(L, w, I, S, T, H, m);
    e = cudaGetLastError();
    if (e != cudaSuccess) st = cuda_fail(e, "reduce_kernel launch");
  }
  if (st == SI_OK) {
    int np = 1;
    while (np < T) np <<= 1;
    const size_t smem = static_cast<size_t>(np) * sizeof(uint64_t);
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) st = cuda_fail(e, "cudaFuncSetAttribute(select_kernel)");
    if (st == SI_OK) {
      select_kernel<<<static_cast<unsigned>(static_cast<long long>(B) * S), 1024, smem, stream>>>(
          I, S, T, m, k, out_idx, out_score);
      e = cudaGetLastError();
      if (e != cudaSuccess) st = cuda_fail(e, "select_kernel launch");
    }
  }
  if (owned) {
    e = cudaFreeAsync(ws, stream);
    if (e != cudaSuccess && st == SI_OK) st = cuda_fail(e, "cudaFreeAsync");
  }
  return st;
}

}  // namespace si
