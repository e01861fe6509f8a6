// Row sort of a top-k result: every row of k (index, score) pairs is put in
// (score descending, index ascending) order, in place.
//
// The streaming kernel's managers select each query's exact top-k but store
// it in pool order; sorting there would take one warp tens of thousands of
// cycles per query while the scoring warps wait on it.  This pass sorts all
// rows afterwards with whole CTAs: the rows are read and written once
// (8 bytes per entry each way), a bitonic network on packed 64-bit keys runs
// in registers and warp shuffles (rows up to 512 entries, one warp per row)
// or in shared memory (longer rows, one CTA per row, block-wide barriers only
// for strides that cross a warp's 64-key window).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"
#include "si_topk.cuh"

namespace si {
namespace {

// (orderable score << 32) | ~index: unsigned order = score descending, then
// index ascending.  -0 ranks with +0.  Padding (-inf, -1) packs to
// 0x007FFFFF00000000, below every finite score and above the sentinel 0.
__device__ __forceinline__ uint64_t pack(float sc, int32_t id) {
  uint32_t u = __float_as_uint(sc);
  if (u == 0x80000000u) u = 0u;
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(o) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(id));
}

__device__ __forceinline__ void unpack(uint64_t key, float* sc, int32_t* id) {
  const uint32_t o = static_cast<uint32_t>(key >> 32);
  *id = static_cast<int32_t>(~static_cast<uint32_t>(key));
  *sc = __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// One row per CTA iteration; np = next power of two >= k (>= 64), entries
// [k, np) hold the sentinel 0.  Pair i of a stage touches keys lo, lo+stride
// with lo = 2i - (i mod stride); for stride < 64 the 32 pairs of warp w stay
// inside keys [64w, 64w+64), so a warp barrier suffices there.
__global__ void __launch_bounds__(256) row_sort_kernel(int32_t* __restrict__ idx,
                                                       float* __restrict__ score, long long rows,
                                                       int k, int np) {
  extern __shared__ uint64_t a[];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int half = np >> 1;
  for (long long r = blockIdx.x; r < rows; r += gridDim.x) {
    int32_t* ir = idx + r * k;
    float* sr = score + r * k;
    for (int i = tid; i < np; i += nt) a[i] = i < k ? pack(sr[i], ir[i]) : 0ull;
    __syncthreads();
    bool prev_wide = false;
    for (int size = 2; size <= np; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const bool wide = stride >= 64;
        if (wide || prev_wide) __syncthreads();
        else __syncwarp();
        for (int i = tid; i < half; i += nt) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool desc = (lo & size) == 0;
          const uint64_t x = a[lo], y = a[hi];
          if ((x < y) == desc) {
            a[lo] = y;
            a[hi] = x;
          }
        }
        prev_wide = wide;
      }
    }
    __syncthreads();
    for (int i = tid; i < k; i += nt) {
      float sc;
      int32_t id;
      unpack(a[i], &sc, &id);
      sr[i] = sc;
      ir[i] = id;
    }
    __syncthreads();
  }
}

// One compare-exchange stage of a bitonic network over the 32*E keys of a
// warp (lane l holds positions [l*E, l*E+E)): partners are `stride` apart and
// the run a position belongs to is sorted descending when
// (position & size) == 0, ascending otherwise, flipped when !desc.  Strides
// below E stay in registers; larger ones exchange with lane ^ (stride / E)
// and keep the larger or the smaller key after one comparison.
template <int E>
__device__ __forceinline__ void bitonic_stage(uint64_t (&v)[E], int lane, int size, int stride,
                                              bool desc) {
  if (stride >= E) {
    const int lm = stride / E;
    const bool lower = (lane & lm) == 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const bool run_desc = ((((lane * E + r) & size) == 0) == desc);
      const bool want_max = run_desc == lower;
      const uint64_t o = topk::shfl_xor_u64(v[r], lm);
      v[r] = ((o > v[r]) == want_max) ? o : v[r];
    }
  } else {
#pragma unroll
    for (int r = 0; r < E; ++r) {
      if (r & stride) continue;
      const bool run_desc = ((((lane * E + r) & size) == 0) == desc);
      const uint64_t a = v[r], b = v[r | stride];
      const bool sw = (a < b) == run_desc;
      v[r] = sw ? b : a;
      v[r | stride] = sw ? a : b;
    }
  }
}

// Full bitonic sort of a warp's 32*E keys, descending (ascending if !desc).
template <int E>
__device__ __forceinline__ void warp_sort(uint64_t (&v)[E], int lane, bool desc) {
#pragma unroll
  for (int size = 2; size <= 32 * E; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) bitonic_stage<E>(v, lane, size, stride, desc);
}

// The last stages of a bitonic sort: the warp's keys form a bitonic sequence;
// leave them sorted descending (ascending if !desc).
template <int E>
__device__ __forceinline__ void warp_merge(uint64_t (&v)[E], int lane, bool desc) {
#pragma unroll
  for (int stride = 16 * E; stride > 0; stride >>= 1) bitonic_stage<E>(v, lane, 64 * E, stride, desc);
}

template <int E>
__device__ __forceinline__ void warp_sort_desc(uint64_t (&v)[E], int lane) {
  warp_sort<E>(v, lane, true);
}

// Rows of up to 32*E entries, one warp per row, entirely in registers: lane
// l holds positions [l*E, l*E+E) and the bitonic network runs in registers
// (strides < E) and warp shuffles (strides >= E).  `vec`: k % 4 == 0 and
// both arrays 16-byte aligned, so each lane moves its entries in 16-byte
// pieces.
template <int E>
__global__ void __launch_bounds__(128) row_sort_warp_kernel(int32_t* __restrict__ idx,
                                                            float* __restrict__ score,
                                                            long long rows, int k, int vec) {
  const int lane = threadIdx.x & 31;
  const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = w0; r < rows; r += nw) {
    int32_t* ir = idx + r * k;
    float* sr = score + r * k;
    uint64_t v[E];
    if (E >= 4 && vec) {
#pragma unroll
      for (int j = 0; j < E; j += 4) {
        const int i = lane * E + j;
        if (i < k) {
          const int4 a = *reinterpret_cast<const int4*>(ir + i);
          const float4 b = *reinterpret_cast<const float4*>(sr + i);
          v[j] = pack(b.x, a.x);
          v[j + 1] = pack(b.y, a.y);
          v[j + 2] = pack(b.z, a.z);
          v[j + 3] = pack(b.w, a.w);
        } else {
          v[j] = v[j + 1] = v[j + 2] = v[j + 3] = 0ull;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < E; ++j) {
        const int i = lane * E + j;
        v[j] = i < k ? pack(sr[i], ir[i]) : 0ull;
      }
    }
    warp_sort_desc<E>(v, lane);
    if (E >= 4 && vec) {
#pragma unroll
      for (int j = 0; j < E; j += 4) {
        const int i = lane * E + j;
        if (i < k) {
          int4 a;
          float4 b;
          unpack(v[j], &b.x, &a.x);
          unpack(v[j + 1], &b.y, &a.y);
          unpack(v[j + 2], &b.z, &a.z);
          unpack(v[j + 3], &b.w, &a.w);
          *reinterpret_cast<int4*>(ir + i) = a;
          *reinterpret_cast<float4*>(sr + i) = b;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < E; ++j) {
        const int i = lane * E + j;
        if (i < k) unpack(v[j], sr + i, ir + i);
      }
    }
  }
}

// Rows of 257..512 entries: two warps per row, 256 keys each in registers.
// Each warp sorts its half (the first descending, the second ascending, so
// the row is bitonic); the halves compare-exchange through shared memory for
// the stride-256 stage; each warp then finishes its half with a descending
// merge.  Twice the warps of the one-warp kernel at half the registers, so
// twice the latency hiding.
__global__ void __launch_bounds__(128) row_sort_pair_kernel(int32_t* __restrict__ idx,
                                                            float* __restrict__ score,
                                                            long long rows, int k, int vec) {
  __shared__ uint64_t xbuf[2][2][256];  // [row slot of the block][half][position]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rs = warp >> 1, h = warp & 1;
  const uint32_t bar_id = 1u + static_cast<uint32_t>(rs);
  for (long long r = static_cast<long long>(blockIdx.x) * 2 + rs; r < rows;
       r += static_cast<long long>(gridDim.x) * 2) {
    int32_t* ir = idx + r * k;
    float* sr = score + r * k;
    const int p0 = h * 256 + lane * 8;
    uint64_t v[8];
    if (vec) {
#pragma unroll
      for (int j = 0; j < 8; j += 4) {
        const int i0 = p0 + j;
        if (i0 < k) {
          const int4 a = *reinterpret_cast<const int4*>(ir + i0);
          const float4 b = *reinterpret_cast<const float4*>(sr + i0);
          v[j] = pack(b.x, a.x);
          v[j + 1] = pack(b.y, a.y);
          v[j + 2] = pack(b.z, a.z);
          v[j + 3] = pack(b.w, a.w);
        } else {
          v[j] = v[j + 1] = v[j + 2] = v[j + 3] = 0ull;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = p0 + j < k ? pack(sr[p0 + j], ir[p0 + j]) : 0ull;
    }
    warp_sort<8>(v, lane, h == 0);
#pragma unroll
    for (int j = 0; j < 8; ++j) xbuf[rs][h][lane * 8 + j] = v[j];
    asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint64_t o = xbuf[rs][h ^ 1][lane * 8 + j];
      v[j] = h == 0 ? (o > v[j] ? o : v[j]) : (o < v[j] ? o : v[j]);
    }
    asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");  // xbuf is free for the next row
    warp_merge<8>(v, lane, true);
    if (vec) {
#pragma unroll
      for (int j = 0; j < 8; j += 4) {
        const int i0 = p0 + j;
        if (i0 < k) {
          int4 a;
          float4 b;
          unpack(v[j], &b.x, &a.x);
          unpack(v[j + 1], &b.y, &a.y);
          unpack(v[j + 2], &b.z, &a.z);
          unpack(v[j + 3], &b.w, &a.w);
          *reinterpret_cast<int4*>(ir + i0) = a;
          *reinterpret_cast<float4*>(sr + i0) = b;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (p0 + j < k) unpack(v[j], sr + p0 + j, ir + p0 + j);
    }
  }
}

template <int E>
si_status launch_warp_sort(int32_t* idx, float* score, long long rows, int k, int n_sm, int vec,
                           cudaStream_t stream) {
  const long long blocks = (rows + 3) / 4;  // 4 warps (rows) per block
  const long long grid = std::min<long long>(blocks, static_cast<long long>(n_sm) * 16);
  row_sort_warp_kernel<E><<<static_cast<unsigned>(grid), 128, 0, stream>>>(idx, score, rows, k, vec);
  return SI_OK;
}

}  // namespace

si_status launch_row_sort(int32_t* idx, float* score, long long rows, int k, cudaStream_t stream) {
  if (rows <= 0) return SI_OK;
  int np = 64;
  while (np < k) np <<= 1;
  // one thread per compare-exchange pair, whole warps, at most 256
  const int threads = std::min(256, np >> 1);
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  const int vec = (k % 4 == 0) && (reinterpret_cast<uintptr_t>(idx) % 16 == 0) &&
                  (reinterpret_cast<uintptr_t>(score) % 16 == 0);
  switch (np) {
    case 64: launch_warp_sort<2>(idx, score, rows, k, n_sm, vec, stream); break;
    case 128: launch_warp_sort<4>(idx, score, rows, k, n_sm, vec, stream); break;
    case 256: launch_warp_sort<8>(idx, score, rows, k, n_sm, vec, stream); break;
    case 512: {
      const long long blocks = (rows + 1) / 2;  // 2 rows (4 warps) per block
      const long long grid = std::min<long long>(blocks, static_cast<long long>(n_sm) * 16);
      row_sort_pair_kernel<<<static_cast<unsigned>(grid), 128, 0, stream>>>(idx, score, rows, k, vec);
      break;
    }
    default: {  // 1024, 2048: too many keys for one warp's registers
      const long long grid = std::min<long long>(rows, static_cast<long long>(n_sm) * 16);
      const size_t smem = static_cast<size_t>(np) * sizeof(uint64_t);
      row_sort_kernel<<<static_cast<unsigned>(grid), threads, smem, stream>>>(idx, score, rows, k, np);
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "row_sort_kernel launch");
  return SI_OK;
}

}  // namespace si
