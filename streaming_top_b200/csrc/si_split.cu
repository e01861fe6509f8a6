// Merge of split-key partial top-ks.
//
// When a call has too few query rows to give every SM a 4-query unit (a row
// range deep into a long sequence, a decode-shaped call), the streaming
// kernel splits each unit's keys into n_split contiguous partitions, one per
// CTA, and each partition's managers store the exact top-k of their keys in
// partition order: parts [row][n_split][k] of (index, score), -1 / -inf
// padded.  StreamIndex's partition-merge (the skills page, "Core Technique"
// and "Implementation Steps": per-partition local top-k, then a merge) makes
// the result exact: the top-k of the union of the partitions is the top-k of
// the union of their top-ks.  This kernel is that merge: one CTA per row
// selects the k best of the row's n_split * k candidates by an MSD radix
// select on packed keys (in shared memory after a bound from the partitions'
// own k-th bests has discarded most of them), then sorts the k winners in
// shared memory (score descending, index ascending) and stores them, padded
// when fewer than k keys are visible.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"

namespace si {
namespace {

constexpr int M_THREADS = 512;
constexpr int M_WARPS = M_THREADS / 32;

// (orderable score << 32) | ~index: unsigned order = score descending, then
// index ascending; padding packs to 0 so that it ranks below every entry.
__device__ __forceinline__ uint64_t pack_entry(float sc, int32_t id) {
  if (id < 0) return 0ull;
  uint32_t u = __float_as_uint(sc);
  if (u == 0x80000000u) u = 0u;
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(o) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(id));
}

__device__ __forceinline__ void unpack_entry(uint64_t key, float* sc, int32_t* id) {
  const uint32_t o = static_cast<uint32_t>(key >> 32);
  *id = static_cast<int32_t>(~static_cast<uint32_t>(key));
  *sc = __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// MSD radix select over `n` distinct packed keys, read through `key_at(i)`
// (0 = no key): leaves in *prefix / *mask the high bits of the `need`-th
// largest key such that exactly `need` keys x satisfy (x & mask) >= prefix.
// hist: [M_WARPS][256], tot: [256].  All threads of the block.
template <typename KeyAt>
__device__ void radix_select(KeyAt key_at, int n, uint32_t need, uint32_t* hist, uint32_t* tot,
                             uint64_t* s_prefix, uint64_t* s_mask, uint32_t* s_need, uint32_t* s_done,
                             int* s_hi) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t vor = 0, vand = ~0ull;
  for (int i = tid; i < n; i += M_THREADS) {
    const uint64_t x = key_at(i);
    if (x) {
      vor |= x;
      vand &= x;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    vor |= __shfl_xor_sync(0xFFFFFFFFu, vor, o);
    vand &= __shfl_xor_sync(0xFFFFFFFFu, vand, o);
  }
  if (tid == 0) {
    *s_prefix = 0;        // reused as the OR, then the prefix
    *s_mask = ~0ull;      // reused as the AND, then the mask
  }
  __syncthreads();
  if (lane == 0) {
    atomicOr(reinterpret_cast<unsigned long long*>(s_prefix), vor);
    atomicAnd(reinterpret_cast<unsigned long long*>(s_mask), vand);
  }
  __syncthreads();
  if (tid == 0) {
    const uint64_t o = *s_prefix, a = *s_mask, diff = o ^ a;
    const int hb = diff ? 63 - __clzll(static_cast<long long>(diff)) : 0;
    *s_mask = hb == 63 ? 0ull : (~0ull << (hb + 1));
    *s_prefix = a & *s_mask;
    *s_need = need;
    *s_done = 0;
    *s_hi = hb + 1;  // the first digit is bits [hb-7, hb]
  }
  __syncthreads();
  int hi = *s_hi;
  while (!*s_done) {
    const int lo = hi > 8 ? hi - 8 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    for (int i = tid; i < M_WARPS * 256; i += M_THREADS) hist[i] = 0;
    __syncthreads();
    const uint64_t prefix = *s_prefix, mask = *s_mask;
    for (int i0 = 0; i0 < n; i0 += M_THREADS) {
      const int i = i0 + tid;
      const uint64_t x = i < n ? key_at(i) : 0ull;
      const bool in = x != 0ull && (x & mask) == prefix;
      const uint32_t d = in ? static_cast<uint32_t>(x >> lo) & dmask : 256u;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, d);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[warp * 256 + d], __popc(peers));
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t c = 0;
      for (int w = 0; w < M_WARPS; ++w) c += hist[w * 256 + tid];
      tot[tid] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l: find the bin where the count
      // from the top reaches `need`
      uint32_t v[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        v[e] = tot[255 - 8 * lane - e];
        sum += v[e];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t nd = *s_need, excl = incl - sum;
      if (excl < nd && nd <= incl) {
        uint32_t run = excl;
        for (int e = 0; e < 8; ++e) {
          if (run + v[e] >= nd) {
            const uint32_t d = 255u - 8u * lane - e;
            *s_prefix = prefix | (static_cast<uint64_t>(d) << lo);
            *s_mask = mask | (static_cast<uint64_t>(dmask) << lo);
            *s_need = nd - run;
            // the boundary digit taken whole, or every bit decided (keys are distinct)
            *s_done = (v[e] == nd - run || lo == 0) ? 1u : 0u;
            break;
          }
          run += v[e];
        }
      }
    }
    __syncthreads();
    hi = lo;
  }
}

// Per row: the k best of the row's n_split * k partial entries.
//  1. Every partition that holds k entries bounds the row's k-th best from
//     below by its own k-th best (its smallest): L = the largest of those.
//  2. The keys >= L (at least k of them) are gathered into shared memory
//     when they fit (the usual case); the radix select then runs there.
//     Otherwise it reads the partials from global memory (L2) each pass.
//  3. The winners are sorted descending in shared memory and stored.
// smem: hist [M_WARPS][256], tot [256], win [np], pool [cap]
__global__ void __launch_bounds__(M_THREADS) merge_splits_kernel(const int32_t* __restrict__ part_idx,
                                                                 const float* __restrict__ part_score, int rows,
                                                                 int n_split, int k, int np, int cap,
                                                                 int32_t* out_idx, float* out_score) {
  extern __shared__ __align__(16) uint8_t s_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(s_raw);
  uint32_t* tot = hist + M_WARPS * 256;
  uint64_t* win = reinterpret_cast<uint64_t*>(tot + 256);
  uint64_t* pool = win + np;
  __shared__ uint64_t s_prefix, s_mask, s_bound;
  __shared__ uint32_t s_need, s_done, s_real, s_cnt, s_out;
  __shared__ int s_hi;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = n_split * k;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    const int32_t* pi = part_idx + static_cast<size_t>(r) * n;
    const float* ps = part_score + static_cast<size_t>(r) * n;
    if (tid == 0) {
      s_bound = 0;
      s_real = 0;
      s_cnt = 0;
      s_out = 0;
    }
    __syncthreads();
    // 1. one warp per partition: its smallest real key, when it holds k
    for (int sp = warp; sp < n_split; sp += M_WARPS) {
      uint64_t mn = ~0ull;
      uint32_t real = 0;
#pragma unroll 4
      for (int i = lane; i < k; i += 32) {
        const uint64_t x = pack_entry(ps[sp * k + i], pi[sp * k + i]);
        if (x) {
          mn = x < mn ? x : mn;
          ++real;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
        mn = y < mn ? y : mn;
        real += __shfl_xor_sync(0xFFFFFFFFu, real, o);
      }
      if (lane == 0) {
        atomicAdd(&s_real, real);
        if (real == static_cast<uint32_t>(k)) atomicMax(reinterpret_cast<unsigned long long*>(&s_bound), mn);
      }
    }
    __syncthreads();
    const uint32_t total = s_real;
    const uint32_t take = total < static_cast<uint32_t>(k) ? total : static_cast<uint32_t>(k);
    const uint64_t bound = s_bound;
    // 2. the keys >= L into shared memory, while they fit
#pragma unroll 4
    for (int i = tid; i < n; i += M_THREADS) {
      const uint64_t x = pack_entry(ps[i], pi[i]);
      if (x && x >= bound) {
        const uint32_t at = atomicAdd(&s_cnt, 1u);
        if (at < static_cast<uint32_t>(cap)) pool[at] = x;
      }
    }
    __syncthreads();
    const uint32_t cnt = s_cnt;
    const bool in_smem = cnt <= static_cast<uint32_t>(cap);
    bool all = total <= static_cast<uint32_t>(k);
    uint64_t prefix = 0, mask = 0;
    if (!all) {
      if (in_smem) {
        if (cnt <= static_cast<uint32_t>(k)) {
          all = true;  // exactly the k keys >= L
        } else {
          radix_select([&](int i) { return pool[i]; }, static_cast<int>(cnt), take, hist, tot, &s_prefix, &s_mask,
                       &s_need, &s_done, &s_hi);
        }
      } else {
        radix_select([&](int i) { return pack_entry(ps[i], pi[i]); }, n, take, hist, tot, &s_prefix, &s_mask,
                     &s_need, &s_done, &s_hi);
      }
      prefix = s_prefix;
      mask = s_mask;
    }
    // the winners: (x & mask) >= prefix selects exactly `take` keys
    for (int i = tid; i < np; i += M_THREADS) win[i] = 0ull;
    __syncthreads();
    if (in_smem) {
      for (int i = tid; i < static_cast<int>(cnt); i += M_THREADS) {
        const uint64_t x = pool[i];
        if (all || (x & mask) >= prefix) win[atomicAdd(&s_out, 1u)] = x;
      }
    } else {
      for (int i = tid; i < n; i += M_THREADS) {
        const uint64_t x = pack_entry(ps[i], pi[i]);
        if (x && (all || (x & mask) >= prefix)) win[atomicAdd(&s_out, 1u)] = x;
      }
    }
    __syncthreads();
    // 3. sort the winners descending (bitonic, in shared memory)
    for (int size = 2; size <= np; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < (np >> 1); i += M_THREADS) {
          const int a = 2 * i - (i & (stride - 1)), b = a + stride;
          const bool desc = (a & size) == 0;
          const uint64_t x = win[a], y = win[b];
          if ((x < y) == desc) {
            win[a] = y;
            win[b] = x;
          }
        }
        __syncthreads();
      }
    }
    int32_t* oi = out_idx + static_cast<size_t>(r) * k;
    float* os = out_score ? out_score + static_cast<size_t>(r) * k : nullptr;
    for (int i = tid; i < k; i += M_THREADS) {
      int32_t id = -1;
      float sc = -__int_as_float(0x7f800000);
      if (static_cast<uint32_t>(i) < take) unpack_entry(win[i], &sc, &id);
      oi[i] = id;
      if (os) os[i] = sc;
    }
    __syncthreads();
  }
}

}  // namespace

si_status launch_merge_splits(const int32_t* part_idx, const float* part_score, long long rows, int n_split, int k,
                              int32_t* out_idx, float* out_score, cudaStream_t stream) {
  if (rows <= 0) return SI_OK;
  int np = 32;
  while (np < k) np <<= 1;
  constexpr int kPoolKeys = 16384;  // candidates >= the partitions' bound kept in shared memory
  const size_t smem = static_cast<size_t>(M_WARPS) * 256 * 4 + 256 * 4 + (static_cast<size_t>(np) + kPoolKeys) * 8;
  cudaError_t e = cudaFuncSetAttribute(merge_splits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(merge_splits_kernel)");
  const unsigned grid = static_cast<unsigned>(std::min<long long>(rows, 65535));
  merge_splits_kernel<<<grid, M_THREADS, smem, stream>>>(part_idx, part_score, static_cast<int>(rows), n_split, k,
                                                         np, kPoolKeys, out_idx, out_score);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "merge_splits_kernel launch");
  return SI_OK;
}

}  // namespace si
