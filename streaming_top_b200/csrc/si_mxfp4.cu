// MXFP4 indexer keys -> bf16.
//
// The V4.1-Flash deployment notes ("two-level sparse attention") store the
// indexer's own keys in MXFP4: OCP Microscaling FP4, E2M1 codes with one
// E8M0 power-of-two scale per 32 values.  The streaming kernel scores bf16
// keys on the kind::f16 tensor-core path, so a call with MXFP4 keys first
// decodes them here: B*T rows of D values, a few MB even at a million tokens
// (the keys are compressed m-fold and shared by every query), against the
// query side's S*H_I rows -- the decode is noise next to the scoring, and the
// hot loop stays on the bf16 path.  Every E2M1 value times 2^(e-127) with
// e <= 252 is exactly a bf16 value, so nothing is rounded.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"

namespace si {
namespace {

// bf16 bit patterns of the E2M1 magnitudes 0, 0.5, 1, 1.5 (low word) and
// 2, 3, 4, 6 (high word), four 16-bit fields each.
constexpr uint64_t kMagLo = 0x3FC03F803F000000ull;
constexpr uint64_t kMagHi = 0x40C0408040404000ull;

__device__ __forceinline__ float e2m1_magnitude(uint32_t c) {
  const uint64_t w = (c & 4u) ? kMagHi : kMagLo;
  const uint32_t bits = static_cast<uint32_t>(w >> ((c & 3u) * 16u)) & 0xFFFFu;
  return __uint_as_float(bits << 16);
}

// 2^(e-127) as fp32: a normal number for e >= 1, 2^-127 (subnormal) for e = 0,
// NaN for 255.
__device__ __forceinline__ float e8m0_value(uint32_t e) {
  if (e == 255u) return __uint_as_float(0x7FC00000u);
  return e == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// One thread per 32-value block: 16 bytes of codes and one scale in, 64
// bytes of bf16 out.
__global__ void __launch_bounds__(256) mxfp4_to_bf16_kernel(const uint4* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales,
                                                            uint4* __restrict__ out, long long n_blocks) {
  for (long long b = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; b < n_blocks;
       b += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 c = codes[b];
    const float sc = e8m0_value(scales[b]);
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      // 8 codes -> 8 bf16 values (one 16-byte store); code j sits in bits 4j..4j+3
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t c0 = (words[wi] >> (8 * j)) & 15u, c1 = (words[wi] >> (8 * j + 4)) & 15u;
        const __nv_bfloat162 v = __floats2bfloat162_rn(e2m1_magnitude(c0) * sc, e2m1_magnitude(c1) * sc);
        uint32_t bits = *reinterpret_cast<const uint32_t*>(&v);
        bits |= ((c0 & 8u) << 12) | ((c1 & 8u) << 28);  // the sign bits
        o[j] = bits;
      }
      out[b * 4 + wi] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace

si_status launch_mxfp4_to_bf16(const void* codes, const void* scales, long long rows, int D, void* out,
                               cudaStream_t stream) {
  const long long n_blocks = rows * (D / 32);
  if (n_blocks <= 0) return SI_OK;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  const long long grid = std::min<long long>((n_blocks + 255) / 256, static_cast<long long>(n_sm) * 8);
  mxfp4_to_bf16_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
      static_cast<const uint4*>(codes), static_cast<const uint8_t*>(scales), static_cast<uint4*>(out),
      n_blocks);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "mxfp4_to_bf16_kernel launch");
  return SI_OK;
}

}  // namespace si
