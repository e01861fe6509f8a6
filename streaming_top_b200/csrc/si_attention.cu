// Sparse attention over the indexer's selected compressed latents (the
// consumer of the top-k).
//
// StreamIndex (abstract): the sparse attention kernel reads only the entries
// the indexer selected.  Reading of the pages (DeepSeek-V3.2 lineage that the
// V4.1 page gives): every one of the H = 64 heads of query t attends over the
// k selected compressed latents of its sequence; a latent is the key (all
// Dk = 576 values: 512 latent + 64 rope) and the value (its first Dv = 512);
// the softmax runs over the selection only with scale 1/sqrt(Dk) (or the
// caller's); index -1 is padding; a row with nothing selected gives O = 0 and
// lse = -inf.
//
// One CTA per SM, persistent over queries.  Per query:
//   QK   S^T[e, h] = sum_d kv[sel[e], d] * q[h, d]: tcgen05 kind::f16, A = 128
//        gathered latent rows (M = entries) x 64 dims per 16 KB stage, SW128
//        K-major; B = q[t] (N = 64 heads, K = 576) TMA-loaded once; fp32 into
//        TMEM columns [64 j, 64 j + 64) for entry tile j.
//   softmax over the k entries per head (4 warps, lane = entry): (1) the max,
//        (2) tile by tile P = exp(scale (s - max)) rounded to bf16 and written
//        as P^T (N = heads, K = entries, SW128 K-major), each tile released to
//        the MMA warp by its own barrier, (3) the sums of the rounded P for the
//        normalisation and lse = scale max + ln sum.
//   PV   O^T[dv, h] = sum_e V[e, dv] P^T[h, e], chunk by chunk (64 entries, the
//        four 128-dv tiles): A = gathered value tiles read MN-major (dv is
//        contiguous in each latent row), B = P^T; fp32 into TMEM columns
//        [256 + 64 v, ...) for dv tile v.
//   out  O[t, h, dv] = O^T * (1 / sum_h), bf16; lse[t, h] fp32.
// Warps: 0 q loads (TMA), 1 MMA issue, 2-3 gather producers (each stage half
// by TMA gather4 from warp 2, half by 16-byte cp.async from warp 3: the two
// copy paths' rates add up), 4-7 softmax and epilogue.  Every wait is bounded;
// on expiry the kernel records SI_ERR_TIMEOUT, drains its copies and MMAs and
// exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"
#include "si_ptx.cuh"

namespace si {
namespace {

constexpr int A_H = 64, A_DK = 576, A_DV = 512, A_KMAX = 512;
constexpr int A_KB = A_DK / 64;             // 9 K-blocks of 64 dims
constexpr int A_THREADS = 256;
constexpr int A_NS = 4;                     // gather stages of 16 KB
constexpr int A_STAGE = 16384;
constexpr int A_Q_BYTES = A_H * A_DK * 2;   // 72 KB: 9 blocks of [64 rows x 128 B]
constexpr int A_P_BYTES = A_H * A_KMAX * 2; // 64 KB: up to 8 blocks of [64 heads x 128 B]

enum { AERR_Q_FREE = 21, AERR_Q_FULL = 22, AERR_STAGE_FREE = 23, AERR_STAGE_FULL = 24, AERR_S_FULL = 25,
       AERR_P_FULL = 26, AERR_O_FULL = 27, AERR_O_FREE = 28, AERR_DRAIN = 29 };

struct AttnParams {
  const uint8_t* kv;      // [B, T, 576] bf16 bytes
  const int32_t* idx;     // [B, S, k]
  __nv_bfloat16* out;     // [B, S, 64, 512]
  float* lse;             // [B, S, 64]
  int* err;
  int B, S, T, k;
  float scale;
  uint64_t wait_limit_ns;
};

struct ACtrl {
  uint64_t full[A_NS], empty[A_NS];
  uint64_t q_full, q_empty, s_full, o_full, o_empty, done;
  uint64_t p_full[4];     // per 128-entry tile: its rounded weights are in P^T
  uint32_t tmem_slot;
  int abort;
  float red[4][A_H];      // per-quadrant partial max / sum
  alignas(16) float head_max[A_H];  // per head: max logit (read as float4)
  float head_inv[A_H];              // per head: 1 / sum of the rounded weights
  alignas(16) int sel[2][A_KMAX];  // each producer warp's copy of the current query's selection: latent rows
};

// 16-byte global -> shared copy (L2 only).
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// The barrier receives one arrival when every cp.async this thread has issued
// so far has landed (its expected count includes that arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// TMA gather of four rows r0..r3 of a 2-D tensor map (box: 64 elements x 1
// row), columns x .. x+63, into four consecutive 128-byte rows at dst
// (swizzled by the map), completing `bytes` on the mbarrier.  No multicast.
__device__ __forceinline__ void tma_gather4(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t r0,
                                            int32_t r1, int32_t r2, int32_t r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// atoms of 8 K-rows x 128 bytes (64 bf16 along M/N); `lbo` = bytes between
// atoms along M/N, `sbo` = bytes between 8-row groups along K (the canonical
// MN-major layout of the tcgen05 matrix descriptor, version 1).
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ void attn_error(const AttnParams& p, volatile int* abort, int where) {
  atomicCAS(p.err, 0, static_cast<int>(SI_ERR_TIMEOUT));
  atomicCAS(p.err + 1, 0, where);
  *abort = 1;
}

__global__ void __launch_bounds__(A_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                       const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem;
  uint8_t* st_s = smem + A_Q_BYTES;
  uint8_t* p_s = st_s + A_NS * A_STAGE;
  ACtrl* C = reinterpret_cast<ACtrl*>(p_s + A_P_BYTES);
  volatile int* abort = &C->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_et = p.k / 128;            // entry tiles of the QK product
  const int n_kc = p.k / 64;             // 64-entry chunks of the PV product
  const int qk_stages = n_et * A_KB, pv_stages = 4 * n_kc;
  if (threadIdx.x == 0) {
    for (int s = 0; s < A_NS; ++s) {
      mbar_init(&C->full[s], 33);  // warp 2's expect-tx arrival + one noinc arrival per lane of warp 3
      mbar_init(&C->empty[s], 1);
    }
    mbar_init(&C->q_full, 1);
    mbar_init(&C->q_empty, 1);
    mbar_init(&C->s_full, 1);
    for (int j = 0; j < 4; ++j) mbar_init(&C->p_full[j], 128);
    mbar_init(&C->o_full, 1);
    mbar_init(&C->o_empty, 128);
    mbar_init(&C->done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kv);
  }
  if (warp == 1) tmem_alloc(&C->tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C->tmem_slot;
  const int nq = p.B * p.S;               // queries, sequence-major
  const int q0 = blockIdx.x, qstep = gridDim.x;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ q rows (TMA)
      uint32_t n = 0;
      for (int t = q0; t < nq; t += qstep, ++n) {
        if (!mbar_wait_bounded(&C->q_empty, (n & 1u) ^ 1u, abort, p.wait_limit_ns)) {
          attn_error(p, abort, AERR_Q_FREE);
          break;
        }
        mbar_arrive_expect_tx(&C->q_full, A_Q_BYTES);
        for (int kb = 0; kb < A_KB; ++kb) tma_load_2d(q_s + kb * 8192, &tm_q, &C->q_full, kb * 64, t * A_H);
      }
      if (n && !mbar_wait_timed(&C->q_full, (n - 1) & 1u, p.wait_limit_ns)) attn_error(p, abort, AERR_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC_QK = idesc_f32acc(1, 1, 128, A_H);
      constexpr uint32_t IDESC_PV = idesc_f32acc(1, 1, 128, A_H) | (1u << 15);  // A (V^T) MN-major
      const uint32_t qa = smem_u32(q_s), sa = smem_u32(st_s), pa = smem_u32(p_s);
      uint32_t stage = 0, phase = 0, n = 0;
      bool stop = false;
      for (int t = q0; t < nq && !stop; t += qstep, ++n) {
        const uint32_t par = n & 1u;
        if (!mbar_wait_bounded(&C->q_full, par, abort, p.wait_limit_ns)) {
          attn_error(p, abort, AERR_Q_FULL);
          break;
        }
        tc_fence_after();
        for (int jt = 0; jt < n_et && !stop; ++jt)
          for (int kb = 0; kb < A_KB; ++kb) {
            if (!mbar_wait_bounded(&C->full[stage], phase, abort, p.wait_limit_ns)) {
              attn_error(p, abort, AERR_STAGE_FULL);
              stop = true;
              break;
            }
            tc_fence_after();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // cp.async data -> MMA operand
            const uint32_t a0 = sa + stage * A_STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(tmem + jt * A_H, sdesc_kmajor_sw128(a0 + kk * 32), sdesc_kmajor_sw128(qa + kb * 8192 + kk * 32),
                       IDESC_QK, (kb | kk) != 0);
            mma_commit(&C->empty[stage]);
            if (++stage == A_NS) {
              stage = 0;
              phase ^= 1u;
            }
          }
        if (stop) break;
        mma_commit(&C->s_full);
        mma_commit(&C->q_empty);
        if (!mbar_wait_bounded(&C->o_empty, par ^ 1u, abort, p.wait_limit_ns)) {
          attn_error(p, abort, AERR_O_FREE);
          break;
        }
        // PV chunk by chunk (64 entries, the four dv tiles each): a tile's two
        // chunks start as soon as the softmax warps have written its weights
        for (int c = 0; c < n_kc && !stop; ++c) {
          if ((c & 1) == 0 && !mbar_wait_bounded(&C->p_full[c >> 1], par, abort, p.wait_limit_ns)) {
            attn_error(p, abort, AERR_P_FULL);
            stop = true;
            break;
          }
          tc_fence_after();
          for (int vt = 0; vt < 4; ++vt) {
            if (!mbar_wait_bounded(&C->full[stage], phase, abort, p.wait_limit_ns)) {
              attn_error(p, abort, AERR_STAGE_FULL);
              stop = true;
              break;
            }
            tc_fence_after();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // cp.async data -> MMA operand
            const uint32_t a0 = sa + stage * A_STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // 16 entries a step: two 8-entry atom rows
              mma_bf16(tmem + 256 + vt * A_H, sdesc_mnmajor_sw128(a0 + kk * 2048, 8192, 1024),
                       sdesc_kmajor_sw128(pa + c * 8192 + kk * 32), IDESC_PV, (c | kk) != 0);
            mma_commit(&C->empty[stage]);
            if (++stage == A_NS) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!stop) mma_commit(&C->o_full);
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(&C->done);
      if (!mbar_wait_timed(&C->done, 0, p.wait_limit_ns)) attn_error(p, abort, AERR_DRAIN);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ gather producers
    // Two copy paths fill each 16 KB stage side by side: warp 2 through the
    // TMA unit (one gather4 of 4 latent rows x 128 B per lane, 16 lanes: half
    // the stage), warp 3 through the load/store path (16-byte cp.async, eight
    // lanes to a row: the other half).  The rows land in the 128-byte-swizzled
    // layout the MMA reads.  Each warp keeps its own copy of the selection, so
    // the two never wait for each other.  The stage's barrier takes warp 2's
    // expect-tx arrival and one noinc arrival per lane of warp 3.
    const bool tma = warp == 2;
    int* sel = C->sel[warp - 2];
    uint32_t stage = 0, phase = 0;
    uint32_t any_load = 0, last_par = 0;  // warp 2, per stage: loaded at all / parity of the last load
    bool stop = false;
    // the selection of the warp's next query, loaded while the current one's
    // stages are issued
    int nxt[A_KMAX / 32];
#pragma unroll
    for (int i = 0; i < A_KMAX / 32; ++i)
      nxt[i] = q0 < nq && 32 * i < p.k ? p.idx[static_cast<size_t>(q0) * p.k + 32 * i + lane] : 0;
    for (int t = q0; t < nq && !stop; t += qstep) {
      const int row_base = (t / p.S) * p.T;  // the sequence's first latent row
      __syncwarp();                          // the warp's copies of the last query have read sel
#pragma unroll
      for (int i = 0; i < A_KMAX / 32; ++i)
        if (32 * i < p.k) {
          const int key = nxt[i];
          sel[32 * i + lane] = row_base + (key >= 0 && key < p.T ? key : 0);  // padding reads row 0; weight 0
        }
      __syncwarp();
      const int tn = t + qstep;
#pragma unroll
      for (int i = 0; i < A_KMAX / 32; ++i)
        nxt[i] = tn < nq && 32 * i < p.k ? p.idx[static_cast<size_t>(tn) * p.k + 32 * i + lane] : 0;
      for (int j = 0; j < qk_stages + pv_stages; ++j) {
        bool got = true;
        if (lane == 0) {
          got = mbar_wait_bounded(&C->empty[stage], phase ^ 1u, abort, p.wait_limit_ns);
          if (!got)
            attn_error(p, abort, AERR_STAGE_FREE);
          else if (tma)
            mbar_arrive_expect_tx(&C->full[stage], A_STAGE / 2);
        }
        if (__shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) == 0) {
          stop = true;
          break;
        }
        __syncwarp();
        uint8_t* dst = st_s + stage * A_STAGE;
        // QK stage (entry tile j / 9, K-block j % 9): 128 rows x 128 B; TMA rows
        // 0-63, cp.async rows 64-127.  PV stage (64-entry chunk jj / 4, dv tile
        // jj % 4): two atoms (64 dv each) of 64 rows x 128 B; TMA atom 0,
        // cp.async atom 1.
        const bool qk = j < qk_stages;
        const int jj = j - qk_stages;
        const int e0 = qk ? (j / A_KB) * 128 : (jj >> 2) * 64;
        const int x = qk ? (j % A_KB) * 64 : (jj & 3) * 128;
        if (tma) {
          if (lane < 16) {
            const int4 r = *reinterpret_cast<const int4*>(&sel[e0 + 4 * lane]);
            tma_gather4(dst + lane * 512, &tm_kv, &C->full[stage], x, r.x, r.y, r.z, r.w);
          }
          any_load |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        } else {
          const uint32_t base = smem_u32(dst) + 8192u;  // rows 64-127 of a QK stage, atom 1 of a PV stage
          const int ro = qk ? 64 : 0, xo = qk ? x : x + 64;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int id = lane + 32 * i, row = id >> 3, ch = id & 7;
            cp16(base + row * 128 + ((ch ^ (row & 7)) << 4),
                 p.kv + static_cast<size_t>(sel[e0 + ro + row]) * (A_DK * 2) + xo * 2 + ch * 16);
          }
          cp_async_arrive_noinc(&C->full[stage]);
        }
        if (++stage == A_NS) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // every copy issued has landed before the CTA can exit
    if (tma) {
      if (lane == 0)
        for (int s = 0; s < A_NS; ++s)
          if (((any_load >> s) & 1u) && !mbar_wait_timed(&C->full[s], (last_par >> s) & 1u, p.wait_limit_ns))
            attn_error(p, abort, AERR_DRAIN);
    } else {
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    // The four warps meet at named barriers, so none may leave the loop early:
    // after a failed wait a warp keeps going through every barrier with ok =
    // false and touches neither TMEM nor the outputs.
    const int quad = warp - 4;
    const float ninf = -__int_as_float(0x7f800000);
    uint32_t n = 0;
    bool ok = true;
    for (int t = q0; t < nq; t += qstep, ++n) {
      const uint32_t par = n & 1u;
      uint32_t vmask = 0;  // bit jt: this thread's entry of tile jt is a real key
#pragma unroll
      for (int jt = 0; jt < 4; ++jt) {
        if (jt >= n_et) break;
        const int key = p.idx[static_cast<size_t>(t) * p.k + jt * 128 + quad * 32 + lane];
        vmask |= (key >= 0 && key < p.T ? 1u : 0u) << jt;
      }
      const bool got = ok && mbar_wait_bounded(&C->s_full, par, abort, p.wait_limit_ns);
      if (ok && !__all_sync(0xFFFFFFFFu, got)) {
        if (lane == 0) attn_error(p, abort, AERR_S_FULL);
        ok = false;
      }
      tc_fence_after();
      // 1. per-head maximum over the valid entries, in two halves of 32 heads
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float m[32];
        uint32_t x[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) m[h] = ninf;
#pragma unroll 1
        for (int jt = 0; jt < n_et && ok; ++jt) {
          tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + jt * A_H + hh * 32, x);
          tmem_ld_wait();
          if ((vmask >> jt) & 1u) {
#pragma unroll
            for (int h = 0; h < 32; ++h) m[h] = fmaxf(m[h], __uint_as_float(x[h]));
          }
        }
#pragma unroll
        for (int h = 0; h < 32; ++h)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m[h] = fmaxf(m[h], __shfl_xor_sync(0xFFFFFFFFu, m[h], o));
        float mine = 0.f;  // m[lane] without a dynamic register index
#pragma unroll
        for (int h = 0; h < 32; ++h) mine = h == lane ? m[h] : mine;
        C->red[quad][hh * 32 + lane] = mine;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (quad == 0)
        for (int hg = lane; hg < A_H; hg += 32)
          C->head_max[hg] = fmaxf(fmaxf(C->red[0][hg], C->red[1][hg]), fmaxf(C->red[2][hg], C->red[3][hg]));
      asm volatile("bar.sync 1, 128;" ::: "memory");  // head_max is complete; red is free
      // 2. tile by tile, the rounded weights of all heads into P^T; each tile's
      //    barrier lets the MMA warp start that tile's PV while the next is done
      float sum[A_H];
#pragma unroll
      for (int h = 0; h < A_H; ++h) sum[h] = 0.f;
#pragma unroll 1
      for (int jt = 0; jt < n_et; ++jt) {
        if (ok) {
          const int e = jt * 128 + quad * 32 + lane, kb = e >> 6, col = e & 63;
          const bool valid = (vmask >> jt) & 1u;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t x[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + jt * A_H + hh * 32, x);
            tmem_ld_wait();
#pragma unroll
            for (int h4 = 0; h4 < 32; h4 += 4) {
              const float4 mx = *reinterpret_cast<const float4*>(&C->head_max[hh * 32 + h4]);
              const float mv[4] = {mx.x, mx.y, mx.z, mx.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int h = h4 + u, hg = hh * 32 + h;
                const float pr = valid ? __expf(p.scale * (__uint_as_float(x[h]) - mv[u])) : 0.f;
                const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
                sum[hg] += __bfloat162float(pb);
                // P^T K-major: block kb = [64 heads][64 entries], row hg, swizzled 16-byte chunk
                const int off = kb * 8192 + hg * 128 + ((((col * 2) >> 4) ^ (hg & 7)) << 4) + ((col * 2) & 15);
                *reinterpret_cast<__nv_bfloat16*>(p_s + off) = pb;
              }
            }
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P is read by the MMA (async proxy)
        tc_fence_before();
        mbar_arrive(&C->p_full[jt]);
      }
      // 3. per-head sums of the rounded weights -> 1 / sum and the log-sum-exp
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float v[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) v[h] = sum[hh * 32 + h];
#pragma unroll
        for (int h = 0; h < 32; ++h)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v[h] += __shfl_xor_sync(0xFFFFFFFFu, v[h], o);
        float mine = 0.f;
#pragma unroll
        for (int h = 0; h < 32; ++h) mine = h == lane ? v[h] : mine;
        C->red[quad][hh * 32 + lane] = mine;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (quad == 0)
        for (int hg = lane; hg < A_H; hg += 32) {
          const float s = C->red[0][hg] + C->red[1][hg] + C->red[2][hg] + C->red[3][hg];
          C->head_inv[hg] = s > 0.f ? 1.0f / s : 0.f;
          if (ok) p.lse[static_cast<size_t>(t) * A_H + hg] = s > 0.f ? p.scale * C->head_max[hg] + __logf(s) : ninf;
        }
      asm volatile("bar.sync 1, 128;" ::: "memory");  // head_inv is complete
      // epilogue: lane = dv, 64 heads a load
      const bool gotO = ok && mbar_wait_bounded(&C->o_full, par, abort, p.wait_limit_ns);
      if (ok && !__all_sync(0xFFFFFFFFu, gotO)) {
        if (lane == 0) attn_error(p, abort, AERR_O_FULL);
        ok = false;
      }
      tc_fence_after();
      uint32_t x[64];
      for (int vt = 0; vt < 4 && ok; ++vt) {
        tmem_ld32_x64(tmem + (static_cast<uint32_t>(quad * 32) << 16) + 256 + vt * A_H, x);
        tmem_ld_wait();
        const int dv = vt * 128 + quad * 32 + lane;
#pragma unroll
        for (int h = 0; h < A_H; ++h)
          p.out[(static_cast<size_t>(t) * A_H + h) * A_DV + dv] =
              __float2bfloat16_rn(__uint_as_float(x[h]) * C->head_inv[h]);
      }
      tc_fence_before();
      mbar_arrive(&C->o_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

si_status launch_sparse_attention(const void* q, const void* kv, const int32_t* idx, int B, int S, int T, int k,
                                  float scale, void* out, float* lse, int* err, uint64_t wait_limit_ns,
                                  cudaStream_t stream) {
  CUtensorMap tm_q, tm_kv;
  si_status st = encode_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, A_DK,
                                static_cast<uint64_t>(B) * S * A_H, A_DK * 2, 64, A_H);
  if (st != SI_OK) return st;
  // the latents as [B*T rows, 576]: gather4 takes a box one row high
  st = encode_tmap_2d(&tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kv, A_DK, static_cast<uint64_t>(B) * T, A_DK * 2, 64,
                      1);
  if (st != SI_OK) return st;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const size_t smem = 1024 + A_Q_BYTES + A_NS * A_STAGE + A_P_BYTES + sizeof(ACtrl);
  e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(sparse_attn_kernel)");
  AttnParams p;
  p.kv = static_cast<const uint8_t*>(kv);
  p.idx = idx;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = err;
  p.B = B;
  p.S = S;
  p.T = T;
  p.k = k;
  p.scale = scale;
  p.wait_limit_ns = wait_limit_ns;
  const long long nq = static_cast<long long>(B) * S;
  const int grid = static_cast<int>(std::min<long long>(nq, n_sm));
  sparse_attn_kernel<<<grid, A_THREADS, smem, stream>>>(tm_q, tm_kv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sparse_attn_kernel launch");
  return SI_OK;
}

}  // namespace si
