// Two-stage indexer top-k for sm_100a.
//
// The V4.1-Flash indexer as its deployment notes describe it ("two-level
// sparse attention", indexer section): a cheap candidate stage first picks,
// per query, blocks of compressed keys -- 2048 blocks of 8 -- and the best
// keys among the candidates are kept -- 512.  The pages do not say how a
// block is scored; the reading taken here: the mean of the block's keys,
// rounded once to bf16, is scored with the same indexer formula, only
// complete visible blocks compete, and the candidates are the kept blocks'
// keys plus the visible keys of the incomplete last block.
//
// Four steps, all on the device:
//   pool    : pooled keys [B, T/G, D] bf16 (double sums, one rounding).
//   coarse  : the streaming top-k kernel itself over the pooled keys with
//             compression m*G (block j is complete for query t iff
//             j*(m*G) + m*G - 1 <= t: the same visibility rule) and k = n_keep,
//             rows left unsorted -- a query's kept blocks.
//   fine    : this file's tcgen05 kernel.  A work unit is 2 queries; each
//             128-candidate tile (both queries, both 64-dim K halves, 64 KB, 3
//             stages) arrives in the 128-byte-swizzled K-major layout the MMA
//             reads: for block sizes divisible by 8 one 3-D TMA box per run of
//             8 key rows, by 4 four 2-D boxes, otherwise 16-byte cp.async.
//             One thread issues M = 128 keys x N = 64 heads MMAs per query
//             into a TMEM double buffer, and 8 scoring warps apply ReLU and
//             the head weights and store each candidate's packed key
//             (orderable score << 32 | ~index).
//   select  : the exact k largest packed keys per row: one pass over 2048
//             bins of the row's score range, a radix select (8-bit digits,
//             warp-aggregated shared-memory histograms) inside the boundary
//             bin; then the row sort orders them.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"
#include "si_ptx.cuh"

namespace si {
namespace {

constexpr int F_QT = 2;                  // queries per fine-stage unit
constexpr int F_HEADS = 64;
constexpr int F_DIM = 128;
constexpr int F_KT = 128;                // candidates per tile (MMA M)
constexpr int F_THREADS = 384;           // 12 warps
constexpr int F_STAGES = 3;              // candidate-tile stages of shared memory
constexpr int F_PRODUCERS = 64;          // cp.async path: warps 2, 3 fill every stage together
constexpr int F_Q_HALF = F_QT * F_HEADS * 128;        // 16 KB: one 64-column half of the q tile
constexpr int F_Q_BYTES = 2 * F_Q_HALF;               // 32 KB
// A stage holds one candidate tile of both queries, both K halves: query j's
// 128 rows in 16 groups of 8 (2 KB each), a group's half h at +1 KB, each a
// 1 KB 128-byte-swizzled atom of 8 rows x 64 dims.  The MMA reads a half as
// K-major rows with 2 KB between 8-row groups.
constexpr int F_GROUP = 2048;                         // 8 rows x 2 halves x 128 B
constexpr int F_A_QUERY = F_KT / 8 * F_GROUP;         // 32 KB: one query's tile
constexpr int F_STAGE_BYTES = F_QT * F_A_QUERY;       // 64 KB
constexpr int F_CTRL_BYTES = 256;
constexpr int F_SMEM = F_Q_BYTES + F_STAGES * F_STAGE_BYTES + F_CTRL_BYTES + 1024;

enum { FERR_Q = 21, FERR_FULL = 22, FERR_EMPTY = 23, FERR_TFULL = 24, FERR_TEMPTY = 25, FERR_QFREE = 26,
       FERR_DRAIN = 27 };

// ---------------------------------------------------------------- pool
// Pooled key j = bf16(round-to-nearest-even(mean of keys jG .. jG+G-1)): the
// G bf16 values are summed exactly in double, divided by G and rounded once.
__global__ void __launch_bounds__(128) pool_keys_kernel(const __nv_bfloat16* __restrict__ kc,
                                                        __nv_bfloat16* __restrict__ kp, int B, int T, int G,
                                                        int nb) {
  const long long n = static_cast<long long>(B) * nb * F_DIM;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int d = static_cast<int>(e % F_DIM);
    const long long bj = e / F_DIM;
    const int j = static_cast<int>(bj % nb), b = static_cast<int>(bj / nb);
    const __nv_bfloat16* src = kc + (static_cast<long long>(b) * T + static_cast<long long>(j) * G) * F_DIM + d;
    double s = 0.0;
    for (int i = 0; i < G; ++i) s += static_cast<double>(__bfloat162float(src[static_cast<long long>(i) * F_DIM]));
    kp[e] = __double2bfloat16(s / G);
  }
}

// ---------------------------------------------------------------- fine
struct FineParams {
  const uint8_t* kc;       // [T, D] bf16 of one sequence (bytes)
  const float* w;          // [R, H] of this chunk
  const int32_t* coarse;   // [R, n_keep] kept blocks, valid first, then -1
  uint64_t* packed;        // [R, ldp]
  int* err;
  int R, T, m, G, n_keep, ldp;
  int nb;                  // complete blocks of the sequence, T / G
  int g_shift;             // log2(G) when G is a power of two, else -1 (divide)
  long long row0;          // absolute position of chunk row 0
  int box_rows;            // 8 (3-D boxes) or 4 (2-D boxes): candidates arrive by TMA; 0: cp.async
  int box3d;               // 1 with box_rows 8: one 3-D box carries 8 rows, both K halves
  uint64_t wait_limit_ns;
};

struct Cand {
  int n_blk_keys;  // keys coming from kept blocks (kept blocks * G)
  int tail0;       // first key of the incomplete block
  int count;       // candidates
};

__device__ __forceinline__ Cand cand_of(const FineParams& p, int r) {
  Cand c;
  const long long t = p.row0 + r;
  long long n = (t + 1) / p.m;
  if (n > p.T) n = p.T;
  const int nbv = static_cast<int>(n / p.G);
  const int kept = nbv < p.n_keep ? nbv : p.n_keep;
  c.n_blk_keys = kept * p.G;
  c.tail0 = nbv * p.G;
  c.count = c.n_blk_keys + static_cast<int>(n - c.tail0);
  return c;
}

// Slot s's block within the kept list and its key within the block: shifts
// for a power-of-two block size (the per-slot hot path), else division.
__device__ __forceinline__ int blk_slot(const FineParams& p, int s) {
  return p.g_shift >= 0 ? s >> p.g_shift : s / p.G;
}
__device__ __forceinline__ int in_blk(const FineParams& p, int s) {
  return p.g_shift >= 0 ? s & (p.G - 1) : s % p.G;
}

// Key index of candidate slot `s` of row r, or -1 past the row's candidates
// (and for a kept-block entry outside [0, nb), which the coarse stage never
// writes: no address outside the keys is ever formed).
__device__ __forceinline__ int key_of(const FineParams& p, const Cand& c, int r, int s) {
  if (s < c.n_blk_keys) {
    const int blk = p.coarse[static_cast<long long>(r) * p.n_keep + blk_slot(p, s)];
    return blk >= 0 && blk < p.nb ? blk * p.G + in_blk(p, s) : -1;
  }
  if (s < c.count) return c.tail0 + (s - c.n_blk_keys);
  return -1;
}

__device__ __forceinline__ int f_unit_of(int i, int n_units) {
  const int Gd = gridDim.x, c = blockIdx.x;
  const long long base = static_cast<long long>(i) * Gd;
  if (base >= n_units) return -1;
  const long long u = base + ((i & 1) ? (Gd - 1 - c) : c);
  return u < n_units ? static_cast<int>(u) : -1;
}

__device__ __forceinline__ uint32_t f_ord(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void f_record(const FineParams& p, volatile int* abort, int where) {
  atomicCAS(p.err, 0, static_cast<int>(SI_ERR_TIMEOUT));
  atomicCAS(p.err + 1, 0, where);
  *abort = 1;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// The barrier receives one arrival when every cp.async this thread has issued
// so far has landed (its expected count includes that arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// 3-D TMA tile load (no multicast) at coordinates (x, y, z), completing its
// bytes on the mbarrier.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// K-major, 128-byte-swizzled operand descriptor with `sbo` bytes between
// 8-row groups (the layout fields as in sdesc_kmajor_sw128).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128_sbo(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

struct FCtrl {
  uint64_t full[F_STAGES], empty[F_STAGES];
  uint64_t q_full, q_empty;
  uint64_t t_full[2], t_empty[2];
  uint64_t mma_done;
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(FCtrl) <= F_CTRL_BYTES, "fine control block");

// Rows of a unit: longest first (later rows have more candidates until the
// block budget saturates), snake-dealt to CTAs.
struct FUnit {
  int r[F_QT];
  Cand c[F_QT];
  int nt;  // candidate tiles (the longer row's)
};

__device__ __forceinline__ FUnit f_decode(const FineParams& p, int u, int n_units) {
  FUnit U;
  const int r0 = F_QT * (n_units - 1 - u);
  U.nt = 0;
#pragma unroll
  for (int j = 0; j < F_QT; ++j) {
    U.r[j] = r0 + j;
    if (U.r[j] < p.R) {
      U.c[j] = cand_of(p, U.r[j]);
    } else {
      U.c[j].n_blk_keys = U.c[j].tail0 = U.c[j].count = 0;
    }
    const int nt = (U.c[j].count + F_KT - 1) / F_KT;
    U.nt = nt > U.nt ? nt : U.nt;
  }
  return U;
}

__global__ void __launch_bounds__(F_THREADS, 1)
    fine_score_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                      const FineParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = smem;
  uint8_t* a_s = smem + F_Q_BYTES;
  FCtrl* C = reinterpret_cast<FCtrl*>(smem + F_Q_BYTES + F_STAGES * F_STAGE_BYTES);
  volatile int* abort = &C->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = (p.R + F_QT - 1) / F_QT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < F_STAGES; ++s) {
      mbar_init(&C->full[s], p.box_rows ? 1 : F_PRODUCERS);
      mbar_init(&C->empty[s], 1);
    }
    mbar_init(&C->q_full, 1);
    mbar_init(&C->q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&C->t_full[b], 1);
      mbar_init(&C->t_empty[b], 8);
    }
    mbar_init(&C->mma_done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    if (p.box_rows) prefetch_tmap(&tm_kc);
  }
  if (warp == 1) tmem_alloc(&C->tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- q tiles (TMA)
      uint32_t qph = 0, issued = 0;
      for (int i = 0;; ++i) {
        const int u = f_unit_of(i, n_units);
        if (u < 0 || *abort) break;
        const FUnit U = f_decode(p, u, n_units);
        if (U.nt == 0) continue;
        if (!mbar_wait_bounded(&C->q_empty, qph ^ 1u, abort, p.wait_limit_ns)) {
          f_record(p, abort, FERR_QFREE);
          break;
        }
        qph ^= 1u;
        mbar_arrive_expect_tx(&C->q_full, F_Q_BYTES);
        tma_load_2d(q_s, &tm_q, &C->q_full, 0, U.r[0] * F_HEADS);
        tma_load_2d(q_s + F_Q_HALF, &tm_q, &C->q_full, 64, U.r[0] * F_HEADS);
        ++issued;
      }
      if (issued && !mbar_wait_timed(&C->q_full, (issued - 1) & 1u, p.wait_limit_ns))
        f_record(p, abort, FERR_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t IDESC = idesc_f32acc(1, 1, F_KT, F_HEADS);
      const uint32_t q_addr = smem_u32(q_s), a_addr = smem_u32(a_s);
      uint32_t stage = 0, phase = 0, qph = 0, acc = 0, accph = 0;
      bool stop = false;
      for (int i = 0; !stop; ++i) {
        const int u = f_unit_of(i, n_units);
        if (u < 0 || *abort) break;
        const FUnit U = f_decode(p, u, n_units);
        if (U.nt == 0) continue;
        if (!mbar_wait_bounded(&C->q_full, qph, abort, p.wait_limit_ns)) {
          f_record(p, abort, FERR_Q);
          break;
        }
        qph ^= 1u;
        tc_fence_after();
        for (int t = 0; t < U.nt && !stop; ++t) {
          if (!mbar_wait_bounded(&C->t_empty[acc], accph ^ 1u, abort, p.wait_limit_ns)) {
            f_record(p, abort, FERR_TEMPTY);
            stop = true;
            break;
          }
          if (!mbar_wait_bounded(&C->full[stage], phase, abort, p.wait_limit_ns)) {
            f_record(p, abort, FERR_FULL);
            stop = true;
            break;
          }
          tc_fence_after();
          fence_proxy_async();  // the cp.async path writes through the generic proxy
          {
            const uint32_t st_addr = a_addr + stage * F_STAGE_BYTES;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int j = 0; j < F_QT; ++j)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint32_t kb = kk * 32;  // 16 bf16 of K inside the 128-byte swizzled row
                  mma_bf16(tmem + acc * (F_QT * F_HEADS) + j * F_HEADS,
                           sdesc_kmajor_sw128_sbo(st_addr + j * F_A_QUERY + h * 1024 + kb, F_GROUP),
                           sdesc_kmajor_sw128(q_addr + h * F_Q_HALF + j * (F_HEADS * 128) + kb), IDESC,
                           (h | kk) != 0);
                }
            mma_commit(&C->empty[stage]);
            if (++stage == F_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (stop) break;
          mma_commit(&C->t_full[acc]);
          if (t == U.nt - 1) mma_commit(&C->q_empty);
          if (++acc == 2) {
            acc = 0;
            accph ^= 1u;
          }
        }
      }
      mma_commit(&C->mma_done);
      if (!mbar_wait_timed(&C->mma_done, 0, p.wait_limit_ns)) f_record(p, abort, FERR_DRAIN);
    }
  } else if (warp < 4 && p.box_rows) {
    // ------------------------------------------------------------ gather producer (TMA boxes)
    // Every group of 8 candidate slots is 8 consecutive key rows that start
    // on a multiple of gcd(G, 8): a kept block's keys (or 8 of them) or the
    // incomplete block's.  Warp 2, lane l, loads group l % 16 of query l / 16
    // into its 2 KB of the stage: with box_rows 8 as one 3-D box (8 rows x
    // both 64-dim K halves), with box_rows 4 as four 2-D boxes (4 rows x 64
    // dims); lane 0 owns the barriers.
    // Slots past the row's candidates read key row 0 (their scores are never
    // stored), rows past the keys read as zero.  Warp 3 has nothing to do.
    if (warp == 2) {
      const bool j1 = (lane >> 4) != 0;  // this lane's query, chosen without a dynamic index
      const int bb = lane & 15;
      uint32_t stage = 0, phase = 0;
      uint32_t any_load = 0, last_par = 0;  // per stage: loaded at all / parity of the last load
      bool stop = false;
      for (int i = 0; !stop; ++i) {
        const int u = f_unit_of(i, n_units);
        if (u < 0 || __any_sync(0xFFFFFFFFu, *abort != 0)) break;  // the warp decides as one
        const FUnit U = f_decode(p, u, n_units);
        const int rj = j1 ? U.r[1] : U.r[0];
        const Cand c = j1 ? U.c[1] : U.c[0];
        const int32_t* crow = p.coarse + static_cast<size_t>(rj < p.R ? rj : 0) * p.n_keep;
        // the key rows of this lane's group of tile t (at most two runs of 4):
        // the kept-block entries of tile t + 1 are loaded (unconditionally,
        // clamped in range) while tile t's boxes are issued, and turned into
        // rows one tile later, so their latency is hidden
        auto load_blk = [&](int t, int* blk) {
#pragma unroll
          for (int x = 0; x < 2; ++x) blk[x] = crow[min(blk_slot(p, t * F_KT + 8 * bb + x * 4), p.n_keep - 1)];
        };
        int blk_next[2];
        load_blk(0, blk_next);
        for (int t = 0; t < U.nt && !stop; ++t) {
          int row[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int s1 = t * F_KT + 8 * bb + x * 4, blk = blk_next[x];
            int kr = 0;
            if (s1 < c.n_blk_keys) kr = blk >= 0 && blk < p.nb ? blk * p.G + in_blk(p, s1) : 0;
            else if (s1 < c.count) kr = c.tail0 + (s1 - c.n_blk_keys);
            row[x] = kr;
          }
          if (t + 1 < U.nt) load_blk(t + 1, blk_next);
          bool got = true;
          if (lane == 0) {
            got = mbar_wait_bounded(&C->empty[stage], phase ^ 1u, abort, p.wait_limit_ns);
            if (!got)
              f_record(p, abort, FERR_EMPTY);
            else
              mbar_arrive_expect_tx(&C->full[stage], F_STAGE_BYTES);
          }
          if (__shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) == 0) {  // the warp gives up as one
            stop = true;
            break;
          }
          __syncwarp();
          uint8_t* dst = a_s + stage * F_STAGE_BYTES + (j1 ? F_A_QUERY : 0) + bb * F_GROUP;
          if (p.box3d) {
            // both K halves of the 8 rows in one box: [half][row][64 dims]
            tma_load_3d(dst, &tm_kc, &C->full[stage], 0, row[0], 0);
          } else {  // box_rows 4: four 2-D boxes of 4 rows x 64 dims
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              tma_load_2d(dst + h * 1024, &tm_kc, &C->full[stage], h * 64, row[0]);
              tma_load_2d(dst + h * 1024 + 512, &tm_kc, &C->full[stage], h * 64, row[1]);
            }
          }
          any_load |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == F_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every load issued has landed before the CTA can exit
      if (lane == 0)
        for (int s2 = 0; s2 < F_STAGES; ++s2)
          if (((any_load >> s2) & 1u) && !mbar_wait_timed(&C->full[s2], (last_par >> s2) & 1u, p.wait_limit_ns))
            f_record(p, abort, FERR_DRAIN);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ gather producers
    // Block sizes not divisible by 4.  Thread pt moves 16-byte chunk (pt & 7)
    // of rows (pt >> 3) + 8x, x = 0..15, of each query's 128-row tile, both K
    // halves: 8 consecutive threads read one 128-byte half row.  Chunk c of
    // row r, half h lands in r's group at h*1024 + (r & 7)*128 + ((c ^ (r & 7))
    // << 4): the 128-byte swizzle the MMA descriptor expects.  Each thread's
    // copies of a stage arrive on its barrier when they land (noinc).
    const int pt = threadIdx.x - 64;
    const int ch = pt & 7, rb = pt >> 3;
    uint32_t stage = 0, phase = 0;
    bool stop = false;
    for (int i = 0; !stop; ++i) {
      const int u = f_unit_of(i, n_units);
      if (u < 0 || __any_sync(0xFFFFFFFFu, *abort != 0)) break;  // the warp decides as one
      const FUnit U = f_decode(p, u, n_units);
      for (int t = 0; t < U.nt && !stop; ++t) {
        // the tile's kept-block indices: 32 unconditional loads (clamped in
        // range) so that they are all in flight at once
        int key[F_QT][16];
#pragma unroll
        for (int j = 0; j < F_QT; ++j) {
          const int32_t* crow = p.coarse + static_cast<size_t>(U.r[j] < p.R ? U.r[j] : 0) * p.n_keep;
#pragma unroll
          for (int x = 0; x < 16; ++x) key[j][x] = crow[min(blk_slot(p, t * F_KT + rb + 8 * x), p.n_keep - 1)];
        }
#pragma unroll
        for (int j = 0; j < F_QT; ++j)
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int s = t * F_KT + rb + 8 * x;
            const Cand& c = U.c[j];
            int kk = -1;
            if (s < c.n_blk_keys) kk = key[j][x] >= 0 && key[j][x] < p.nb ? key[j][x] * p.G + in_blk(p, s) : -1;
            else if (s < c.count) kk = c.tail0 + (s - c.n_blk_keys);
            key[j][x] = kk < 0 ? 0 : kk;  // an empty slot reads key 0; its score is never stored
          }
        const bool got = mbar_wait_bounded(&C->empty[stage], phase ^ 1u, abort, p.wait_limit_ns);
        if (!__all_sync(0xFFFFFFFFu, got)) {  // the warp gives up as one
          if (lane == 0) f_record(p, abort, FERR_EMPTY);
          stop = true;
          break;
        }
        const uint32_t base = smem_u32(a_s + stage * F_STAGE_BYTES);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < F_QT; ++j)
#pragma unroll
            for (int x = 0; x < 16; ++x) {  // row rb + 8x is row rb of group x
              const uint8_t* src = p.kc + static_cast<size_t>(key[j][x]) * (F_DIM * 2) + h * 128 + ch * 16;
              cp_async16(base + j * F_A_QUERY + x * F_GROUP + h * 1024 + rb * 128 + ((ch ^ rb) << 4), src);
            }
        cp_async_arrive_noinc(&C->full[stage]);
        if (++stage == F_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    cp_async_wait_0();  // every copy issued has landed before the CTA can exit
  } else {
    // ------------------------------------------------------------ scoring warps
    const int quad = warp & 3;               // TMEM lanes 32*quad .. +31
    const int j = (warp - 4) >> 2;           // this warp's query of the unit
    uint32_t acc = 0, accph = 0;
    bool ok = !__any_sync(0xFFFFFFFFu, *abort != 0);
    for (int i = 0; ok; ++i) {
      const int u = f_unit_of(i, n_units);
      if (u < 0) break;
      const FUnit U = f_decode(p, u, n_units);
      if (U.nt == 0) continue;
      const int r = U.r[j];
      const bool row_ok = r < p.R;
      float wr[F_HEADS];
#pragma unroll
      for (int h4 = 0; h4 < F_HEADS / 4; ++h4) {
        const float4 v = row_ok ? reinterpret_cast<const float4*>(p.w + static_cast<size_t>(r) * F_HEADS)[h4]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        wr[4 * h4] = v.x;
        wr[4 * h4 + 1] = v.y;
        wr[4 * h4 + 2] = v.z;
        wr[4 * h4 + 3] = v.w;
      }
      // each tile's key is fetched one tile ahead, so its load latency
      // hides behind the previous tile
      int key_next = row_ok ? key_of(p, U.c[j], r, quad * 32 + lane) : -1;
      for (int t = 0; t < U.nt; ++t) {
        const int s = t * F_KT + quad * 32 + lane;
        const int key = key_next;
        key_next = row_ok && t + 1 < U.nt ? key_of(p, U.c[j], r, s + F_KT) : -1;
        const bool got = mbar_wait_bounded(&C->t_full[acc], accph, abort, p.wait_limit_ns);
        if (!__all_sync(0xFFFFFFFFu, got)) {  // the warp gives up as one
          if (lane == 0) f_record(p, abort, FERR_TFULL);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t x[64];
        tmem_ld32_x64(tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * (F_QT * F_HEADS) + j * F_HEADS, x);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&C->t_empty[acc]);
        if (++acc == 2) {
          acc = 0;
          accph ^= 1u;
        }
        if (key >= 0) {
          float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < F_HEADS; ++h) a[h & 3] = fmaf(wr[h], fmaxf(__uint_as_float(x[h]), 0.f), a[h & 3]);
          const float sc = (a[0] + a[1]) + (a[2] + a[3]);
          p.packed[static_cast<size_t>(r) * p.ldp + s] =
              (static_cast<uint64_t>(f_ord(sc)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(key));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------- select
// Exact top-k of a row's packed candidate keys (distinct: the low half is
// ~index).  A first pass bins the keys by where their orderable score falls in
// the row's own range (2048 bins, shared-memory atomics) and finds the bin B
// that holds the k-th largest; the keys above B are in.  When B is not taken
// whole, its keys (usually a handful) go to a list and a radix select (8 bits
// a pass from the top, per-warp histograms fed by warp-aggregated atomics)
// picks the ones still needed; a bin of more than S_LCAP keys (many equal
// scores) falls back to the radix select over the whole row.  The k keys are
// stored in no particular order (the row sort orders them).
constexpr int S_THREADS = 512;
constexpr int S_WARPS = S_THREADS / 32;
constexpr int S_BINS = 2048;   // first-pass bins, 4 a thread
constexpr int S_LCAP = 4096;   // largest boundary bin handled as a list
static_assert(S_BINS == 4 * S_THREADS, "the bin scan gives each thread 4 bins");

// Block-wide: the largest prefix p such that at least `need` of keys[0..cnt)
// are >= p, built 8 bits a pass from the top (the threshold of the need-th
// largest key).  `hist` is [S_WARPS][256], `tot` [256].
__device__ uint64_t radix_threshold(const uint64_t* keys, int cnt, uint32_t need, uint32_t* hist, uint32_t* tot,
                                    uint64_t* s_prefix, uint32_t* s_need, uint32_t* s_done) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __syncthreads();  // the caller's shared state is settled
  if (tid == 0) {
    *s_prefix = 0;
    *s_need = need;
    *s_done = static_cast<uint32_t>(cnt) <= need ? 1u : 0u;
  }
  __syncthreads();
  uint64_t mask = 0;
  for (int shift = 56; shift >= 0 && !*s_done; shift -= 8) {
    for (int i = tid; i < S_WARPS * 256; i += S_THREADS) hist[i] = 0;
    __syncthreads();
    const uint64_t prefix = *s_prefix;
    for (int i0 = 0; i0 < cnt; i0 += S_THREADS) {
      const int i = i0 + tid;
      const bool in = i < cnt && (keys[i < cnt ? i : 0] & mask) == prefix;
      const uint32_t d = in ? static_cast<uint32_t>(keys[i] >> shift) & 255u : 256u;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, d);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[warp * 256 + d], __popc(peers));
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t sum = 0;
      for (int w = 0; w < S_WARPS; ++w) sum += hist[w * 256 + tid];
      tot[tid] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l; find the bin where the count
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
        uint32_t above = excl;
        int b = 0;
        for (int e = 0; e < 8; ++e) {
          if (above + v[e] >= nd) {
            b = 255 - 8 * lane - e;
            break;
          }
          above += v[e];
        }
        *s_prefix = prefix | (static_cast<uint64_t>(b) << shift);
        *s_need = nd - above;
        if (nd - above == tot[b]) *s_done = 1u;  // the whole bin is in: threshold found
      }
    }
    mask |= static_cast<uint64_t>(255) << shift;
    __syncthreads();
  }
  const uint64_t thr = *s_prefix;
  __syncthreads();  // every thread has read the threshold
  return thr;
}

__global__ void __launch_bounds__(S_THREADS) select_topk_kernel(const uint64_t* __restrict__ packed,
                                                                const FineParams p, int k, int32_t* out_idx,
                                                                float* out_score) {
  extern __shared__ __align__(16) uint8_t s_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(s_raw);          // [S_WARPS][256]
  uint32_t* tot = hist + S_WARPS * 256;                          // [256]
  uint32_t* bins = tot + 256 + 4;                                // [S_BINS]
  uint64_t* list = reinterpret_cast<uint64_t*>(bins + S_BINS);   // [S_LCAP]
  uint64_t* keys = list + S_LCAP;                                // [ldp]
  __shared__ uint64_t s_prefix;
  __shared__ uint32_t s_need, s_done, s_out, s_nl, s_B, s_A, s_cB;
  __shared__ uint32_t s_max[S_WARPS], s_min[S_WARPS], s_wsum[S_WARPS];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int r = blockIdx.x; r < p.R; r += gridDim.x) {
    const Cand c = cand_of(p, r);
    const int cnt = c.count;
    const uint64_t* row = packed + static_cast<size_t>(r) * p.ldp;
    int32_t* oi = out_idx + static_cast<size_t>(r) * k;
    float* os = out_score + static_cast<size_t>(r) * k;
    // keys into shared memory, and the range of their orderable scores
    uint32_t mx = 0u, mn = 0xFFFFFFFFu;
    for (int i = tid; i < cnt; i += S_THREADS) {
      const uint64_t x = row[i];
      keys[i] = x;
      const uint32_t hi = static_cast<uint32_t>(x >> 32);
      mx = max(mx, hi);
      mn = min(mn, hi);
    }
    for (int i = tid; i < S_BINS; i += S_THREADS) bins[i] = 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      mn = min(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, o));
    }
    if (lane == 0) {
      s_max[warp] = mx;
      s_min[warp] = mn;
    }
    if (tid == 0) {
      s_out = 0;
      s_nl = 0;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < S_WARPS; ++w) {
      mx = max(mx, s_max[w]);
      mn = min(mn, s_min[w]);
    }
    // modes: 0 take all, 1 bins <= B, 2 bins < B plus the list's best, 3 keys >= thr
    int mode = 0, B = 0, sh = 0;
    uint64_t thr = 0ull;
    if (cnt > k) {
      const uint32_t range = mx - mn;
      const int bl = range ? 32 - __clz(static_cast<int>(range)) : 0;
      sh = bl > 11 ? bl - 11 : 0;
      for (int i = tid; i < cnt; i += S_THREADS)
        atomicAdd(&bins[(mx - static_cast<uint32_t>(keys[i] >> 32)) >> sh], 1u);
      __syncthreads();
      // exclusive scan of the bins from the top: thread t owns bins 4t .. 4t+3
      uint32_t cb[4], sum = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        cb[e] = bins[4 * tid + e];
        sum += cb[e];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) s_wsum[warp] = incl;
      __syncthreads();
      uint32_t excl = incl - sum;
      for (int w = 0; w < warp; ++w) excl += s_wsum[w];
      const uint32_t kk = static_cast<uint32_t>(k);
      if (excl < kk && kk <= excl + sum) {
        uint32_t above = excl;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (above + cb[e] >= kk) {
            s_B = 4 * tid + e;
            s_A = above;
            s_cB = cb[e];
            break;
          }
          above += cb[e];
        }
      }
      __syncthreads();
      B = static_cast<int>(s_B);
      const uint32_t need = kk - s_A, cB = s_cB;
      if (need == cB) {
        mode = 1;
      } else if (cB <= static_cast<uint32_t>(S_LCAP)) {
        for (int i = tid; i < cnt; i += S_THREADS) {
          const uint64_t x = keys[i];
          if (static_cast<int>((mx - static_cast<uint32_t>(x >> 32)) >> sh) == B) list[atomicAdd(&s_nl, 1u)] = x;
        }
        thr = radix_threshold(list, static_cast<int>(cB), need, hist, tot, &s_prefix, &s_need, &s_done);
        mode = 2;
      } else {
        thr = radix_threshold(keys, cnt, kk, hist, tot, &s_prefix, &s_need, &s_done);
        mode = 3;
      }
    }
    // the chosen keys: exactly min(k, cnt) of them
    for (int i0 = 0; i0 < cnt; i0 += S_THREADS) {
      const int i = i0 + tid;
      bool take = false;
      uint64_t x = 0ull;
      if (i < cnt) {
        x = keys[i];
        const int b = static_cast<int>((mx - static_cast<uint32_t>(x >> 32)) >> sh);
        take = mode == 0 || (mode == 1 && b <= B) || (mode == 2 && (b < B || (b == B && x >= thr))) ||
               (mode == 3 && x >= thr);
      }
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, take);
      uint32_t base = 0;
      if (lane == 0 && bal) base = atomicAdd(&s_out, __popc(bal));
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
      if (take) {
        const uint32_t pos = base + __popc(bal & ((1u << lane) - 1u));
        if (pos < static_cast<uint32_t>(k)) {
          const uint32_t o = static_cast<uint32_t>(x >> 32);
          oi[pos] = static_cast<int32_t>(~static_cast<uint32_t>(x));
          os[pos] = __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
        }
      }
    }
    for (int x = (cnt < k ? cnt : k) + tid; x < k; x += S_THREADS) {
      oi[x] = -1;
      os[x] = -__int_as_float(0x7f800000);
    }
    __syncthreads();
  }
}

}  // namespace

size_t two_stage_workspace_bytes(int B, int S, int T, int G, int n_keep, int chunk) {
  const size_t nb = static_cast<size_t>(T / G);
  const size_t ldp = (static_cast<size_t>(n_keep) * G + G + 15) / 16 * 16;
  const size_t ch = static_cast<size_t>(std::min(chunk, S));
  const size_t a = 256;
  return (B * nb * F_DIM * 2 + a) + (ch * n_keep * 4 + a) + (ch * ldp * 8 + a) + a;
}

si_status launch_two_stage(const void* q, const void* kc, const float* w, int B, int S, int T, int m, int k,
                           int G, int n_keep, int chunk, int32_t* out_idx, float* out_score, void* workspace,
                           size_t workspace_bytes, uint64_t wait_limit_ns, int* err, cudaStream_t stream) {
  const size_t need = two_stage_workspace_bytes(B, S, T, G, n_keep, chunk);
  void* raw = nullptr;
  void* ws = workspace;
  if (ws) {
    if (workspace_bytes < need)
      return fail(SI_ERR_INVALID_ARGUMENT, "workspace of %zu bytes < %zu needed", workspace_bytes, need);
  } else {
    const si_status sa = scratch_alloc(&raw, need, stream, "the two-stage scratch");
    if (sa != SI_OK) return sa;
    ws = raw;
  }
  auto carve = [](uintptr_t& cur, size_t bytes) {
    cur = (cur + 255) & ~static_cast<uintptr_t>(255);
    const uintptr_t at = cur;
    cur += bytes;
    return reinterpret_cast<void*>(at);
  };
  const int nb = T / G;
  const int ldp = (n_keep * G + G + 15) / 16 * 16;
  const int ch = std::min(chunk, S);
  uintptr_t cur = reinterpret_cast<uintptr_t>(ws);
  auto* kp = static_cast<__nv_bfloat16*>(carve(cur, static_cast<size_t>(B) * nb * F_DIM * 2));
  auto* coarse = static_cast<int32_t*>(carve(cur, static_cast<size_t>(ch) * n_keep * 4));
  auto* packed = static_cast<uint64_t*>(carve(cur, static_cast<size_t>(ch) * ldp * 8));

  si_status st = SI_OK;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) st = cuda_fail(e, "device query");
  if (st == SI_OK && nb > 0) {
    const long long n = static_cast<long long>(B) * nb * F_DIM;
    const long long grid = std::min<long long>((n + 127) / 128, static_cast<long long>(n_sm) * 16);
    pool_keys_kernel<<<static_cast<unsigned>(grid), 128, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(kc), kp, B, T, G, nb);
    e = cudaGetLastError();
    if (e != cudaSuccess) st = cuda_fail(e, "pool_keys_kernel launch");
  }
  if (st == SI_OK) {
    e = cudaFuncSetAttribute(fine_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM);
    if (e != cudaSuccess) st = cuda_fail(e, "cudaFuncSetAttribute(fine_score_kernel)");
  }
  const size_t sel_smem = static_cast<size_t>(S_WARPS) * 256 * 4 + 256 * 4 + 16 + S_BINS * 4 +
                          static_cast<size_t>(S_LCAP) * 8 + static_cast<size_t>(ldp) * 8;
  if (st == SI_OK) {
    e = cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sel_smem));
    if (e != cudaSuccess) st = cuda_fail(e, "cudaFuncSetAttribute(select_topk_kernel)");
  }
  // the coarse stage's partition size: 512 keys, halved until its pool fits;
  // a budget above 1024 blocks leaves the pool little room over n_keep, and
  // 128-key partitions (which compact it less often) measured 3x faster than
  // 256 at n_keep = 2048
  int key_tile = n_keep > 1024 ? 128 : 512;
  {
    int ns = 0, cap = 0;
    size_t bytes = 0;
    while (key_tile > 64 && !stream_smem_plan(n_keep, key_tile, 0, &ns, &cap, &bytes)) key_tile >>= 1;
  }
  const size_t row_q = static_cast<size_t>(F_HEADS) * F_DIM * 2;  // bytes of one query row of q
  for (int b = 0; b < B && st == SI_OK; ++b) {
    for (int c0 = 0; c0 < S && st == SI_OK; c0 += ch) {
      const int R = std::min(ch, S - c0);
      const uint8_t* qb = static_cast<const uint8_t*>(q) + (static_cast<size_t>(b) * S + c0) * row_q;
      const float* wb = w + (static_cast<size_t>(b) * S + c0) * F_HEADS;
      if (nb > 0) {
        StreamConfig cfg;
        cfg.query_chunk = 0;
        cfg.key_tile = key_tile;
        cfg.fp8 = 0;
        cfg.q_scale = nullptr;
        cfg.kc_scale = nullptr;
        cfg.wait_limit_ns = wait_limit_ns;
        cfg.test_withhold = 0;
        cfg.unsorted = true;
        cfg.row0 = c0;
        cfg.err = err;
        st = launch_stream_topk(qb, kp + static_cast<size_t>(b) * nb * F_DIM, wb, 1, R, nb, F_HEADS, F_DIM, m * G,
                                n_keep, coarse, nullptr, stream, cfg);
        if (st != SI_OK) break;
      }
      CUtensorMap tm_q, tm_kc;
      st = encode_tmap_2d(&tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qb, F_DIM, static_cast<uint64_t>(R) * F_HEADS,
                          F_DIM * 2, 64, F_QT * F_HEADS);
      if (st != SI_OK) break;
      // candidates come in runs of gcd(G, 8) consecutive key rows starting on
      // a multiple of it; runs of 4 or 8 rows load as TMA boxes of the keys
      // a multiple of 8 loads both K halves of 8 rows as one 3-D box (the keys
      // seen as [2 halves][T rows][64 dims]) where the driver takes that
      // layout; a multiple of 4 (or a refused 3-D map) as 2-D boxes of 4 rows
      int box_rows = (G % 4 == 0) ? 4 : 0;
      int box3d = 0;
      tm_kc = tm_q;  // unused unless box_rows
      const uint8_t* kcb = static_cast<const uint8_t*>(kc) + static_cast<size_t>(b) * T * F_DIM * 2;
      if (G % 8 == 0) {
        const uint64_t dims[3] = {64, static_cast<uint64_t>(T), 2};
        const uint64_t strides[2] = {F_DIM * 2, 128};
        const uint32_t box[3] = {64, 8, 2};
        box3d = try_encode_tmap_3d(&tm_kc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kcb, dims, strides, box) ? 1 : 0;
        if (box3d) box_rows = 8;
      }
      if (box_rows == 4) {
        st = encode_tmap_2d(&tm_kc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kcb, F_DIM, static_cast<uint64_t>(T),
                            F_DIM * 2, 64, 4);
        if (st != SI_OK) break;
      }
      FineParams fp;
      fp.kc = static_cast<const uint8_t*>(kc) + static_cast<size_t>(b) * T * F_DIM * 2;
      fp.w = wb;
      fp.coarse = coarse;
      fp.packed = packed;
      fp.err = err;
      fp.R = R;
      fp.T = T;
      fp.m = m;
      fp.G = G;
      fp.n_keep = n_keep;
      fp.ldp = ldp;
      fp.nb = nb;
      fp.g_shift = (G & (G - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(G)) : -1;
      fp.row0 = c0;
      fp.box_rows = box_rows;
      fp.box3d = box3d;
      fp.wait_limit_ns = wait_limit_ns;
      const int units = (R + F_QT - 1) / F_QT;
      fine_score_kernel<<<static_cast<unsigned>(std::min(units, n_sm)), F_THREADS, F_SMEM, stream>>>(tm_q, tm_kc, fp);
      e = cudaGetLastError();
      if (e != cudaSuccess) {
        st = cuda_fail(e, "fine_score_kernel launch");
        break;
      }
      const size_t ob = (static_cast<size_t>(b) * S + c0) * k;
      select_topk_kernel<<<static_cast<unsigned>(std::min(R, n_sm * 4)), S_THREADS, sel_smem, stream>>>(
          packed, fp, k, out_idx + ob, out_score + ob);
      e = cudaGetLastError();
      if (e != cudaSuccess) st = cuda_fail(e, "select_topk_kernel launch");
    }
  }
  if (st == SI_OK) st = launch_row_sort(out_idx, out_score, static_cast<long long>(B) * S, k, stream);
  if (raw) {
    e = cudaFreeAsync(raw, stream);
    if (e != cudaSuccess && st == SI_OK) st = cuda_fail(e, "cudaFreeAsync");
  }
  return st;
}

}  // namespace si
