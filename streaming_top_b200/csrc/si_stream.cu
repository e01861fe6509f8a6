// Streaming lightning-indexer top-k for sm_100a.
//
// StreamIndex (abstract): the indexer scores compressed keys and a chunked
// partition-merge top-k keeps the per-query top-k without ever materialising
// the [B, S, H_I, T] fp32 score tensor.  Score (DeepSeek-V3.2 indexer form):
//   I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . kc[s,:]),  key s visible iff s*m+m-1 <= t.
//
// One CTA per SM (persistent).  A work unit is a tile of QT = 4 consecutive
// queries of one sequence; units are taken longest-first (the causal triangle
// makes late queries see the most keys) and dealt to CTAs in snake order.
//
// Warp roles (16 warps):
//   warp 0 (one lane)   TMA: the unit's q tile [4 queries x 64 heads, 128]
//                       (stationary), then key tiles [128 keys, 128] through
//                       an N-stage mbarrier ring -- only tiles holding a
//                       visible key.
//   warp 1 (one lane)   tcgen05.mma, A = key tile (M = 128 keys), B = q tile
//                       (N = 256 = 4 queries x 64 heads), K = 128, fp32
//                       accumulator in TMEM, double buffered (2 x 256
//                       columns) so the MMA of tile j+1 overlaps the
//                       epilogue of tile j.
//   warps 8..15         scoring.  Warp = TMEM lane quadrant (warp % 4, 32
//                       keys) x 2 of the 4 queries.  tcgen05.ld 32x32b gives
//                       each thread one key's 64 head logits per query (the
//                       32-lane shape drains TMEM several times faster than
//                       the 16-lane ones); the accumulator is released as
//                       soon as it is in registers.  ReLU and the w-weighted
//                       head sum run in registers: one query's weights sit in
//                       registers, the other's are read from a per-warp
//                       shared-memory table by broadcast loads.  Causal mask,
//                       then threshold early-reject: a key becomes a
//                       candidate only if its score beats the threshold its
//                       manager last published; each warp compacts its
//                       candidates into its segment of a slot of a ring of
//                       per-tile candidate buffers.
//   warps 4..7          top-k managers, one per query: per tile they move the
//                       query's candidates from the ring slot into the
//                       query's running pool and count them into a 256-bin
//                       histogram of its scores; at the end of every
//                       partition of `key_tile` keys (the pages' key tile)
//                       they raise and publish the threshold and compact the
//                       pool when it fills; at the end of the unit they
//                       select the exact k best and store them (sorted only
//                       when no scores are stored; otherwise a row-sort pass
//                       orders the rows) -- while the scoring warps already
//                       work on the next unit.
//   warps 2, 3          idle (they complete warpgroup 0).
//
// Keys are packed as (orderable fp32 score << 32) | ~index, so one unsigned
// 64-bit comparison orders by score descending, then index ascending, and
// every key is distinct.  Because key tiles are visited in index order and a
// threshold only ever comes from keys of earlier partitions, a new key whose
// score merely ties the threshold has a larger index than the k-th kept key
// and is correctly rejected: the filter needs the score only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"
#include "si_ptx.cuh"
#include "si_topk.cuh"

namespace si {
namespace {

constexpr int QT = 4;              // queries per unit
constexpr int HEADS = 64;          // indexer heads (H_I)
constexpr int DIM = 128;           // head dim (D)
constexpr int KT = 128;            // keys per MMA tile (M)
constexpr int NCOLS = QT * HEADS;  // 256 = MMA N
constexpr int THREADS = 512;       // 16 warps
constexpr int N_SCORE_WARPS = 8;
constexpr int HIST_BINS = 256;
// Candidate ring between scorers and managers: per slot (one key tile) and
// query, one segment of up to 32 candidates per TMEM lane quadrant.
constexpr int RING = 4;
constexpr int RING_BYTES = RING * QT * 4 * 32 * 8;
constexpr int CTRL_BYTES = 1024;
// Head weights of the current unit, one private copy per scoring warp (its
// two queries x 64 heads, fp32).
constexpr int WTAB_BYTES = N_SCORE_WARPS * 2 * 64 * 4;
// Register budgets: launched at 128 per thread (512 threads); warpgroup 0
// (producer, MMA) and warpgroup 1 (managers) give registers to the two
// scoring warpgroups: 128 * 40 + 128 * 120 + 256 * 176 = 65536.
constexpr uint32_t REGS_PIPE = 40;
constexpr uint32_t REGS_MGR = 120;
constexpr uint32_t REGS_SCORE = 176;
static_assert(128 * REGS_PIPE + 128 * REGS_MGR + 256 * REGS_SCORE <= 512 * 128, "register split");


enum { ERR_WAIT_Q = 1, ERR_WAIT_KC = 2, ERR_WAIT_TMEM_EMPTY = 3, ERR_WAIT_TMEM_FULL = 4,
       ERR_WAIT_QFREE = 5, ERR_WAIT_KFREE = 6, ERR_WAIT_DRAIN = 7, ERR_WAIT_RING_FREE = 8,
       ERR_WAIT_RING_FULL = 9 };

struct Params {
  const float* w;         // [B,S,H]
  const float* q_scale;   // fp8: [B,S,H]
  const float* kc_scale;  // fp8: [B,T]
  int32_t* out_idx;       // [B,S,k]
  float* out_score;       // [B,S,k] or null
  int* err;               // device error record
  int B, S, T, m, k;      // S: rows held per sequence (q, w and outputs hold S rows)
  int row0;               // absolute position of row 0 (causal visibility uses row0 + t)
  int qt_begin, qt_end;   // query tiles (per sequence) of this launch
  int key_tile;           // partition length in keys (64 or multiple of 128)
  int cap;                // main-region entries per query pool
  int n_stages;
  uint64_t wait_limit_ns;
  int test_withhold;
  int sort_rows;          // finalize sorts each row itself (no scores to sort by later)
};

// A work item: one unit (4 consecutive queries of one sequence) and, when
// the unit's keys are split over CTAs, one contiguous range of its key
// tiles [kt0, kt1).
struct SplitParams {
  int n_split;            // key partitions per unit, each on its own CTA (1: none)
  int32_t* part_idx;      // n_split > 1: per-partition top-k [B][part_rows][n_split][k]
  float* part_score;
  int part_rows;          // rows per sequence in the partials (the launch's query tiles x 4)
};

struct Unit {
  int b, t0, n_keys, kt0, kt1, sp;
};

// SPLIT: the launch splits units' keys over CTAs (n_split partitions); the
// other instantiation keeps whole units (n_split == 1) and pays nothing for it.
template <bool SPLIT>
__device__ __forceinline__ Unit decode_unit(int w, const Params& p, const SplitParams& x) {
  Unit r;
  const int u = SPLIT ? w / x.n_split : w;
  r.sp = SPLIT ? w - u * x.n_split : 0;
  r.b = u % p.B;
  const int qt = p.qt_end - 1 - u / p.B;
  r.t0 = qt * QT;
  const int t_last = min(r.t0 + QT, p.S) - 1;
  const int n = (p.row0 + t_last + 1) / p.m;
  r.n_keys = n < p.T ? n : p.T;
  const int n_kt = (r.n_keys + KT - 1) / KT;
  r.kt0 = SPLIT ? static_cast<int>(static_cast<long long>(r.sp) * n_kt / x.n_split) : 0;
  r.kt1 = SPLIT ? static_cast<int>(static_cast<long long>(r.sp + 1) * n_kt / x.n_split) : n_kt;
  return r;
}

// Unit index handed to this CTA in round i (snake order), or -1 when done.
__device__ __forceinline__ int unit_of(int i, int n_units) {
  const int G = gridDim.x, c = blockIdx.x;
  const long long base = static_cast<long long>(i) * G;
  if (base >= n_units) return -1;
  const long long u = base + ((i & 1) ? (G - 1 - c) : c);
  return u < n_units ? static_cast<int>(u) : -1;
}

__device__ __forceinline__ uint32_t f32_ord(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void record_error(const Params& p, volatile int* abort, int where) {
  atomicCAS(p.err, 0, static_cast<int>(SI_ERR_TIMEOUT));
  atomicCAS(p.err + 1, 0, where);
  *abort = 1;
}

// Packed fp32 pair FMA (sm_100): d = a * b + d on two lanes of a 64-bit register.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rd, {%0, %1};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rd;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ float relu_u(uint32_t x) { return fmaxf(__uint_as_float(x), 0.f); }

// One query's score for the thread's key: x holds the key's 64 head logits
// (a 32x32b TMEM load: thread = key, register = head), w the query's 64 head
// weights in shared memory (every lane reads the same address: broadcast).
// Four independent packed-FMA chains of 8 steps each.
__device__ __forceinline__ float score_key(const uint32_t (&x)[64], const float* w) {
  float a[4][2];
#pragma unroll
  for (int c = 0; c < 4; ++c) a[c][0] = a[c][1] = 0.f;
  const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float4 wv = w4[c];
    fma2(a[c & 3][0], a[c & 3][1], wv.x, wv.y, relu_u(x[4 * c]), relu_u(x[4 * c + 1]));
    fma2(a[(c + 2) & 3][0], a[(c + 2) & 3][1], wv.z, wv.w, relu_u(x[4 * c + 2]), relu_u(x[4 * c + 3]));
  }
  return ((a[0][0] + a[0][1]) + (a[1][0] + a[1][1])) + ((a[2][0] + a[2][1]) + (a[3][0] + a[3][1]));
}

// The same with the query's 64 head weights in registers.
__device__ __forceinline__ float score_key_regs(const uint32_t (&x)[64], const float (&w)[64]) {
  float a[4][2];
#pragma unroll
  for (int c = 0; c < 4; ++c) a[c][0] = a[c][1] = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    fma2(a[c & 3][0], a[c & 3][1], w[4 * c], w[4 * c + 1], relu_u(x[4 * c]), relu_u(x[4 * c + 1]));
    fma2(a[(c + 2) & 3][0], a[(c + 2) & 3][1], w[4 * c + 2], w[4 * c + 3], relu_u(x[4 * c + 2]),
         relu_u(x[4 * c + 3]));
  }
  return ((a[0][0] + a[0][1]) + (a[1][0] + a[1][1])) + ((a[2][0] + a[2][1]) + (a[3][0] + a[3][1]));
}

// Shared-memory layout (offsets from a 1024-byte aligned base).
template <int OPB>
struct Layout {
  static constexpr int Q_HALF = NCOLS * 128;         // one 128-byte-wide K column block of q
  static constexpr int Q_BYTES = NCOLS * DIM * OPB;  // 64 KB bf16, 32 KB fp8
  static constexpr int KC_HALF = KT * 128;
  static constexpr int KC_BYTES = KT * DIM * OPB;    // 32 KB bf16, 16 KB fp8
  static constexpr int N_MMA = DIM * OPB / 32;       // K steps of 32 bytes
};

struct Smem {
  uint32_t q, kc, pool, hist, ring, wtab, ctrl;
};

// Per-query pools of `cap` entries, then the histograms, the candidate ring
// ([slot][query][quadrant][32] packed keys), the weight tables and the
// control block.
__host__ __device__ inline Smem carve(int n_stages, int cap, int q_bytes, int kc_bytes) {
  Smem s;
  s.q = 0;
  s.kc = q_bytes;
  s.pool = s.kc + n_stages * kc_bytes;
  s.hist = s.pool + QT * cap * 8;
  s.ring = s.hist + QT * HIST_BINS * 4;
  s.wtab = s.ring + RING_BYTES;
  s.ctrl = s.wtab + WTAB_BYTES;
  return s;
}

// Control block (CTRL_BYTES): mbarriers, manager state, TMEM slot, abort flag.
struct Ctrl {
  uint64_t full[4], empty[4];
  uint64_t q_full, q_empty;
  uint64_t t_full[2], t_empty[2];
  uint64_t mma_done;
  uint64_t ring_full[RING];   // the 8 scoring warps have written the slot
  uint64_t ring_free[RING];   // the 4 managers have read the slot
  uint64_t pub[QT];           // (unit tag << 32) | threshold, published by the managers
  alignas(16) topk::QState qs[QT];
  alignas(16) uint32_t ring_cnt[RING][QT][4];
  uint32_t tmem_slot;
  int abort;
};
static_assert(sizeof(Ctrl) <= CTRL_BYTES, "control block");

template <int OPB, bool SPLIT>
__global__ void __launch_bounds__(THREADS, 1)
    stream_topk_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_kc, const Params p, const SplitParams x) {
  using L = Layout<OPB>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Smem so = carve(p.n_stages, p.cap, L::Q_BYTES, L::KC_BYTES);
  uint8_t* q_s = smem + so.q;
  uint8_t* kc_s = smem + so.kc;
  uint64_t* pools = reinterpret_cast<uint64_t*>(smem + so.pool);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + so.hist);
  uint64_t* ring = reinterpret_cast<uint64_t*>(smem + so.ring);
  float* wtab = reinterpret_cast<float*>(smem + so.wtab);
  Ctrl* C = reinterpret_cast<Ctrl*>(smem + so.ctrl);
  volatile int* abort = &C->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(&C->full[s], 1);
      mbar_init(&C->empty[s], 1);
    }
    mbar_init(&C->q_full, 1);
    mbar_init(&C->q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&C->t_full[b], 1);
      mbar_init(&C->t_empty[b], N_SCORE_WARPS);
    }
    mbar_init(&C->mma_done, 1);
    for (int r = 0; r < RING; ++r) {
      mbar_init(&C->ring_full[r], N_SCORE_WARPS);
      mbar_init(&C->ring_free[r], QT);
    }
    for (int q = 0; q < QT; ++q) C->pub[q] = 0ull;
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kc);
  }
  if (warp == 1) tmem_alloc(&C->tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C->tmem_slot;

  const int n_units = p.B * (p.qt_end - p.qt_begin) * (SPLIT ? x.n_split : 1);  // work items
  const int q_bytes = L::Q_BYTES, kc_bytes = L::KC_BYTES;

  if (warp < 4) {
    regs_dec<REGS_PIPE>();
    if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0, qph = 0;
      uint32_t any_load = 0, last_par = 0;  // per stage bit: loaded at all / parity of last load
      uint32_t q_issued = 0;
      bool withheld = false;
      for (int i = 0;; ++i) {
        const int u = unit_of(i, n_units);
        if (u < 0 || *abort) break;
        const Unit U = decode_unit<SPLIT>(u, p, x);
        if (U.kt1 == U.kt0) continue;
        if (!mbar_wait_bounded(&C->q_empty, qph ^ 1u, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_QFREE);
          break;
        }
        mbar_arrive_expect_tx(&C->q_full, q_bytes);
        const int qrow = (U.b * p.S + U.t0) * HEADS;
        for (int h = 0; h < OPB; ++h)
          tma_load_2d(q_s + h * L::Q_HALF, &tm_q, &C->q_full, h * (128 / OPB), qrow);
        ++q_issued;
        qph ^= 1u;
        bool stop = false;
        for (int j = U.kt0; j < U.kt1; ++j) {
          if (!mbar_wait_bounded(&C->empty[stage], phase ^ 1u, abort, p.wait_limit_ns)) {
            record_error(p, abort, ERR_WAIT_KFREE);
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&C->full[stage], kc_bytes);
          const int krow = U.b * p.T + j * KT;
          if (p.test_withhold && !withheld && blockIdx.x == 0) {
            withheld = true;  // test hook: never deliver this tile
          } else {
            uint8_t* dst = kc_s + stage * kc_bytes;
            for (int h = 0; h < OPB; ++h)
              tma_load_2d(dst + h * L::KC_HALF, &tm_kc, &C->full[stage], h * (128 / OPB), krow);
            any_load |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == static_cast<uint32_t>(p.n_stages)) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (stop) break;
      }
      // drain: the last real load of every stage has landed before exit
      for (int s = 0; s < p.n_stages; ++s) {
        if (!((any_load >> s) & 1u)) continue;
        if (!mbar_wait_timed(&C->full[s], (last_par >> s) & 1u, p.wait_limit_ns))
          record_error(p, abort, ERR_WAIT_DRAIN);
      }
      if (q_issued && !mbar_wait_timed(&C->q_full, (q_issued - 1) & 1u, p.wait_limit_ns))
        record_error(p, abort, ERR_WAIT_DRAIN);
    } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC = OPB == 2 ? idesc_f32acc(1, 1, KT, NCOLS) : idesc_f32acc(0, 0, KT, NCOLS);
      const uint32_t q_addr = smem_u32(q_s), kc_addr = smem_u32(kc_s);
      uint32_t stage = 0, phase = 0, qph = 0, acc = 0, accph = 0;
      for (int i = 0;; ++i) {
        const int u = unit_of(i, n_units);
        if (u < 0 || *abort) break;
        const Unit U = decode_unit<SPLIT>(u, p, x);
        if (U.kt1 == U.kt0) continue;
        if (!mbar_wait_bounded(&C->q_full, qph, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_Q);
          break;
        }
        qph ^= 1u;
        tc_fence_after();
        bool stop = false;
        for (int j = U.kt0; j < U.kt1; ++j) {
          if (!mbar_wait_bounded(&C->t_empty[acc], accph ^ 1u, abort, p.wait_limit_ns)) {
            record_error(p, abort, ERR_WAIT_TMEM_EMPTY);
            stop = true;
            break;
          }
          if (!mbar_wait_bounded(&C->full[stage], phase, abort, p.wait_limit_ns)) {
            record_error(p, abort, ERR_WAIT_KC);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + acc * NCOLS;
          const uint32_t a0 = kc_addr + stage * kc_bytes;
#pragma unroll
          for (int kk = 0; kk < L::N_MMA; ++kk) {
            const uint32_t kb = kk * 32;
            const uint32_t aoff = (kb >> 7) * L::KC_HALF + (kb & 127);
            const uint32_t boff = (kb >> 7) * L::Q_HALF + (kb & 127);
            if constexpr (OPB == 2)
              mma_bf16(d_tmem, sdesc_kmajor_sw128(a0 + aoff), sdesc_kmajor_sw128(q_addr + boff), IDESC, kk > 0);
            else
              mma_f8(d_tmem, sdesc_kmajor_sw128(a0 + aoff), sdesc_kmajor_sw128(q_addr + boff), IDESC, kk > 0);
          }
          mma_commit(&C->empty[stage]);
          mma_commit(&C->t_full[acc]);
          if (j == U.kt1 - 1) mma_commit(&C->q_empty);
          if (++stage == static_cast<uint32_t>(p.n_stages)) {
            stage = 0;
            phase ^= 1u;
          }
          if (++acc == 2) {
            acc = 0;
            accph ^= 1u;
          }
        }
        if (stop) break;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(&C->mma_done);
      if (!mbar_wait_timed(&C->mma_done, 0, p.wait_limit_ns)) record_error(p, abort, ERR_WAIT_DRAIN);
    }
  } else if (warp < 8) {
    regs_dec<REGS_MGR>();
    // ------------------------------------------------------------ top-k managers
    const int q = warp - 4;   // this manager's query in the unit
    const int k = p.k;
    const int room = p.key_tile;  // appends one partition can bring
    const int tpp = p.key_tile < KT ? 1 : p.key_tile / KT;  // tiles per partition
    uint64_t* pool = pools + q * p.cap;
    uint32_t* qh = hist + q * HIST_BINS;
    topk::QState* st = &C->qs[q];
    uint32_t tix = 0;         // score tiles consumed (ring position)
    bool ok = true;
    for (int i = 0;; ++i) {
      const int u = unit_of(i, n_units);
      if (u < 0) break;
      const Unit U = decode_unit<SPLIT>(u, p, x);
      if (lane == 0) {
        st->cnt = 0;
        st->thr = 0;
        st->base = 0;
        st->shift = 0;
        st->binned = 0;
      }
      __syncwarp();
      const int t = U.t0 + q;
      int in_part = 0;
      // the running state in registers between refreshes (st holds it for them)
      uint32_t rn = 0, rbase = 0, rshift = 0;
      bool rbinned = false;
      for (int j = U.kt0; j < U.kt1; ++j, ++tix) {
        const uint32_t slot = tix & (RING - 1), par = (tix / RING) & 1u;
        if (ok && !*abort && !mbar_wait_bounded(&C->ring_full[slot], par, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_RING_FULL);
          ok = false;
        }
        ok = ok && !*abort;
        const uint64_t* area = ring + (slot * QT + q) * 4 * 32;
        if (ok && p.key_tile < KT) {
          // 64-key partitions: quadrants 0-1 hold keys 0-63 of the tile, 2-3 the rest
          topk::merge_r(rn, rbinned, rbase, rshift, pool, area, C->ring_cnt[slot][q], qh, lane, 0, 2);
          __syncwarp();
          if (lane == 0) st->cnt = rn;
          __syncwarp();
          topk::refresh(st, pool, qh, k, p.cap, room, lane);
          {
            const uint4 sv = *reinterpret_cast<const uint4*>(st);
            rn = sv.x; rbase = sv.z; rshift = sv.w; rbinned = st->binned != 0;
          }
          topk::merge_r(rn, rbinned, rbase, rshift, pool, area, C->ring_cnt[slot][q], qh, lane, 2, 4);
        } else if (ok) {
          topk::merge_r(rn, rbinned, rbase, rshift, pool, area, C->ring_cnt[slot][q], qh, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C->ring_free[slot]);  // the slot has been read
        const bool last = j == U.kt1 - 1;
        if (++in_part == tpp || last) {
          in_part = 0;
          // at the unit's end only a histogram that does not exist yet is worth
          // building (finalize selects from it); no threshold is needed any more
          __syncwarp();
          if (lane == 0) st->cnt = rn;
          __syncwarp();
          if (ok && (!last || !rbinned)) {
            topk::refresh(st, pool, qh, k, p.cap, room, lane);
            {
              const uint4 sv = *reinterpret_cast<const uint4*>(st);
              rn = sv.x; rbase = sv.z; rshift = sv.w; rbinned = st->binned != 0;
            }
            if (lane == 0)
              *reinterpret_cast<volatile uint64_t*>(&C->pub[q]) = (static_cast<uint64_t>(i) << 32) | st->thr;
          }
        }
      }
      // finalize this unit's query while the scorers move on
      if (t < p.S) {
        if (!ok && lane == 0) st->cnt = 0;  // after an abort: contents unspecified
        __syncwarp();
        if (SPLIT) {
          // this key partition's exact top-k, for the merge kernel
          const size_t pr = static_cast<size_t>(U.b) * x.part_rows + (t - p.qt_begin * QT);
          const size_t ob = (pr * x.n_split + U.sp) * static_cast<size_t>(k);
          topk::finalize(st, pool, qh, k, x.part_idx + ob, x.part_score + ob, false, lane);
        } else {
          const size_t ob = (static_cast<size_t>(U.b) * p.S + t) * static_cast<size_t>(k);
          topk::finalize(st, pool, qh, k, p.out_idx + ob, p.out_score ? p.out_score + ob : nullptr,
                         p.sort_rows != 0, lane);
        }
      }
    }
  } else {
    regs_inc<REGS_SCORE>();
    // ------------------------------------------------------------ scoring warps
    const int quad = warp & 3;        // TMEM lanes 32*quad .. 32*quad+31
    const int qp = (warp - 8) >> 2;   // this warp's queries: 2*qp (weights in registers), 2*qp+1 (table)
    const int key_off = quad * 32 + lane;  // key (within the tile) this lane scores
    float* wt = wtab + (warp - 8) * (2 * HEADS);
    const uint32_t lanemask = (1u << lane) - 1u;
    uint32_t acc = 0, accph = 0, tix = 0;
    bool ok = !*abort;
    for (int i = 0;; ++i) {
      const int u = unit_of(i, n_units);
      if (u < 0) break;
      const Unit U = decode_unit<SPLIT>(u, p, x);
      if (U.kt1 == U.kt0) continue;
      // the two queries' head weights (times the q scales for fp8) into this
      // warp's table, 0 for queries past the end of the sequence; the first
      // query's then go to registers
      __syncwarp();
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int x = r * 32 + lane;
        const int t = U.t0 + 2 * qp + (x >> 6);
        float wv = 0.f;
        if (t < p.S) {
          const size_t wi = (static_cast<size_t>(U.b) * p.S + t) * HEADS + (x & 63);
          wv = p.w[wi];
          if (OPB == 1) wv *= p.q_scale[wi];
        }
        wt[x] = wv;
      }
      __syncwarp();
      float w0[64];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = reinterpret_cast<const float4*>(wt)[c];
        w0[4 * c] = v.x;
        w0[4 * c + 1] = v.y;
        w0[4 * c + 2] = v.z;
        w0[4 * c + 3] = v.w;
      }
      int nvis[2];
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {
        const int t = U.t0 + 2 * qp + qi;
        const int n = t < p.S ? (p.row0 + t + 1) / p.m : 0;
        nvis[qi] = n < p.T ? n : p.T;
      }
      uint32_t thr0 = 0u, thr1 = 0u;
      // fp8: the key scales of the next tile are fetched one tile ahead
      const float* ks_row = OPB == 1 ? p.kc_scale + static_cast<size_t>(U.b) * p.T : nullptr;
      float ksc_next = 1.f;
      if (OPB == 1 && U.kt0 * KT + key_off < p.T) ksc_next = ks_row[U.kt0 * KT + key_off];
      for (int j = U.kt0; j < U.kt1; ++j, ++tix) {
        ok = ok && !*abort;
        if (ok && !mbar_wait_bounded(&C->t_full[acc], accph, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_TMEM_FULL);
          ok = false;
        }
        const int s = j * KT + key_off;
        uint32_t ord0 = 0u, ord1 = 0u;
        if (ok) {
          tc_fence_after();
          const uint32_t ta = tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * NCOLS + (2 * qp) * HEADS;
          const float ksc = ksc_next;
          if (OPB == 1) ksc_next = (j + 1 < U.kt1 && s + KT < p.T) ? ks_row[s + KT] : 1.f;
          {
            uint32_t x[64];
            tmem_ld32_x64(ta, x);
            tmem_ld_wait();
            ord0 = f32_ord(score_key_regs(x, w0) * ksc);
          }
          {
            uint32_t x[64];
            tmem_ld32_x64(ta + HEADS, x);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&C->t_empty[acc]);  // the logits are in registers now
            ord1 = f32_ord(score_key(x, wt + HEADS) * ksc);
          }
          // adopt the managers' latest thresholds for this unit
          const uint64_t pv0 = *reinterpret_cast<volatile uint64_t*>(&C->pub[2 * qp]);
          const uint64_t pv1 = *reinterpret_cast<volatile uint64_t*>(&C->pub[2 * qp + 1]);
          if (static_cast<int>(pv0 >> 32) == i) thr0 = max(thr0, static_cast<uint32_t>(pv0));
          if (static_cast<int>(pv1 >> 32) == i) thr1 = max(thr1, static_cast<uint32_t>(pv1));
        }
        if (++acc == 2) {
          acc = 0;
          accph ^= 1u;
        }
        // hand the tile's candidates (visible keys above the threshold) to the
        // managers: this warp's segment of the ring slot, per query
        const uint32_t slot = tix & (RING - 1), par = (tix / RING) & 1u;
        if (ok && !mbar_wait_bounded(&C->ring_free[slot], par ^ 1u, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_RING_FREE);
          ok = false;
        }
        const bool p0 = ok && s < nvis[0] && ord0 > thr0;
        const bool p1 = ok && s < nvis[1] && ord1 > thr1;
        const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, p0), b1 = __ballot_sync(0xFFFFFFFFu, p1);
        const uint32_t low = static_cast<uint32_t>(~static_cast<uint32_t>(s));
        uint64_t* seg0 = ring + ((slot * QT + 2 * qp) * 4 + quad) * 32;
        if (p0) seg0[__popc(b0 & lanemask)] = (static_cast<uint64_t>(ord0) << 32) | low;
        if (p1) seg0[4 * 32 + __popc(b1 & lanemask)] = (static_cast<uint64_t>(ord1) << 32) | low;
        if (lane == 0) {
          C->ring_cnt[slot][2 * qp][quad] = __popc(b0);
          C->ring_cnt[slot][2 * qp + 1][quad] = __popc(b1);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C->ring_full[slot]);  // release: the candidates are visible
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

bool stream_smem_plan(int k, int key_tile, int fp8, int* n_stages, int* pool_cap, size_t* bytes) {
  const int opb = fp8 ? 1 : 2;
  int np2 = 32;
  while (np2 < k) np2 <<= 1;
  const int room = key_tile;  // one partition's appends
  // the pool takes a whole partition on top of k survivors and holds the
  // padded final sort; a larger pool makes compaction rarer, which is worth
  // more than a third key-tile stage (the key tiles come from L2)
  const int cap_min = std::max(k + room, np2);
  const int cap_want = std::max(cap_min, 4 * k + room);
  const size_t q_bytes = static_cast<size_t>(NCOLS) * DIM * opb;
  const size_t kc_bytes = static_cast<size_t>(KT) * DIM * opb;
  const size_t limit = 227 * 1024;
  for (int ns = 3; ns >= 2; --ns) {
    const size_t fixed = q_bytes + ns * kc_bytes + RING_BYTES + QT * HIST_BINS * 4 + WTAB_BYTES +
                         CTRL_BYTES + 1024 /* alignment slack */;
    if (fixed >= limit) continue;
    const int cap_max = static_cast<int>((limit - fixed) / (QT * 8));
    if (cap_max < cap_min || (ns > 2 && cap_max < cap_want)) continue;
    const int cap = std::min(cap_max, cap_want);
    *n_stages = ns;
    *pool_cap = cap;
    *bytes = fixed + static_cast<size_t>(QT) * cap * 8;
    return true;
  }
  return false;
}

// Key partitions per unit for a launch of n_units units whose longest unit
// spans max_kt key tiles: when the units cannot give every SM one, each
// unit's keys are split over several CTAs (at least 4 tiles a partition, and
// at most 32768 partial entries a row, which the merge selects from quickly).
int stream_split_count(long long n_units, int max_kt, int n_sm, int k) {
  if (n_units <= 0 || n_units >= n_sm) return 1;
  const long long by_sm = n_sm / n_units;
  const long long by_len = max_kt / 4;
  const long long by_k = 32768 / k;
  const long long s = std::min(std::min(by_sm, by_len), by_k);
  return s > 1 ? static_cast<int>(s) : 1;
}

size_t stream_split_bytes_bound(int B, int S, int k, int query_chunk, int n_sm) {
  const long long rows = query_chunk > 0 ? std::min(S, query_chunk) : S;
  const long long units = static_cast<long long>(B) * ((rows + QT - 1) / QT);
  if (units >= n_sm) return 0;
  // B * part_rows * n_split <= QT * units * (n_sm / units) <= QT * n_sm
  return static_cast<size_t>(QT) * n_sm * k * 8 + 512;
}

si_status launch_stream_topk(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H, int D, int m, int k, int32_t* out_idx, float* out_score,
                             cudaStream_t stream, const StreamConfig& cfg) {
  (void)H;
  (void)D;
  int n_stages = 0, cap = 0;
  size_t smem = 0;
  if (!stream_smem_plan(k, cfg.key_tile, cfg.fp8, &n_stages, &cap, &smem))
    return fail(SI_ERR_UNSUPPORTED, "k=%d with key_tile=%d does not fit in shared memory", k, cfg.key_tile);
  const int opb = cfg.fp8 ? 1 : 2;
  const CUtensorMapDataType dt = cfg.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tm_q, tm_kc;
  const uint32_t box_inner = 128 / opb;  // 128 bytes: one swizzle row
  si_status st = encode_tmap_2d(&tm_q, dt, q, DIM, static_cast<uint64_t>(B) * S * HEADS,
                                static_cast<uint64_t>(DIM) * opb, box_inner, NCOLS);
  if (st != SI_OK) return st;
  st = encode_tmap_2d(&tm_kc, dt, kc, DIM, static_cast<uint64_t>(B) * T,
                      static_cast<uint64_t>(DIM) * opb, box_inner, KT);
  if (st != SI_OK) return st;
  int* err = cfg.err;
  if (!err) {
    st = device_error_record(&err);
    if (st != SI_OK) return st;
  }

  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");

  auto kern = cfg.fp8 ? stream_topk_kernel<1, false> : stream_topk_kernel<2, false>;
  auto kern_split = cfg.fp8 ? stream_topk_kernel<1, true> : stream_topk_kernel<2, true>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern_split, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");

  Params p;
  p.w = w;
  p.q_scale = cfg.q_scale;
  p.kc_scale = cfg.kc_scale;
  p.out_idx = out_idx;
  p.out_score = out_score;
  p.err = err;
  p.B = B;
  p.S = S;
  p.row0 = cfg.row0;
  p.T = T;
  p.m = m;
  p.k = k;
  p.key_tile = cfg.key_tile;
  p.cap = cap;
  p.n_stages = n_stages;
  p.wait_limit_ns = cfg.wait_limit_ns;
  p.test_withhold = cfg.test_withhold;
  // with scores stored, the rows are sorted afterwards by a separate pass
  // over the output; without them the managers sort before storing
  p.sort_rows = (!cfg.unsorted && out_score == nullptr) ? 1 : 0;

  // chunk driver: one persistent launch per chunk of queries; a chunk with
  // fewer units than SMs splits its units' keys over CTAs (partials in
  // scratch, then the merge kernel)
  const int n_qt_total = (S + QT - 1) / QT;
  const int chunk_qt = cfg.query_chunk > 0 ? std::max(1, cfg.query_chunk / QT) : n_qt_total;
  auto chunk_split = [&](int qt0, int qt1) {
    const int t_last = std::min(qt1 * QT, S) - 1;
    const long long n = std::min<long long>((static_cast<long long>(cfg.row0) + t_last + 1) / m, T);
    const int max_kt = static_cast<int>((n + KT - 1) / KT);
    return cfg.allow_split ? stream_split_count(static_cast<long long>(B) * (qt1 - qt0), max_kt, n_sm, k) : 1;
  };
  size_t part_bytes = 0;
  for (int qt0 = 0; qt0 < n_qt_total; qt0 += chunk_qt) {
    const int qt1 = std::min(n_qt_total, qt0 + chunk_qt);
    const int ns = chunk_split(qt0, qt1);
    if (ns > 1)
      part_bytes = std::max(part_bytes, static_cast<size_t>(B) * (qt1 - qt0) * QT * ns * k * 8 + 256);
  }
  void* part_raw = nullptr;
  uint8_t* part_base = nullptr;
  if (part_bytes) {
    if (cfg.split_ws && cfg.split_ws_bytes >= part_bytes) {
      part_base = static_cast<uint8_t*>(cfg.split_ws);
    } else {
      st = scratch_alloc(&part_raw, part_bytes, stream, "the split-key partial top-ks");
      if (st != SI_OK) return st;
      part_base = static_cast<uint8_t*>(part_raw);
    }
    part_base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(part_base) + 255) & ~static_cast<uintptr_t>(255));
  }
  bool merged_sorted = true;
  SplitParams x;
  for (int qt0 = 0; qt0 < n_qt_total && st == SI_OK; qt0 += chunk_qt) {
    p.qt_begin = qt0;
    p.qt_end = std::min(n_qt_total, qt0 + chunk_qt);
    x.n_split = chunk_split(p.qt_begin, p.qt_end);
    x.part_rows = (p.qt_end - p.qt_begin) * QT;
    const size_t part_entries = static_cast<size_t>(B) * x.part_rows * x.n_split * k;
    x.part_idx = x.n_split > 1 ? reinterpret_cast<int32_t*>(part_base) : nullptr;
    x.part_score = x.n_split > 1 ? reinterpret_cast<float*>(part_base + part_entries * 4) : nullptr;
    const long long n_work = static_cast<long long>(B) * (p.qt_end - p.qt_begin) * x.n_split;
    const int grid = static_cast<int>(std::min<long long>(n_sm, n_work));
    if (x.n_split > 1)
      kern_split<<<grid, THREADS, smem, stream>>>(tm_q, tm_kc, p, x);
    else
      kern<<<grid, THREADS, smem, stream>>>(tm_q, tm_kc, p, x);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
      st = cuda_fail(e, "stream_topk_kernel launch");
      break;
    }
    if (x.n_split > 1) {
      // the exact top-k of each row's partials, sorted, into the outputs
      const int rows = std::min(x.part_rows, S - p.qt_begin * QT);
      for (int b = 0; b < B && st == SI_OK; ++b) {
        const size_t pb = static_cast<size_t>(b) * x.part_rows * x.n_split * k;
        const size_t ob = (static_cast<size_t>(b) * S + p.qt_begin * QT) * k;
        st = launch_merge_splits(x.part_idx + pb, x.part_score + pb, rows, x.n_split, k, out_idx + ob,
                                 out_score ? out_score + ob : nullptr, stream);
      }
    } else {
      merged_sorted = false;
    }
  }
  if (part_raw) {
    e = cudaFreeAsync(part_raw, stream);
    if (e != cudaSuccess && st == SI_OK) st = cuda_fail(e, "cudaFreeAsync");
  }
  if (cfg.out_sorted) *cfg.out_sorted = st == SI_OK && merged_sorted;
  return st;
}

}  // namespace si
