// Streaming lightning-indexer top-k for sm_100a.
//
// StreamIndex (abstract): the indexer scores compressed keys and a chunked
// partition-merge top-k keeps the per-query top-k without ever materialising
// the [B, S, H_I, T] fp32 score tensor.  Score (DeepSeek-V3.2 indexer form):
//   I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . kc[s,:]),  key s visible iff s*m+m-1 <= t.
//
// One CTA per SM (persistent).  A work unit is a tile of QT = 4 consecutive
// queries of one sequence; units are taken longest-first (the causal triangle
// makes late queries see the most keys), dealt to CTAs in snake order.
//
// Per unit:
//   warp 0 (one lane)  TMA: the unit's q tile [4 queries x 64 heads, 128]
//                      (stationary) and then key tiles [128 keys, 128]
//                      through an N-stage mbarrier ring, only the tiles
//                      that hold a visible key.
//   warp 1 (one lane)  tcgen05.mma, A = key tile (M = 128 keys), B = q tile
//                      (N = 256 = 4 queries x 64 heads), K = 128, fp32
//                      accumulator in TMEM, double buffered (2 x 256 columns)
//                      so the MMA of tile j+1 overlaps the epilogue of tile j.
//   warps 2..9         epilogue.  Thread = one key (TMEM lane), warp = 2 of
//                      the 4 queries: tcgen05.ld of 64 head logits per query,
//                      ReLU and w-weighted head sum in registers, causal mask,
//                      then the partition-merge top-k:
//                        - threshold early-reject: a key is appended to its
//                          query's candidate pool only if its score beats the
//                          k-th best score found at the last merge;
//                        - at the end of every partition of `key_tile` keys
//                          (the pages' key tile), a merge keeps exactly the k
//                          best keys of the pool (radix select on the packed
//                          key) and refreshes the threshold;
//                        - at the end of the unit the k survivors are sorted
//                          (bitonic, one warp per query) and stored.
//
// Keys are packed as (orderable fp32 score << 32) | ~index, so one unsigned
// 64-bit comparison orders by score descending, then index ascending, and
// every key is distinct.  Because key tiles are visited in index order, a new
// key whose score merely ties the threshold has a larger index than the k-th
// kept key and is correctly rejected: the filter needs the score only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "si_internal.h"
#include "si_ptx.cuh"

namespace si {
namespace {

constexpr int QT = 4;          // queries per unit
constexpr int HEADS = 64;      // indexer heads (H_I)
constexpr int DIM = 128;       // head dim (D)
constexpr int KT = 128;        // keys per MMA tile (M)
constexpr int NCOLS = QT * HEADS;  // 256 = MMA N
constexpr int THREADS = 320;   // 10 warps
constexpr int EPI_THREADS = 256;
constexpr int HIST_BINS = 256;

enum { ERR_WAIT_Q = 1, ERR_WAIT_KC = 2, ERR_WAIT_TMEM_EMPTY = 3, ERR_WAIT_TMEM_FULL = 4,
       ERR_WAIT_QFREE = 5, ERR_WAIT_KFREE = 6, ERR_WAIT_DRAIN = 7 };

struct Params {
  const float* w;         // [B,S,H]
  const float* q_scale;   // fp8: [B,S,H]
  const float* kc_scale;  // fp8: [B,T]
  int32_t* out_idx;       // [B,S,k]
  float* out_score;       // [B,S,k] or null
  int* err;               // device error record
  int B, S, T, m, k;
  int qt_begin, qt_end;   // query tiles (per sequence) of this launch
  int key_tile;           // partition length in keys (64 or multiple of 128)
  int pool_cap;           // pool entries per query
  int n_stages;
  uint64_t wait_limit_ns;
  int test_withhold;
};

struct Unit {
  int b, t0, n_keys, n_kt;
};

__device__ __forceinline__ Unit decode_unit(int u, const Params& p) {
  Unit r;
  r.b = u % p.B;
  const int qt = p.qt_end - 1 - u / p.B;
  r.t0 = qt * QT;
  const int t_last = min(r.t0 + QT, p.S) - 1;
  const int n = (t_last + 1) / p.m;
  r.n_keys = n < p.T ? n : p.T;
  r.n_kt = (r.n_keys + KT - 1) / KT;
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

__device__ __forceinline__ float ord_f32(uint32_t o) {
  const uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  return __uint_as_float(u);
}

__device__ __forceinline__ void record_error(const Params& p, volatile int* abort, int where) {
  atomicCAS(p.err, 0, static_cast<int>(SI_ERR_TIMEOUT));
  atomicCAS(p.err + 1, 0, where);
  *abort = 1;
}

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory");
}

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v), m);
  const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 32), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Merge step of the partition-merge top-k, one warp: keep exactly the k
// largest packed keys of pool[0, n) (n > k), in place, and return the
// threshold (orderable score of the k-th key).  Radix select, most
// significant digit first, starting below the bits all keys share.
__device__ uint32_t pool_shrink(uint64_t* pool, int n, int k, uint32_t* hist, int lane) {
  uint64_t vor = 0, vand = ~0ull;
  for (int i = lane; i < n; i += 32) {
    const uint64_t x = pool[i];
    vor |= x;
    vand &= x;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vor |= shfl_xor_u64(vor, o);
    vand &= shfl_xor_u64(vand, o);
  }
  const uint64_t diff = vor ^ vand;  // non-zero: keys are distinct and n >= 2
  const int hb = 63 - __clzll(static_cast<long long>(diff));
  uint64_t mask = hb == 63 ? 0ull : (~0ull << (hb + 1));
  uint64_t prefix = vand & mask;
  int need = k;
  int hi = hb + 1;
  for (;;) {
    const int lo = hi > 8 ? hi - 8 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    for (int i = lane; i < HIST_BINS; i += 32) hist[i] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint64_t x = pool[i];
      if ((x & mask) == prefix) atomicAdd(&hist[static_cast<uint32_t>(x >> lo) & dmask], 1u);
    }
    __syncwarp();
    // lane l owns digits 255-8l .. 248-8l (descending)
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = hist[255 - 8 * lane - i];
      sum += c[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - sum;
    const bool mine = excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl;
    const uint32_t owners = __ballot_sync(0xFFFFFFFFu, mine);
    const int owner = __ffs(owners) - 1;
    int d = 0;
    uint32_t above = 0, cd = 0;
    if (lane == owner) {
      uint32_t run = excl;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (run + c[i] >= static_cast<uint32_t>(need)) {
          d = 255 - 8 * lane - i;
          above = run;
          cd = c[i];
          break;
        }
        run += c[i];
      }
    }
    d = __shfl_sync(0xFFFFFFFFu, d, owner);
    above = __shfl_sync(0xFFFFFFFFu, above, owner);
    cd = __shfl_sync(0xFFFFFFFFu, cd, owner);
    need -= static_cast<int>(above);
    prefix |= static_cast<uint64_t>(d) << lo;
    mask |= static_cast<uint64_t>(dmask) << lo;
    __syncwarp();
    if (cd == static_cast<uint32_t>(need) || lo == 0) break;
    hi = lo;
  }
  // keep the keys whose leading bits are >= prefix: exactly k of them
  int kept = 0;
  uint64_t kmin = ~0ull;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const uint64_t x = i < n ? pool[i] : 0ull;
    const bool keep = i < n && (x & mask) >= prefix;
    const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
    __syncwarp();
    if (keep) {
      pool[kept + __popc(bal & ((1u << lane) - 1u))] = x;
      kmin = x < kmin ? x : kmin;
    }
    kept += __popc(bal);
    __syncwarp();
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t y = shfl_xor_u64(kmin, o);
    kmin = y < kmin ? y : kmin;
  }
  return static_cast<uint32_t>(kmin >> 32);
}

// Bitonic sort of a[0, np) into descending order, one warp (np power of two).
__device__ void warp_sort_desc(uint64_t* a, int np, int lane) {
  for (int size = 2; size <= np; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (np >> 1); i += 32) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t x = a[lo], y = a[hi];
        if ((x < y) == desc) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncwarp();
    }
  }
}

// sum_h w[h] * ReLU(L[h]) over the 64 head logits of one (key, query) pair,
// held as two 32-column TMEM loads; four partial sums for ILP.
__device__ __forceinline__ float head_sum(const uint32_t (&lo)[32], const uint32_t (&hi)[32],
                                          const float* w) {
  const float4* w4 = reinterpret_cast<const float4*>(w);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int h = 0; h < 32; h += 4) {
    const float4 ww = w4[h >> 2];
    a0 = fmaf(ww.x, fmaxf(__uint_as_float(lo[h + 0]), 0.f), a0);
    a1 = fmaf(ww.y, fmaxf(__uint_as_float(lo[h + 1]), 0.f), a1);
    a2 = fmaf(ww.z, fmaxf(__uint_as_float(lo[h + 2]), 0.f), a2);
    a3 = fmaf(ww.w, fmaxf(__uint_as_float(lo[h + 3]), 0.f), a3);
  }
#pragma unroll
  for (int h = 0; h < 32; h += 4) {
    const float4 ww = w4[8 + (h >> 2)];
    a0 = fmaf(ww.x, fmaxf(__uint_as_float(hi[h + 0]), 0.f), a0);
    a1 = fmaf(ww.y, fmaxf(__uint_as_float(hi[h + 1]), 0.f), a1);
    a2 = fmaf(ww.z, fmaxf(__uint_as_float(hi[h + 2]), 0.f), a2);
    a3 = fmaf(ww.w, fmaxf(__uint_as_float(hi[h + 3]), 0.f), a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// Shared-memory layout (offsets from a 1024-byte aligned base).
template <int OPB>
struct Layout {
  static constexpr int Q_HALF = NCOLS * 128;               // bytes per 128-byte-wide K column block of q
  static constexpr int Q_BYTES = NCOLS * DIM * OPB;        // 64 KB bf16, 32 KB fp8
  static constexpr int KC_HALF = KT * 128;
  static constexpr int KC_BYTES = KT * DIM * OPB;          // 32 KB bf16, 16 KB fp8
  static constexpr int N_MMA = DIM * OPB / 32;             // K steps of 32 bytes
};

struct Smem {
  uint32_t q, kc, pool, w, hist, ctrl;
};

__device__ __forceinline__ Smem carve(int n_stages, int pool_cap, int q_bytes, int kc_bytes) {
  Smem s;
  s.q = 0;
  s.kc = q_bytes;
  s.pool = s.kc + n_stages * kc_bytes;
  s.w = s.pool + QT * pool_cap * 8;
  s.hist = s.w + QT * HEADS * 4;
  s.ctrl = s.hist + QT * HIST_BINS * 4;
  return s;
}

template <int OPB>
__global__ void __launch_bounds__(THREADS, 1)
    stream_topk_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_kc, const Params p) {
  using L = Layout<OPB>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Smem so = carve(p.n_stages, p.pool_cap, L::Q_BYTES, L::KC_BYTES);
  uint8_t* q_s = smem + so.q;
  uint8_t* kc_s = smem + so.kc;
  uint64_t* pool = reinterpret_cast<uint64_t*>(smem + so.pool);
  float* w_s = reinterpret_cast<float*>(smem + so.w);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + so.hist);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + so.ctrl);
  uint64_t* full = bars;                        // [n_stages]
  uint64_t* empty = bars + 4;                   // [n_stages]
  uint64_t* q_full = bars + 8;
  uint64_t* q_empty = bars + 9;
  uint64_t* t_full = bars + 10;                 // [2]
  uint64_t* t_empty = bars + 12;                // [2]
  uint64_t* mma_done = bars + 14;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(bars + 16);  // [QT]
  uint32_t* thr = cnt + QT;                                // [QT]
  uint32_t* tmem_slot = thr + QT;
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], 8);  // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kc);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_units = p.B * (p.qt_end - p.qt_begin);
  const int q_bytes = L::Q_BYTES, kc_bytes = L::KC_BYTES;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, qph = 0;
      uint32_t any_load = 0, last_par = 0;  // per stage bit: loaded at all / parity of last load
      uint32_t q_issued = 0;
      bool withheld = false;
      for (int i = 0;; ++i) {
        const int u = unit_of(i, n_units);
        if (u < 0 || *abort) break;
        const Unit U = decode_unit(u, p);
        if (U.n_kt == 0) continue;
        if (!mbar_wait_bounded(q_empty, qph ^ 1u, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_QFREE);
          break;
        }
        mbar_arrive_expect_tx(q_full, q_bytes);
        const int qrow = (U.b * p.S + U.t0) * HEADS;
        for (int h = 0; h < OPB; ++h) tma_load_2d(q_s + h * L::Q_HALF, &tm_q, q_full, h * (128 / OPB), qrow);
        ++q_issued;
        qph ^= 1u;
        bool stop = false;
        for (int j = 0; j < U.n_kt; ++j) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort, p.wait_limit_ns)) {
            record_error(p, abort, ERR_WAIT_KFREE);
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kc_bytes);
          const int krow = U.b * p.T + j * KT;
          if (p.test_withhold && !withheld && blockIdx.x == 0) {
            withheld = true;  // test hook: never deliver this tile
          } else {
            uint8_t* dst = kc_s + stage * kc_bytes;
            for (int h = 0; h < OPB; ++h) tma_load_2d(dst + h * L::KC_HALF, &tm_kc, &full[stage], h * (128 / OPB), krow);
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
        if (!mbar_wait_timed(&full[s], (last_par >> s) & 1u, p.wait_limit_ns))
          record_error(p, abort, ERR_WAIT_DRAIN);
      }
      if (q_issued && !mbar_wait_timed(q_full, (q_issued - 1) & 1u, p.wait_limit_ns))
        record_error(p, abort, ERR_WAIT_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = OPB == 2 ? idesc_f32acc(1, 1, KT, NCOLS) : idesc_f32acc(0, 0, KT, NCOLS);
      const uint32_t q_addr = smem_u32(q_s), kc_addr = smem_u32(kc_s);
      uint32_t stage = 0, phase = 0, qph = 0, acc = 0, accph = 0;
      for (int i = 0;; ++i) {
        const int u = unit_of(i, n_units);
        if (u < 0 || *abort) break;
        const Unit U = decode_unit(u, p);
        if (U.n_kt == 0) continue;
        if (!mbar_wait_bounded(q_full, qph, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_Q);
          break;
        }
        qph ^= 1u;
        tc_fence_after();
        bool stop = false;
        for (int j = 0; j < U.n_kt; ++j) {
          if (!mbar_wait_bounded(&t_empty[acc], accph ^ 1u, abort, p.wait_limit_ns)) {
            record_error(p, abort, ERR_WAIT_TMEM_EMPTY);
            stop = true;
            break;
          }
          if (!mbar_wait_bounded(&full[stage], phase, abort, p.wait_limit_ns)) {
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
          mma_commit(&empty[stage]);
          mma_commit(&t_full[acc]);
          if (j == U.n_kt - 1) mma_commit(q_empty);
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
      mma_commit(mma_done);
      if (!mbar_wait_timed(mma_done, 0, p.wait_limit_ns)) record_error(p, abort, ERR_WAIT_DRAIN);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int etid = threadIdx.x - 64;  // 0..255
    const int ew = warp - 2;            // 0..7
    const int quad = warp & 3;          // TMEM lanes 32*quad .. 32*quad+31
    const int qp = ew >> 2;             // this warp's queries: 2*qp, 2*qp+1
    const int k = p.k;
    const bool half_parts = p.key_tile < KT;
    const int part_tiles = half_parts ? 1 : p.key_tile / KT;
    uint32_t acc = 0, accph = 0;
    for (int i = 0;; ++i) {
      const int u = unit_of(i, n_units);
      if (u < 0) break;
      const Unit U = decode_unit(u, p);
      const bool live = !*abort;
      {
        const int q = etid >> 6, h = etid & 63, t = U.t0 + q;
        float wv = 0.f;
        if (t < p.S) {
          const size_t wi = (static_cast<size_t>(U.b) * p.S + t) * HEADS + h;
          wv = p.w[wi];
          if (OPB == 1) wv *= p.q_scale[wi];
        }
        w_s[q * HEADS + h] = wv;
        if (etid < QT) {
          cnt[etid] = 0;
          thr[etid] = 0;
        }
      }
      int nvis[2];
#pragma unroll
      for (int qi = 0; qi < 2; ++qi) {
        const int t = U.t0 + 2 * qp + qi;
        const int n = t < p.S ? (t + 1) / p.m : 0;
        nvis[qi] = n < p.T ? n : p.T;
      }
      epi_sync();
      for (int j = 0; j < U.n_kt; ++j) {
        bool ok = live && !*abort;
        if (ok && !mbar_wait_bounded(&t_full[acc], accph, abort, p.wait_limit_ns)) {
          record_error(p, abort, ERR_WAIT_TMEM_FULL);
          ok = false;
        }
        const int s = j * KT + quad * 32 + lane;
        uint64_t key[2] = {0ull, 0ull};
        bool pass[2] = {false, false};
        if (ok) {
          tc_fence_after();
          const uint32_t ta =
              tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * NCOLS + (2 * qp) * HEADS;
          float ksc = 1.f;
          if (OPB == 1 && s < p.T) ksc = p.kc_scale[static_cast<size_t>(U.b) * p.T + s];
          float sc[2];
#pragma unroll
          for (int qi = 0; qi < 2; ++qi) {
            uint32_t v0[32], v1[32];
            tmem_ld32(ta + qi * HEADS, v0);
            tmem_ld32(ta + qi * HEADS + 32, v1);
            tmem_ld_wait();
            sc[qi] = head_sum(v0, v1, w_s + (2 * qp + qi) * HEADS) * ksc;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&t_empty[acc]);  // accumulator may be overwritten now
          const float s0 = sc[0], s1 = sc[1];
          key[0] = (static_cast<uint64_t>(f32_ord(s0)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(s));
          key[1] = (static_cast<uint64_t>(f32_ord(s1)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(s));
          pass[0] = s < nvis[0];
          pass[1] = s < nvis[1];
        }
        if (++acc == 2) {
          acc = 0;
          accph ^= 1u;
        }
        // append survivors of the threshold; with 64-key partitions the two
        // halves of the tile are separate partitions (merge in between)
        const int n_phase = half_parts ? 2 : 1;
        for (int ph = 0; ph < n_phase; ++ph) {
          const bool mine = !half_parts || (quad >> 1) == ph;
          if (mine) {
#pragma unroll
            for (int qi = 0; qi < 2; ++qi) {
              const int q = 2 * qp + qi;
              const bool pq = pass[qi] && static_cast<uint32_t>(key[qi] >> 32) > thr[q];
              const uint32_t bal = __ballot_sync(0xFFFFFFFFu, pq);
              if (bal) {
                uint32_t base = 0;
                if (lane == 0) base = atomicAdd(&cnt[q], static_cast<uint32_t>(__popc(bal)));
                base = __shfl_sync(0xFFFFFFFFu, base, 0);
                if (pq) pool[q * p.pool_cap + base + __popc(bal & ((1u << lane) - 1u))] = key[qi];
              }
            }
          }
          const bool part_end = half_parts || ((j + 1) % part_tiles == 0) || (j == U.n_kt - 1);
          if (part_end) {
            epi_sync();
            if (ew < QT && static_cast<int>(cnt[ew]) > k) {
              thr[ew] = pool_shrink(pool + ew * p.pool_cap, cnt[ew], k, hist + ew * HIST_BINS, lane);
              __syncwarp();
              if (lane == 0) cnt[ew] = k;
            }
            epi_sync();
          }
        }
      }
      // finalize: sort the <= k survivors of each query and store them
      if (ew < QT) {
        const int t = U.t0 + ew;
        if (t < p.S) {
          uint64_t* pl = pool + ew * p.pool_cap;
          const int n = static_cast<int>(cnt[ew]);
          int np = 32;
          while (np < n) np <<= 1;
          for (int x = n + lane; x < np; x += 32) pl[x] = 0ull;
          __syncwarp();
          warp_sort_desc(pl, np, lane);
          const size_t ob = (static_cast<size_t>(U.b) * p.S + t) * static_cast<size_t>(k);
          for (int x = lane; x < k; x += 32) {
            int32_t id = -1;
            float sc = -__int_as_float(0x7f800000);
            if (x < n) {
              const uint64_t key = pl[x];
              id = static_cast<int32_t>(~static_cast<uint32_t>(key));
              sc = ord_f32(static_cast<uint32_t>(key >> 32));
            }
            p.out_idx[ob + x] = id;
            if (p.out_score) p.out_score[ob + x] = sc;
          }
        }
      }
      epi_sync();
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
  const int cap = std::max(k + key_tile, np2);
  const size_t q_bytes = static_cast<size_t>(NCOLS) * DIM * opb;
  const size_t kc_bytes = static_cast<size_t>(KT) * DIM * opb;
  const size_t fixed = q_bytes + static_cast<size_t>(QT) * cap * 8 + QT * HEADS * 4 +
                       QT * HIST_BINS * 4 + 256 + 1024 /* alignment slack */;
  const size_t limit = 227 * 1024;
  for (int ns = 4; ns >= 2; --ns) {
    const size_t tot = fixed + ns * kc_bytes;
    if (tot <= limit) {
      *n_stages = ns;
      *pool_cap = cap;
      *bytes = tot;
      return true;
    }
  }
  return false;
}

si_status launch_stream_topk(const void* q, const void* kc, const float* w, int B, int S, int T,
                             int H, int D, int m, int k, int32_t* out_idx, float* out_score,
                             cudaStream_t stream, const StreamConfig& cfg) {
  (void)H;
  (void)D;
  int n_stages = 0, pool_cap = 0;
  size_t smem = 0;
  if (!stream_smem_plan(k, cfg.key_tile, cfg.fp8, &n_stages, &pool_cap, &smem))
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
  int* err = nullptr;
  st = device_error_record(&err);
  if (st != SI_OK) return st;

  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");

  auto kern = cfg.fp8 ? stream_topk_kernel<1> : stream_topk_kernel<2>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
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
  p.T = T;
  p.m = m;
  p.k = k;
  p.key_tile = cfg.key_tile;
  p.pool_cap = pool_cap;
  p.n_stages = n_stages;
  p.wait_limit_ns = cfg.wait_limit_ns;
  p.test_withhold = cfg.test_withhold;

  // chunk driver: one persistent launch per chunk of queries
  const int n_qt_total = (S + QT - 1) / QT;
  const int chunk_qt = cfg.query_chunk > 0 ? std::max(1, cfg.query_chunk / QT) : n_qt_total;
  for (int qt0 = 0; qt0 < n_qt_total; qt0 += chunk_qt) {
    p.qt_begin = qt0;
    p.qt_end = std::min(n_qt_total, qt0 + chunk_qt);
    const long long n_units = static_cast<long long>(B) * (p.qt_end - p.qt_begin);
    const int grid = static_cast<int>(std::min<long long>(n_sm, n_units));
    kern<<<grid, THREADS, smem, stream>>>(tm_q, tm_kc, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "stream_topk_kernel launch");
  }
  return SI_OK;
}

}  // namespace si
