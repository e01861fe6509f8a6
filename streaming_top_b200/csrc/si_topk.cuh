// Warp-level primitives of the streaming top-k: a per-query candidate pool
// of packed 64-bit keys in shared memory, an adaptive 256-bin histogram of
// the pool's scores that turns every threshold refresh into a 256-bin scan,
// compaction, exact radix select, and a register-resident bitonic sort.
//
// A packed key is (orderable fp32 score << 32) | ~index: unsigned order of
// keys = score descending, then index ascending; all keys are distinct.
#pragma once
#include <cstdint>

namespace si {
namespace topk {

constexpr int BINS = 256;

// Per-query state of the running top-k (shared memory).
struct alignas(16) QState {
  uint32_t cnt;     // entries in the pool's main region
  uint32_t thr;     // candidates must have orderable score > thr
  uint32_t base;    // histogram: bin = min(255, (ord - base) >> shift)
  uint32_t shift;
  uint32_t binned;  // histogram valid
  uint32_t pad[3];
};

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v), m);
  const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 32), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ uint32_t bin_of(uint32_t o, uint32_t base, uint32_t shift) {
  const uint32_t d = o > base ? (o - base) >> shift : 0u;
  return d < 255u ? d : 255u;
}

// Bin width so that a span of ord values covers at most 192 bins, leaving the
// top 64 bins for scores above the range seen so far.
__device__ __forceinline__ uint32_t shift_for(uint32_t span) {
  uint32_t s = 0;
  while ((span >> s) >= 192u) ++s;
  return s;
}

// hist <- histogram of the orderable scores of pool[0, n).  One warp.
// Loops over pool entries take four 32-entry chunks per step: their loads
// are all issued before any result is used, which hides shared-memory
// latency four times better than one chunk per step.
constexpr int UNR = 4;

__device__ __forceinline__ void hist_build(uint32_t* hist, const uint64_t* pool, int n,
                                           uint32_t base, uint32_t shift, int lane) {
  for (int i = lane; i < BINS; i += 32) hist[i] = 0u;
  __syncwarp();
  for (int i0 = 0; i0 < n; i0 += 32 * UNR) {
    uint32_t o[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = i0 + 32 * u + lane;
      o[u] = i < n ? static_cast<uint32_t>(pool[i] >> 32) : 0u;
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u)
      if (i0 + 32 * u + lane < n) atomicAdd(&hist[bin_of(o[u], base, shift)], 1u);
  }
  __syncwarp();
}

// The bin b at which the count of entries in bins >= b first reaches k
// (scanning from the top), or -1 when the histogram holds fewer than k.
// *above receives the count in bins > b.  Lane l reads bins [8l, 8l+8) with
// two conflict-free 16-byte loads; a suffix sum over lanes finds the lane
// holding the crossing.  One warp; the result is warp-uniform.
__device__ __forceinline__ int hist_find(const uint32_t* hist, uint32_t k, int lane,
                                         uint32_t* above) {
  const uint4 lo = reinterpret_cast<const uint4*>(hist)[2 * lane];
  const uint4 hi = reinterpret_cast<const uint4*>(hist)[2 * lane + 1];
  const uint32_t c[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) sum += c[i];
  uint32_t incl = sum;  // entries in bins >= 8*lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += v;
  }
  const uint32_t excl = incl - sum;  // entries in bins >= 8*lane + 8
  const uint32_t owners = __ballot_sync(0xFFFFFFFFu, excl < k && k <= incl);
  if (!owners) return -1;
  const int owner = __ffs(owners) - 1;
  int b = 0;
  uint32_t ab = 0;
  if (lane == owner) {
    uint32_t run = excl;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (run + c[i] >= k) {
        b = 8 * lane + i;
        ab = run;
        break;
      }
      run += c[i];
    }
  }
  *above = __shfl_sync(0xFFFFFFFFu, ab, owner);
  return __shfl_sync(0xFFFFFFFFu, b, owner);
}

// Keep the entries of pool[0, n) whose orderable score is >= thr, in place.
// (New candidates must beat thr strictly; entries already in the pool at
// exactly thr may be the k-th key and its score ties, so they stay.)
// Returns the kept count; *mx receives their largest orderable score (0 if
// none).  One warp; results are warp-uniform.
__device__ __forceinline__ int pool_compact(uint64_t* pool, int n, uint32_t thr, int lane,
                                            uint32_t* mx) {
  int kept = 0;
  uint32_t m = 0;
  const uint32_t lm = (1u << lane) - 1u;
  for (int base = 0; base < n; base += 32 * UNR) {
    uint64_t x[UNR];
    bool keep[UNR];
    uint32_t bal[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int i = base + 32 * u + lane;
      x[u] = i < n ? pool[i] : 0ull;
      keep[u] = i < n && static_cast<uint32_t>(x[u] >> 32) >= thr;
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) bal[u] = __ballot_sync(0xFFFFFFFFu, keep[u]);
    __syncwarp();  // every load of this step precedes its stores (they land at or below it)
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      if (keep[u]) {
        pool[kept + __popc(bal[u] & lm)] = x[u];
        const uint32_t o = static_cast<uint32_t>(x[u] >> 32);
        m = o > m ? o : m;
      }
      kept += __popc(bal[u]);
    }
    __syncwarp();
  }
  *mx = warp_max_u32(m);
  return kept;
}

// Keep exactly the k largest keys of pool[0, n) (n > k), in place, and
// return the orderable score of the k-th.  Radix select, most significant
// digit first, beginning below the bits all keys share; 8-bit digits.
// hist (256 words) is scratch.  One warp.
__device__ inline uint32_t pool_select(uint64_t* pool, int n, int k, uint32_t* hist, int lane) {
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
  uint32_t need = static_cast<uint32_t>(k);
  int hi = hb + 1;
  for (;;) {
    const int lo = hi > 8 ? hi - 8 : 0;
    const uint32_t dmask = (1u << (hi - lo)) - 1u;
    for (int i = lane; i < BINS; i += 32) hist[i] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint64_t x = pool[i];
      if ((x & mask) == prefix) atomicAdd(&hist[static_cast<uint32_t>(x >> lo) & dmask], 1u);
    }
    __syncwarp();
    uint32_t above = 0;
    const int d = hist_find(hist, need, lane, &above);
    const uint32_t cd = hist[d];
    need -= above;
    prefix |= static_cast<uint64_t>(d) << lo;
    mask |= static_cast<uint64_t>(dmask) << lo;
    __syncwarp();
    if (cd == need || lo == 0) break;
    hi = lo;
  }
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

// Bitonic sort of the 32*E keys held by a warp, lane l holding positions
// [l*E, l*E+E), into descending order (ascending if !desc).  Strides below E
// stay in registers; larger strides exchange with lane ^ (stride / E).
template <int E>
__device__ __forceinline__ void sort_regs(uint64_t (&v)[E], int lane, bool desc = true) {
#pragma unroll
  for (int size = 2; size <= 32 * E; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= E) {
        const int lm = stride / E;
        const bool lower = (lane & lm) == 0;
#pragma unroll
        for (int r = 0; r < E; ++r) {
          const bool d = (((lane * E + r) & size) == 0) == desc;
          const uint64_t p = shfl_xor_u64(v[r], lm);
          const uint64_t mx = v[r] > p ? v[r] : p, mn = v[r] > p ? p : v[r];
          v[r] = (lower == d) ? mx : mn;
        }
      } else {
#pragma unroll
        for (int r = 0; r < E; ++r) {
          if (r & stride) continue;
          const bool d = (((lane * E + r) & size) == 0) == desc;
          const uint64_t a = v[r], b = v[r | stride];
          if ((a < b) == d) {
            v[r] = b;
            v[r | stride] = a;
          }
        }
      }
    }
  }
}

// The last log2(32E) stages of a bitonic sort: v holds a bitonic sequence;
// leave it sorted descending (ascending if !desc).
template <int E>
__device__ __forceinline__ void merge_regs(uint64_t (&v)[E], int lane, bool desc) {
#pragma unroll
  for (int stride = 16 * E; stride > 0; stride >>= 1) {
    if (stride >= E) {
      const int lm = stride / E;
      const bool lower = (lane & lm) == 0;
#pragma unroll
      for (int r = 0; r < E; ++r) {
        const uint64_t p = shfl_xor_u64(v[r], lm);
        const uint64_t mx = v[r] > p ? v[r] : p, mn = v[r] > p ? p : v[r];
        v[r] = (lower == desc) ? mx : mn;
      }
    } else {
#pragma unroll
      for (int r = 0; r < E; ++r) {
        if (r & stride) continue;
        const uint64_t a = v[r], b = v[r | stride];
        if ((a < b) == desc) {
          v[r] = b;
          v[r | stride] = a;
        }
      }
    }
  }
}

template <int E>
__device__ __forceinline__ void pool_sort_regs(uint64_t* pool, int n, int lane) {
  uint64_t v[E];
#pragma unroll
  for (int r = 0; r < E; ++r) {
    const int i = lane * E + r;
    v[r] = i < n ? pool[i] : 0ull;
  }
  sort_regs<E>(v, lane);
  __syncwarp();
#pragma unroll
  for (int r = 0; r < E; ++r) pool[lane * E + r] = v[r];
  __syncwarp();
}

// Bitonic sort of a[0, np) (np a power of two >= 512) descending: 256-key
// chunks sort in registers, strides >= 256 run as shared-memory
// compare-exchange stages, strides < 256 again in registers chunk by chunk.
__device__ __forceinline__ void pool_sort_big(uint64_t* a, int np, int lane) {
  const int nch = np >> 8;
#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    uint64_t v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = a[c * 256 + lane * 8 + r];
    sort_regs<8>(v, lane, (c & 1) == 0);
#pragma unroll
    for (int r = 0; r < 8; ++r) a[c * 256 + lane * 8 + r] = v[r];
  }
  __syncwarp();
#pragma unroll 1
  for (int size = 512; size <= np; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride >= 256; stride >>= 1) {
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
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      uint64_t v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = a[c * 256 + lane * 8 + r];
      merge_regs<8>(v, lane, ((c * 256) & size) == 0);
#pragma unroll
      for (int r = 0; r < 8; ++r) a[c * 256 + lane * 8 + r] = v[r];
    }
    __syncwarp();
  }
}

// Sort pool[0, n) descending; entries [n, np) are overwritten with the
// sentinel 0 (np = padded power of two <= capacity).
__device__ __forceinline__ void pool_sort(uint64_t* pool, int n, int lane) {
  int np = 32;
  while (np < n) np <<= 1;
  switch (np) {
    case 32: pool_sort_regs<1>(pool, n, lane); break;
    case 64: pool_sort_regs<2>(pool, n, lane); break;
    case 128: pool_sort_regs<4>(pool, n, lane); break;
    case 256: pool_sort_regs<8>(pool, n, lane); break;
    default:
      for (int i = n + lane; i < np; i += 32) pool[i] = 0ull;
      __syncwarp();
      pool_sort_big(pool, np, lane);
  }
}

// merge_r(): move the query's candidates -- segments w_lo .. w_hi-1 of four
// 32-entry segments at `area`, segment w holding seg[w] entries -- to the end
// of its main region, counting them into the histogram once it exists.  The
// manager keeps its running state in registers between refreshes: n (the
// main region's count) is updated in place, and binned / base / shift are
// its copies of the histogram parameters.  One warp; the four segments'
// loads are in flight together.
__device__ __forceinline__ void merge_r(uint32_t& n, bool binned, uint32_t base, uint32_t shift, uint64_t* pool,
                                        const uint64_t* area, const uint32_t* seg, uint32_t* hist, int lane,
                                        int w_lo = 0, int w_hi = 4) {
  const uint4 cv = *reinterpret_cast<const uint4*>(seg);
  const uint32_t c0 = w_lo <= 0 && 0 < w_hi ? cv.x : 0u, c1 = w_lo <= 1 && 1 < w_hi ? cv.y : 0u;
  const uint32_t c2 = w_lo <= 2 && 2 < w_hi ? cv.z : 0u, c3 = w_lo <= 3 && 3 < w_hi ? cv.w : 0u;
  const uint32_t cw[4] = {c0, c1, c2, c3}, ow[4] = {0u, c0, c0 + c1, c0 + c1 + c2};
  uint64_t x[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) x[w] = static_cast<uint32_t>(lane) < cw[w] ? area[w * 32 + lane] : 0ull;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    if (static_cast<uint32_t>(lane) < cw[w]) {
      pool[n + ow[w] + lane] = x[w];
      if (binned) atomicAdd(&hist[bin_of(static_cast<uint32_t>(x[w] >> 32), base, shift)], 1u);
    }
  }
  n += c0 + c1 + c2 + c3;
}

// refresh(), at the end of a partition of keys:
//  - the first time the main region holds >= k entries, fit the histogram
//    range to them and count them;
//  - raise the threshold to just below the histogram bin in which the k-th
//    best entry lies (exact order is kept by the entries themselves);
//  - if the main region could not take another partition (`room` entries),
//    drop the entries below the threshold and zero the histogram bins below
//    it (their entries are gone; an undercounting histogram only lowers later
//    thresholds, which stays safe); refit the range when the threshold has
//    climbed past half the bins; if still too full, reduce the pool to
//    exactly k by radix select and refit.
// Invariant: every processed key that can still be in the final top-k is in
// the pool, and once thr > 0 at least k entries have orderable score >= thr.
__device__ inline void refresh(QState* st, uint64_t* pool, uint32_t* hist, int k, int cap, int room,
                        int lane) {
  int n = static_cast<int>(st->cnt);
  uint32_t thr = st->thr, base = st->base, shift = st->shift;
  bool binned = st->binned != 0;
  if (!binned && n >= k) {
    uint32_t mn = ~0u, mx = 0u;
    for (int i0 = 0; i0 < n; i0 += 32 * UNR) {
      uint32_t o[UNR];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int i = i0 + 32 * u + lane;
        o[u] = i < n ? static_cast<uint32_t>(pool[i] >> 32) : 0u;
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        if (i0 + 32 * u + lane < n) {
          mn = o[u] < mn ? o[u] : mn;
          mx = o[u] > mx ? o[u] : mx;
        }
      }
    }
    mn = warp_min_u32(mn);
    mx = warp_max_u32(mx);
    base = mn;
    shift = shift_for(mx - mn);
    hist_build(hist, pool, n, base, shift, lane);
    binned = true;
  }
  if (binned) {
    uint32_t above = 0;
    const int b = hist_find(hist, static_cast<uint32_t>(k), lane, &above);
    if (b > 0) {
      const uint32_t t = base + (static_cast<uint32_t>(b) << shift) - 1u;
      thr = t > thr ? t : thr;
    }
    if (n > cap - room) {
      uint32_t mx = 0;
      n = pool_compact(pool, n, thr, lane, &mx);
      bool rebuild = b > 128;
      if (n > cap - room) {
        thr = pool_select(pool, n, k, hist, lane);
        n = k;
        uint32_t m = 0;
        for (int i = lane; i < n; i += 32) m = max(m, static_cast<uint32_t>(pool[i] >> 32));
        mx = warp_max_u32(m);
        rebuild = true;
      }
      if (rebuild) {
        base = thr;
        shift = shift_for(mx >= base ? mx - base : 0u);
        hist_build(hist, pool, n, base, shift, lane);
      } else if (b > 0) {
        for (int i = lane; i < b; i += 32) hist[i] = 0u;
        __syncwarp();
      }
    }
  }
  __syncwarp();
  if (lane == 0) {
    st->cnt = static_cast<uint32_t>(n);
    st->thr = thr;
    st->base = base;
    st->shift = shift;
    st->binned = binned ? 1u : 0u;
  }
  __syncwarp();
}

// Final step for one query: exactly the k best pool entries, stored to
// out_idx / out_score ([k] each; -1 / -inf after the valid ones), sorted by
// (score desc, index asc) when `sort`, else in pool order (a later pass over
// the stored rows sorts them).  With a histogram, one pass keeps the entries
// of the bins above the k-th's bin and gathers that boundary bin's entries
// (into the histogram's memory, when they fit: 128 entries), a small sort
// picks the boundary keys still needed; otherwise radix select.  One warp.
__device__ inline void finalize(QState* st, uint64_t* pool, uint32_t* hist, int k, int32_t* out_idx,
                         float* out_score, bool sort, int lane) {
  int n = static_cast<int>(st->cnt);
  if (n > k) {
    bool done = false;
    if (st->binned) {
      const uint32_t base = st->base, shift = st->shift;
      uint32_t above = 0;
      const int b = hist_find(hist, static_cast<uint32_t>(k), lane, &above);
      const uint32_t nb = b >= 0 ? hist[b] : 0u;
      // The counts of the bins at and above the boundary are exact: every pool
      // entry is counted when it arrives or when the histogram is rebuilt from
      // the pool, and compaction zeroes only bins below the threshold, which
      // lies below every later boundary.  So `above` entries lie above bin b
      // and nb in it; the k - above best of those nb complete the top k.
      const int cs = static_cast<int>(above), ce = static_cast<int>(nb);
      if (b >= 0 && nb <= 128u && k - cs >= 0 && k - cs <= ce) {
        __syncwarp();
        uint64_t* scratch = reinterpret_cast<uint64_t*>(hist);
        int kept = 0, nbd = 0;
        const uint32_t lt = (1u << lane) - 1u;
        for (int b0 = 0; b0 < n; b0 += 32 * UNR) {
          uint64_t x[UNR];
          bool sure[UNR], edge[UNR];
#pragma unroll
          for (int u = 0; u < UNR; ++u) {
            const int i = b0 + 32 * u + lane;
            x[u] = i < n ? pool[i] : 0ull;
            const uint32_t bx = i < n ? bin_of(static_cast<uint32_t>(x[u] >> 32), base, shift) : 0u;
            sure[u] = i < n && bx > static_cast<uint32_t>(b);
            edge[u] = i < n && bx == static_cast<uint32_t>(b);
          }
          __syncwarp();  // every load of this step precedes its stores (they land at or below it)
#pragma unroll
          for (int u = 0; u < UNR; ++u) {
            const uint32_t bs = __ballot_sync(0xFFFFFFFFu, sure[u]);
            const uint32_t be = __ballot_sync(0xFFFFFFFFu, edge[u]);
            if (sure[u]) pool[kept + __popc(bs & lt)] = x[u];
            const int pe = nbd + __popc(be & lt);
            if (edge[u] && pe < 128) scratch[pe] = x[u];  // never past the 128-entry scratch
            kept += __popc(bs);
            nbd += __popc(be);
          }
          __syncwarp();
        }
        nbd = min(nbd, 128);
        const int need = max(0, min(k - kept, nbd));
        // sort the boundary entries (<= 128) and take the best `need`
        if (nbd <= 32) {
          uint64_t v[1] = {lane < nbd ? scratch[lane] : 0ull};
          sort_regs<1>(v, lane);
          if (lane < need) pool[kept + lane] = v[0];
        } else if (nbd <= 64) {
          uint64_t v[2];
#pragma unroll
          for (int r = 0; r < 2; ++r) v[r] = lane * 2 + r < nbd ? scratch[lane * 2 + r] : 0ull;
          sort_regs<2>(v, lane);
#pragma unroll
          for (int r = 0; r < 2; ++r)
            if (lane * 2 + r < need) pool[kept + lane * 2 + r] = v[r];
        } else {
          uint64_t v[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) v[r] = lane * 4 + r < nbd ? scratch[lane * 4 + r] : 0ull;
          sort_regs<4>(v, lane);
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (lane * 4 + r < need) pool[kept + lane * 4 + r] = v[r];
        }
        __syncwarp();
        n = kept + need;  // k, as the histogram's counts are exact
        done = true;
      }
      if (!done && n > k) {
        uint32_t mx;
        n = pool_compact(pool, n, st->thr, lane, &mx);
      }
    }
    if (!done && n > k) {
      pool_select(pool, n, k, hist, lane);
      n = k;
    }
  }
  if (sort) pool_sort(pool, n, lane);
#pragma unroll 4
  for (int x = lane; x < k; x += 32) {
    int32_t id = -1;
    float sc = -__int_as_float(0x7f800000);
    if (x < n) {
      const uint64_t key = pool[x];
      const uint32_t o = static_cast<uint32_t>(key >> 32);
      id = static_cast<int32_t>(~static_cast<uint32_t>(key));
      sc = __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
    }
    out_idx[x] = id;
    if (out_score) out_score[x] = sc;
  }
}

}  // namespace topk
}  // namespace si
