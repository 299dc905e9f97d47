// Many-row path: one persistent CTA per SM, three warp roles.
//
//   producer (1 warp, one lane)  : cp.async.bulk copies of the CTA's rows, in
//                                  32 KB stages, into a 3-stage shared ring
//                                  (full / empty mbarriers).
//   filter   (8 warps)           : every stage, each lane compares its 32
//                                  values with the row's running threshold t
//                                  (keep x unless x < t; NaN always kept); the
//                                  warps meet at one barrier per stage to place
//                                  the survivors' (key, index) pairs in a
//                                  shared candidate buffer. Once m candidates
//                                  at or above t are held, t becomes strict (a
//                                  later equal value has a larger index, so it
//                                  loses its tie). When the buffer passes half
//                                  full it is compacted: an approximate radix
//                                  cut when one suffices, else an exact select
//                                  with the tie cut by index. At the end of the
//                                  row the candidates are handed over.
//   finisher (6 warps)           : ranks the handed-over candidates by (key
//                                  descending, index ascending) with bucket
//                                  passes over a composite key (a bitonic sort
//                                  when a bucket stays crowded with equal
//                                  keys), then writes the first m indices and
//                                  -1 padding while the filter warps already
//                                  stream the next row.
//
// A row starts with a speculative threshold: from the row the finisher
// completed two rows earlier (half the gap between that row's 3k/4-th and
// k-th largest below its k-th), else from the bound the filter held on its
// previous row, else from a sample of the row itself. If fewer than m values
// pass it, the filter warps re-read the row from global memory with no
// threshold; the result is exact either way, only the time changes.
//
// The selection follows the pages' histogram / cumulative-sum / threshold /
// gt-eq split (SGLang PR #34167 code excerpt, the radix top-k kernel), made
// exact: ties at the threshold go to the lowest indices (a second radix select
// over the indices of the tied keys) instead of a capped tie list.
namespace rows {

constexpr int kFilterWarps = 8;
constexpr int kFilterThreads = kFilterWarps * 32;  // 256
constexpr int kFinishWarps = 6;
constexpr int kFinishThreads = kFinishWarps * 32;  // 192
constexpr int kProducerWarp = kFilterWarps + kFinishWarps;
constexpr int kThreads = (kProducerWarp + 1) * 32;  // 480
constexpr int kGroups = 8;                              // float4 groups per lane and stage
constexpr int kVals = 4 * kGroups;                      // 32 values per lane and stage
constexpr int kWarpElems = 32 * kVals;                  // 1024 per warp and stage
constexpr int kStageElems = kFilterWarps * kWarpElems;  // 8192
constexpr uint32_t kStageBytes = kStageElems * 4;       // 32 KB
constexpr int kStages = 3;                              // 96 KB ring
constexpr int kFiltCap = 8192;                          // candidate buffer entries
constexpr int kTrigger = kFiltCap / 2;                  // compact after a stage that leaves more
constexpr int kHandCap = 4096;                          // handed-over candidates, at most
constexpr int kBuckets = 3840;                          // finisher bucket counters (20 per thread)
constexpr int kPerThread = (kFiltCap + kFilterThreads - 1) / kFilterThreads;  // entries per filter thread
constexpr int kScanPer = kBuckets / kFinishThreads;     // 32 counters per finisher thread
constexpr uint32_t kInfKey = 0xFF800000u;               // key of +inf
constexpr int kRounds = 4;                              // radix rounds of 8 bits
constexpr int kKeepLimit = 2560;                        // approximate compaction keeps at most this many
constexpr int kSampleChunks = kFilterWarps * kGroups;   // runs of 128 sampled for a row's first threshold
constexpr int64_t kSampleMinLen = 4 * kStageElems;      // shorter rows start with no threshold
constexpr int kBigBucket = 64;                          // finisher: larger buckets are sorted instead
constexpr int kSmallBucket = 16;                        // finisher: largest bucket ranked by direct counting
constexpr int kSortPasses = 3;                          // finisher: bucket count passes, at most

static_assert(kVals <= 32, "a lane's survivors of one stage form a 32-bit mask");
static_assert(kFiltCap - kTrigger >= kStageElems / 2, "half a stage fits after a compaction");
static_assert(kFilterWarps % 2 == 0 && kKeepLimit + kStageElems / 2 <= kFiltCap, "split halves fit after a compaction");
static_assert(kHandCap >= kMaxK && kTrigger >= kMaxK, "buffers must hold k entries");
static_assert(kBuckets >= 2048, "bucket_shift narrows a 12-bit slice by at most one more bit");
static_assert(kBuckets == kScanPer * kFinishThreads && kBuckets <= 4096 && kScanPer % 4 == 0,
              "bucket counters split evenly over the finisher threads");

struct __align__(128) Smem {
  float ring[kStages][kStageElems];
  uint32_t fkey[kFiltCap];  // filter candidates
  uint32_t fidx[kFiltCap];
  uint32_t hkey[kHandCap];  // handed over to the finishers
  uint32_t hidx[kHandCap];
  uint32_t bcnt[kBuckets];  // finisher bucket counters / ends
  uint16_t perm[kHandCap];  // finisher: candidates grouped by bucket
  int32_t ostage[kMaxK];    // finisher: the row's output, written out coalesced
  uint32_t hist[256];       // filter radix histogram
  uint4 red[2][(kFilterWarps + 3) / 4];  // per-warp survivor counts, by stage parity
  uint32_t fred[4][kFilterWarps];
  uint32_t nred[5][kFinishWarps];
  uint32_t bc[8];
  uint32_t small[32];
  uint32_t rec[2];  // finisher: keys at ranks k-1 and 3k/4-1
  // handover (filter -> finisher)
  int64_t h_row, h_len;
  int32_t h_n, h_m;
  // speculative threshold (finisher -> filter), by handover parity
  int64_t est_len[2];
  float est[2];
  int32_t est_ok[2];
  // the filter warps' own estimate: an earlier row of length own_len held at
  // least k candidates with key >= own_key (own_len 0: none yet)
  uint32_t own_key;
  int32_t own_len;
  unsigned long long full[kStages], empty[kStages];
  unsigned long long hfull, hempty;
};
static_assert(sizeof(Smem) <= 232448, "shared memory budget of one CTA per SM");

__device__ __forceinline__ void bar_filter() { asm volatile("bar.sync 1, %0;" ::"n"(kFilterThreads) : "memory"); }
__device__ __forceinline__ void bar_finish() { asm volatile("bar.sync 2, %0;" ::"n"(kFinishThreads) : "memory"); }

// Warp sum by shuffles (the per-stage path avoids redux.sync, whose
// throughput is far lower than that of shuffles).
__device__ __forceinline__ uint32_t warp_sum(uint32_t x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
  return x;
}

// Smallest float threshold t with (!(x < t)) == (key(x) > T) for every non-NaN x.
// T at or above +inf's key has no such float: +inf is returned, which also
// keeps +inf itself (a superset, harmless: the final ranking is exact).
__device__ __forceinline__ float above(uint32_t T) {
  return T < kInfKey ? from_key(T + 1u) : __int_as_float(0x7f800000);
}

// The 16-byte aligned byte span covering row entries [0, L).
struct RowSpan {
  const char* src;
  int64_t j0;           // row index of the span's first float (-3..0)
  int nst;              // 16 KB stages
  uint32_t last_bytes;  // bytes of the last stage
};

__device__ __forceinline__ RowSpan row_span(const float* row, int64_t L) {
  RowSpan sp;
  const uintptr_t a = reinterpret_cast<uintptr_t>(row);
  const uintptr_t as = a & ~static_cast<uintptr_t>(15);
  sp.src = reinterpret_cast<const char*>(as);
  sp.j0 = -static_cast<int64_t>((a - as) >> 2);
  if (L <= 0) {
    sp.nst = 0;
    sp.last_bytes = 0;
    return sp;
  }
  const uintptr_t ee = (reinterpret_cast<uintptr_t>(row + L) + 15) & ~static_cast<uintptr_t>(15);
  const uint64_t bytes = ee - as;
  sp.nst = static_cast<int>((bytes + kStageBytes - 1) / kStageBytes);
  sp.last_bytes = static_cast<uint32_t>(bytes - static_cast<uint64_t>(sp.nst - 1) * kStageBytes);
  return sp;
}

// ------------------------------------------------------------ filter warps
// Position of value j (0..15) of a lane inside its stage: float4 group j/4 at
// warp*kWarpElems + (j/4)*128 + lane*4 (conflict-free 128-bit shared loads).
__device__ __forceinline__ int val_offset(int w, int lane, int j) {
  return w * kWarpElems + (j >> 2) * 128 + lane * 4 + (j & 3);
}

__device__ __forceinline__ uint32_t pass_mask(const float (&v)[kVals], float t) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < kVals; ++j) m |= static_cast<uint32_t>(!(v[j] < t)) << j;
  return m;
}

// Stage-local offsets [lo, hi) of a stage whose first float has row index
// sj0 that hold row indices in [0, L).
__device__ __forceinline__ void stage_bounds(int64_t sj0, int64_t L, int& lo, int& hi) {
  const int64_t a = -sj0, b = L - sj0;
  lo = static_cast<int>(a < 0 ? 0 : (a > kStageElems ? kStageElems : a));
  hi = static_cast<int>(b < 0 ? 0 : (b > kStageElems ? kStageElems : b));
}

// Bits of this lane's values whose stage offset lies in [lo, hi).
__device__ __forceinline__ uint32_t range_mask(int w, int lane, int lo, int hi) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < kVals; ++j) {
    const int o = val_offset(w, lane, j);
    m |= static_cast<uint32_t>(o >= lo && o < hi) << j;
  }
  return m;
}

// min / max of v(e) over candidates [0, n) with pred(e) (filter threads).
template <class V, class P>
__device__ void filter_minmax(Smem& s, int n, V v, P pred, uint32_t& lo, uint32_t& hi, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int e = tid; e < n; e += kFilterThreads) {
    if (!pred(e)) continue;
    const uint32_t x = v(e);
    mn = min(mn, x);
    mx = max(mx, x);
  }
  mn = __reduce_min_sync(kFull, mn);
  mx = __reduce_max_sync(kFull, mx);
  if (lane == 0) {
    s.fred[0][w] = mn;
    s.fred[1][w] = mx;
  }
  bar_filter();
  lo = __reduce_min_sync(kFull, lane < kFilterWarps ? s.fred[0][lane] : 0xFFFFFFFFu);
  hi = __reduce_max_sync(kFull, lane < kFilterWarps ? s.fred[1][lane] : 0u);
  bar_filter();
}

// need-th largest of v(e) over the candidates with pred(e) (1 <= need <= their
// number). Radix rounds over 8-bit windows below the highest bit where the
// bounds differ; a bucket of <= 32 values is finished by one warp.
template <class V, class P>
__device__ uint32_t filter_kth(Smem& s, int n, uint32_t need, V v, P pred, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t lo, hi;
  filter_minmax(s, n, v, pred, lo, hi, tid);
  for (int round = 0; lo != hi; ++round) {
    if (round == kRounds) {  // unreachable for a consistent histogram
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    const int sh = window_shift(lo, hi);
    for (int i = tid; i < 256; i += kFilterThreads) s.hist[i] = 0u;
    if (tid == 0) {
      s.bc[0] = 0xFFFFFFFFu;
      s.bc[2] = 0u;
    }
    bar_filter();
    uint32_t cur = 0xFFFFFFFFu, run = 0;
    for (int e = tid; e < n; e += kFilterThreads) {
      if (!pred(e)) continue;
      const uint32_t x = v(e);
      if (x < lo || x > hi) continue;
      const uint32_t d = (x >> sh) & 255u;
      if (d != cur) {
        if (run) atomicAdd(&s.hist[cur], run);
        cur = d;
        run = 0;
      }
      ++run;
    }
    if (run) atomicAdd(&s.hist[cur], run);
    bar_filter();
    if (w == 0) find_bucket_warp0(s.hist, need, s.bc, lane);
    bar_filter();
    const uint32_t bsel = s.bc[0], above_b = s.bc[1];
    if (bsel == 0xFFFFFFFFu) {
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    const uint32_t in_bucket = s.hist[bsel];
    need -= above_b;
    narrow(lo, hi, sh, bsel);
    if (in_bucket <= 32u && lo != hi) {
      for (int e = tid; e < n; e += kFilterThreads) {
        if (!pred(e)) continue;
        const uint32_t x = v(e);
        if (x >= lo && x <= hi) {
          const uint32_t slot = atomicAdd(&s.bc[2], 1u);
          if (slot < 32u) s.small[slot] = x;
        }
      }
      bar_filter();
      if (w == 0) {
        const uint32_t t = small_kth(lane < static_cast<int>(in_bucket) ? s.small[lane] : 0u, need);
        if (lane == 0) s.bc[3] = t;
      }
      bar_filter();
      lo = hi = s.bc[3];
    }
    bar_filter();
  }
  return lo;
}

struct FKey {
  const Smem* s;
  __device__ uint32_t operator()(int e) const { return s->fkey[e]; }
};
struct FNotIdx {  // larger value = smaller index
  const Smem* s;
  __device__ uint32_t operator()(int e) const { return ~s->fidx[e]; }
};
struct FAll {
  __device__ bool operator()(int) const { return true; }
};
struct FKeyIs {
  const Smem* s;
  uint32_t T;
  __device__ bool operator()(int e) const { return s->fkey[e] == T; }
};

// Keeps, in place and in any order, the candidates with key > A and, when
// kTies, those with key == A and index <= I. Every filter thread reads its
// entries before any is written. Returns the kept count (uniform).
template <bool kTies>
__device__ uint32_t keep_pass(Smem& s, int n, uint32_t A, uint32_t I, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t kk[kPerThread], ii[kPerThread], keep = 0;
#pragma unroll
  for (int it = 0; it < kPerThread; ++it) {
    const int e = it * kFilterThreads + tid;
    kk[it] = 0u;
    ii[it] = 0u;
    if (e < n) {
      kk[it] = s.fkey[e];
      ii[it] = s.fidx[e];
    }
    const bool kp = e < n && (kk[it] > A || (kTies && kk[it] == A && ii[it] <= I));
    keep |= static_cast<uint32_t>(kp) << it;
  }
  const uint32_t nk = __popc(keep);
  uint32_t incl = nk;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s.fred[0][w] = incl;
  bar_filter();
  uint32_t pos = incl - nk, total = 0;
#pragma unroll
  for (int ww = 0; ww < kFilterWarps; ++ww) {
    const uint32_t c = s.fred[0][ww];
    pos += ww < w ? c : 0u;
    total += c;
  }
#pragma unroll
  for (int it = 0; it < kPerThread; ++it) {
    if ((keep >> it) & 1u) {
      s.fkey[pos] = kk[it];
      s.fidx[pos] = ii[it];
      ++pos;
    }
  }
  bar_filter();
  return total;
}

// Exact: keeps the top m of candidates [0, n) by (key descending, index
// ascending), n > m >= 1. Returns the m-th largest key.
__device__ __noinline__ uint32_t compact_exact(Smem& s, int n, int m, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  bar_filter();  // every append is visible
  const uint32_t T = filter_kth(s, n, static_cast<uint32_t>(m), FKey{&s}, FAll{}, tid);
  uint32_t ngt = 0, neq = 0;
  for (int e = tid; e < n; e += kFilterThreads) {
    const uint32_t key = s.fkey[e];
    ngt += key > T;
    neq += key == T;
  }
  ngt = __reduce_add_sync(kFull, ngt);
  neq = __reduce_add_sync(kFull, neq);
  if (lane == 0) {
    s.fred[2][w] = ngt;
    s.fred[3][w] = neq;
  }
  bar_filter();
  ngt = __reduce_add_sync(kFull, lane < kFilterWarps ? s.fred[2][lane] : 0u);
  neq = __reduce_add_sync(kFull, lane < kFilterWarps ? s.fred[3][lane] : 0u);
  bar_filter();
  const uint32_t need = static_cast<uint32_t>(m) - ngt;  // entries equal to T that stay
  uint32_t I = 0xFFFFFFFFu;                               // largest index of a kept tie
  if (neq > need) I = ~filter_kth(s, n, need, FNotIdx{&s}, FKeyIs{&s, T}, tid);
  keep_pass<true>(s, n, T, I, tid);
  return T;
}

// Approximate: narrows the radix bucket holding the m-th largest key until
// every key at or above the bucket's lower end fits in kKeepLimit entries,
// then keeps exactly those (a superset of the top m). Returns false, having
// changed nothing, when that needs more than kRounds rounds or the bucket is
// one tied key with too many entries: the exact pass must run.
struct FastCut {
  uint32_t ok, lo, kept;
};

__device__ __noinline__ FastCut compact_fast(Smem& s, int n, int m, int tid) {
  uint32_t kept = 0;
  const int w = tid >> 5, lane = tid & 31;
  bar_filter();  // every append is visible
  uint32_t lo, hi;
  filter_minmax(s, n, FKey{&s}, FAll{}, lo, hi, tid);
  uint32_t need = static_cast<uint32_t>(m), above = 0;
  bool ok = false;
  for (int round = 0; round < kRounds && lo != hi; ++round) {
    const int sh = window_shift(lo, hi);
    for (int i = tid; i < 256; i += kFilterThreads) s.hist[i] = 0u;
    if (tid == 0) s.bc[0] = 0xFFFFFFFFu;
    bar_filter();
    uint32_t cur = 0xFFFFFFFFu, run = 0;
    for (int e = tid; e < n; e += kFilterThreads) {
      const uint32_t x = s.fkey[e];
      if (x < lo || x > hi) continue;
      const uint32_t d = (x >> sh) & 255u;
      if (d != cur) {
        if (run) atomicAdd(&s.hist[cur], run);
        cur = d;
        run = 0;
      }
      ++run;
    }
    if (run) atomicAdd(&s.hist[cur], run);
    bar_filter();
    if (w == 0) find_bucket_warp0(s.hist, need, s.bc, lane);
    bar_filter();
    const uint32_t bsel = s.bc[0];
    const uint32_t above_b = s.bc[1];
    const uint32_t in_b = bsel == 0xFFFFFFFFu ? 0u : s.hist[bsel];
    bar_filter();  // hist and bc are rewritten by the next round
    if (bsel == 0xFFFFFFFFu) {
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    above += above_b;
    need -= above_b;
    narrow(lo, hi, sh, bsel);
    if (above + in_b <= static_cast<uint32_t>(kKeepLimit)) {
      ok = true;
      kept = above + in_b;
      break;
    }
  }
  if (!ok) return FastCut{0u, 0u, 0u};
  keep_pass<false>(s, n, lo - 1u, 0u, tid);  // key >= lo (every real key is >= 1)
  return FastCut{1u, lo, kept};
}

struct Filter {
  uint32_t cnt;       // candidates held (the same in every filter thread)
  float t;            // keep x unless x < t
  int par;            // stage parity of s.red on the synchronous path
  bool compacted;     // the row was compacted at least once
  bool strict;        // t already excludes values equal to the held m-th key
  bool bounded;       // last_key is set
  uint32_t last_key;  // at least m candidates with key >= last_key are held
};

// Holding at least m candidates, every one at or above the threshold t: a
// later value equal to t has a larger index than all of them and cannot enter
// the top m, so the threshold becomes strict (rows of tied values then stop
// filling the buffer).
__device__ __forceinline__ void tighten(Filter& f, int m) {
  if (!f.strict && m > 0 && f.cnt >= static_cast<uint32_t>(m)) {
    f.last_key = to_key(f.t);
    f.bounded = true;
    f.t = above(f.last_key);
    f.strict = true;
  }
}

// Bounds the buffer again: the approximate pass, else the exact one.
__device__ __forceinline__ void compact_any(Smem& s, Filter& f, int m, int tid) {
  const FastCut c = compact_fast(s, static_cast<int>(f.cnt), m, tid);
  if (c.ok) {
    f.cnt = c.kept;
    f.t = c.lo > kInfKey ? __int_as_float(0x7f800000) : from_key(c.lo);
    f.last_key = c.lo;
    f.bounded = true;
    f.strict = false;
    tighten(f, m);
  } else {
    const uint32_t T = compact_exact(s, static_cast<int>(f.cnt), m, tid);
    f.cnt = static_cast<uint32_t>(m);
    f.t = above(T);
    f.last_key = T;
    f.bounded = true;
    f.strict = true;
  }
  f.compacted = true;
}

// Writes this warp's survivors (bit j of msk: value j of the lane; values
// re-read from src, the stage in the ring or in global memory) at positions
// pos.., up to two survivors per lane and round.
template <bool kRing>
__device__ __forceinline__ void put_survivors(Smem& s, const float* src, uint32_t msk, uint32_t idx0, uint32_t pos,
                                              int w, int lane) {
  const uint32_t lt = lanemask_lt();
  uint32_t rest = msk;
  for (;;) {  // two survivors per lane and iteration: their loads overlap
    const bool a1 = rest != 0u;
    const uint32_t b1 = __ballot_sync(kFull, a1);
    if (b1 == 0u) break;
    const int j1 = __ffs(rest) - 1;
    rest &= rest - 1u;
    const bool a2 = rest != 0u;
    const uint32_t b2 = __ballot_sync(kFull, a2);
    const int j2 = __ffs(rest) - 1;
    rest &= rest - 1u;
    const uint32_t n1 = __popc(b1);
    const int o1 = val_offset(w, lane, j1 & 31), o2 = val_offset(w, lane, j2 & 31);
    float x1 = 0.f, x2 = 0.f;
    if (a1) x1 = kRing ? src[o1] : __ldg(src + o1);
    if (a2) x2 = kRing ? src[o2] : __ldg(src + o2);
    if (a1) {
      const uint32_t p = pos + __popc(b1 & lt);
      s.fkey[p] = to_key(x1);
      s.fidx[p] = idx0 + static_cast<uint32_t>(o1);
    }
    if (a2) {
      const uint32_t p = pos + n1 + __popc(b2 & lt);
      s.fkey[p] = to_key(x2);
      s.fidx[p] = idx0 + static_cast<uint32_t>(o2);
    }
    pos += n1 + __popc(b2);
  }
}

// A stage whose survivors do not fit behind the buffer's contents (rare: no
// usable threshold yet, or values rising along the row): the warps write in
// two halves, compacting first whenever a half would not fit. A half
// with more than the free space implies more than kTrigger >= m entries held,
// so the compaction applies; afterwards a half (<= kStageElems / 2) fits. Masks
// taken before a compaction are supersets of the current ones, which is
// harmless: the final ranking is exact.
// (Rare paths take and return the filter state by value so that it never has
// an address and stays in registers in the hot loop. This one and the re-read
// below are inlined: a real call inside the row loop made the compiler keep
// loop state in local memory, reloaded on every stage; inlining them took
// about a tenth off a 4096-row launch.)
template <bool kRing>
__device__ __forceinline__ Filter take_stage_split(Smem& s, Filter f, const uint32_t* red, const float* src, uint32_t msk,
                                              uint32_t idx0, int m, int tid) {
  constexpr int kHalf = kFilterWarps / 2;
  const int w = tid >> 5, lane = tid & 31;
  for (int half = 0; half < 2; ++half) {
    uint32_t tot = 0, before = 0;
#pragma unroll
    for (int i = 0; i < kHalf; ++i) {
      const int ww = kHalf * half + i;
      const uint32_t c = red[ww];
      tot += c;
      before += ww < w ? c : 0u;
    }
    if (f.cnt + tot > static_cast<uint32_t>(kFiltCap)) compact_any(s, f, m, tid);
    if (w / kHalf == half) put_survivors<kRing>(s, src, msk, idx0, f.cnt + before, w, lane);
    f.cnt += tot;
    bar_filter();  // this half's entries are visible to a following compaction
  }
  return f;
}

// Takes one stage after the filter barrier that completed its per-warp counts.
template <bool kRing>
__device__ __forceinline__ void take_stage(Smem& s, Filter& f, const uint4* red, const float* src, uint32_t msk,
                                           uint32_t idx0, int m, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t r[4 * ((kFilterWarps + 3) / 4)];
#pragma unroll
  for (int i = 0; i < (kFilterWarps + 3) / 4; ++i) {
    const uint4 q = red[i];
    r[4 * i + 0] = q.x;
    r[4 * i + 1] = q.y;
    r[4 * i + 2] = q.z;
    r[4 * i + 3] = q.w;
  }
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kFilterWarps; ++i) {
    before += i < w ? r[i] : 0u;
    tot += r[i];
  }
  if (f.cnt + tot <= static_cast<uint32_t>(kFiltCap)) {
    put_survivors<kRing>(s, src, msk, idx0, f.cnt + before, w, lane);
    f.cnt += tot;
  } else {
    f = take_stage_split<kRing>(s, f, reinterpret_cast<const uint32_t*>(red), src, msk, idx0, m, tid);
  }
}

// Publishes this warp's survivor count (read after the next filter barrier).
__device__ __forceinline__ void publish(uint4* red, uint32_t msk, int w, int lane) {
  const uint32_t wt = __reduce_add_sync(kFull, __popc(msk));
  if (lane == 0) reinterpret_cast<uint32_t*>(red)[w] = wt;
}

__device__ __forceinline__ uint32_t stage_mask(const float (&v)[kVals], float t, bool edge, int64_t sj0, int64_t L,
                                               int w, int lane) {
  uint32_t msk = pass_mask(v, t);
  if (edge) {
    int lo, hi;
    stage_bounds(sj0, L, lo, hi);
    msk &= range_mask(w, lane, lo, hi);
  }
  return msk;
}

// The speculative threshold let fewer than m values through: stream the row
// again from global memory with no threshold (one filter barrier per stage).
__device__ __forceinline__ Filter refilter_from_global(Smem& s, Filter f, RowSpan sp, int64_t L, int m, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  f.cnt = 0;
  f.t = __int_as_float(0xff800000);  // -inf: keep everything
  f.compacted = false;
  f.strict = false;
  f.bounded = false;
  for (int st = 0; st < sp.nst; ++st) {
    const float* src = reinterpret_cast<const float*>(sp.src + static_cast<uint64_t>(st) * kStageBytes);
    const uint32_t avail = st + 1 == sp.nst ? sp.last_bytes : kStageBytes;
    const int64_t sj0 = sp.j0 + static_cast<int64_t>(st) * kStageElems;
    float v[kVals];
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int off = w * kWarpElems + q * 128 + lane * 4;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (4u * static_cast<uint32_t>(off) + 16u <= avail) x = __ldg(reinterpret_cast<const float4*>(src + off));
      v[4 * q + 0] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
    }
    const uint32_t msk = stage_mask(v, f.t, st == 0 || st + 1 == sp.nst, sj0, L, w, lane);
    publish(&s.red[f.par][0], msk, w, lane);
    bar_filter();
    take_stage<false>(s, f, &s.red[f.par][0], src, msk, static_cast<uint32_t>(sj0), m, tid);
    f.par ^= 1;
    if (f.cnt > static_cast<uint32_t>(kTrigger)) compact_any(s, f, m, tid);
    tighten(f, m);
  }
  bar_filter();
  return f;
}

// A threshold for a row with no estimate, from a sample of kStageElems values
// in kSampleChunks evenly spaced runs of 128 (aligned 16-byte blocks inside
// the row): the value with as many sampled values above it as 1.5 times the
// share of m in the sample, plus 16. Returns -inf when the sample gives none.
__device__ __noinline__ float sample_threshold(Smem& s, const float* row, int64_t L, int m, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  const uintptr_t a = reinterpret_cast<uintptr_t>(row);
  const uintptr_t as = a & ~static_cast<uintptr_t>(15);
  const int64_t j0 = -static_cast<int64_t>((a - as) >> 2);  // row index of the aligned base
  const int64_t span = L - j0;                               // floats from the aligned base to the row end
#pragma unroll
  for (int q = 0; q < kGroups; ++q) {
    const int64_t c = w * kGroups + q;
    const int64_t b = ((span - 128) * c / (kSampleChunks - 1)) & ~static_cast<int64_t>(3);
    const float4 x = __ldg(reinterpret_cast<const float4*>(as) + (b >> 2) + lane);
    const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t j = j0 + b + 4 * lane + i;
      s.fkey[val_offset(w, lane, 4 * q + i)] = (j >= 0 && j < L) ? to_key(xv[i]) : 0u;  // 0: below every key
    }
  }
  bar_filter();
  const double share = static_cast<double>(kStageElems) * m / static_cast<double>(L);
  const uint32_t need = min(static_cast<uint32_t>(kStageElems - 8), static_cast<uint32_t>(1.5 * share) + 16u);
  const uint32_t T = filter_kth(s, kStageElems, need, FKey{&s}, FAll{}, tid);
  return (T == 0u || T >= kInfKey) ? __int_as_float(0xff800000) : from_key(T);
}

__device__ __forceinline__ void load_slot(const Smem& s, int slot, int w, int lane, float (&v)[kVals]) {
#pragma unroll
  for (int q = 0; q < kGroups; ++q) {
    const float4 x = *reinterpret_cast<const float4*>(&s.ring[slot][w * kWarpElems + q * 128 + lane * 4]);
    v[4 * q + 0] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
}

__device__ void filter_loop(Smem& s, const float* logits, int64_t row_stride, const int32_t* lengths,
                            int64_t num_rows, int k, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  int slot = 0;         // ring slot of the next stage
  uint32_t phase = 0u;  // its full-barrier phase parity
  uint32_t par = 0u;    // parity of the per-stage counts in s.red
  Filter f;
  f.par = 0;
  int h = 0;
  int64_t row = blockIdx.x;
  int32_t L_next = row < num_rows ? static_cast<int32_t>(clamp_len(lengths, row, row_stride)) : 0;
  for (; row < num_rows; row += gridDim.x, ++h) {
    const int32_t L = L_next;  // lengths are int32, so is every clamped length
    if (row + gridDim.x < num_rows) L_next = static_cast<int32_t>(clamp_len(lengths, row + gridDim.x, row_stride));
    const int m = static_cast<int>(min64(k, L));
    const RowSpan sp = row_span(logits + row * row_stride, L);
    const int eb = h & 1;  // estimate written by the finisher two rows back
    bool spec = false;
    f.t = __int_as_float(0xff800000);
    if (m == k) {
      if (s.est_ok[eb] && L >= s.est_len[eb] - (s.est_len[eb] >> 3)) {
        spec = true;
        f.t = s.est[eb];
      } else if (s.own_len > 0 && L >= s.own_len - (s.own_len >> 3)) {
        spec = true;
        f.t = s.own_key > kInfKey ? __int_as_float(0x7f800000) : from_key(s.own_key);
      }
    }
    if (m == k && !spec && L >= kSampleMinLen) {
      const float ts = sample_threshold(s, logits + row * row_stride, L, m, tid);
      if (ts > __int_as_float(0xff800000)) {
        spec = true;
        f.t = ts;
      }
    }
    f.cnt = 0;
    f.compacted = false;
    f.strict = false;
    f.bounded = false;
    int32_t sj0 = static_cast<int32_t>(sp.j0);  // row index of the stage's first float (< L <= INT32_MAX)
    for (int st = 0; st < sp.nst; ++st, sj0 += kStageElems) {
      mbar_wait(&s.full[slot], phase);
      float v[kVals];
      load_slot(s, slot, w, lane, v);
      const uint32_t msk = stage_mask(v, f.t, st == 0 || st + 1 == sp.nst, sj0, L, w, lane);
      publish(&s.red[par][0], msk, w, lane);
      bar_filter();  // every warp's count of this stage is published
      take_stage<true>(s, f, &s.red[par][0], &s.ring[slot][0], msk, static_cast<uint32_t>(sj0), m, tid);
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.empty[slot]);
      if (f.cnt > static_cast<uint32_t>(kTrigger)) compact_any(s, f, m, tid);
      tighten(f, m);
      par ^= 1u;
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
    }
    bar_filter();  // every append is visible
    if (spec && !f.compacted && f.cnt < static_cast<uint32_t>(m)) f = refilter_from_global(s, f, sp, L, m, tid);
    if (f.cnt > static_cast<uint32_t>(kHandCap)) compact_any(s, f, m, tid);
    if (tid == 0 && m == k && f.bounded) {
      s.own_key = f.last_key;
      s.own_len = L;
    }
    bar_filter();  // the own estimate is read at the next row's start
    // hand over: wait until the finishers released the previous handover
    mbar_wait_sleep(&s.hempty, (h & 1) ^ 1);
    for (int e = tid; e < static_cast<int>(f.cnt); e += kFilterThreads) {
      s.hkey[e] = s.fkey[e];
      s.hidx[e] = s.fidx[e];
    }
    if (tid == 0) {
      s.h_row = row;
      s.h_len = L;
      s.h_n = static_cast<int32_t>(f.cnt);
      s.h_m = m;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.hfull);
  }
}

// ---------------------------------------------------------- finisher warps
// Ranks the handed-over candidates by the composite C = (kmax - key) << 32 |
// index (ascending C = key descending, index ascending; all C distinct).
// Buckets are 12-bit slices of C: count, scan, then find the bucket holding
// rank m-1. While a bucket at or before it is large, the range shrinks to the
// buckets up to it (everything after has rank >= m) and the count repeats.
// Then the candidates are grouped by bucket and each one's rank is its
// bucket's start plus the number of bucket members ahead of it.
__device__ __forceinline__ int bucket_shift(uint64_t cmax) {
  const int bits = cmax ? 64 - __clzll(static_cast<long long>(cmax)) : 0;
  int sh = bits > 12 ? bits - 12 : 0;  // cmax >> sh < 4096
  if ((cmax >> sh) >= static_cast<uint64_t>(kBuckets)) ++sh;
  return sh;
}

// Candidates [0, n) ordered in place by (key descending, index ascending) with
// a bitonic network over the next power of two (padding keys 0 sort last),
// then the first m indices written. Ends with a finisher barrier.
__device__ __noinline__ void finish_sorted(Smem& s, int n, int m, int k, int32_t* __restrict__ o, int fid) {
  int N = 1;
  while (N < n) N <<= 1;
  for (int e = n + fid; e < N; e += kFinishThreads) {
    s.hkey[e] = 0u;
    s.hidx[e] = 0xFFFFFFFFu;
  }
  bar_finish();
  for (int size = 2; size <= N; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = fid; t < (N >> 1); t += kFinishThreads) {
        const int i = 2 * t - (t & (stride - 1));
        const int j = i + stride;
        const uint32_t ki = s.hkey[i], ii = s.hidx[i], kj = s.hkey[j], ij = s.hidx[j];
        const bool j_first = kj > ki || (kj == ki && ij < ii);  // j belongs before i
        if (j_first == ((i & size) == 0)) {
          s.hkey[i] = kj;
          s.hidx[i] = ij;
          s.hkey[j] = ki;
          s.hidx[j] = ii;
        }
      }
      bar_finish();
    }
  }
  const int a = k >= 4 ? (3 * k) / 4 - 1 : 0;
  for (int p = fid; p < m; p += kFinishThreads) {
    o[p] = static_cast<int32_t>(s.hidx[p]);
    if (p == k - 1) s.rec[0] = s.hkey[p];
    if (p == a) s.rec[1] = s.hkey[p];
  }
  bar_finish();
}

__device__ void finish_one(Smem& s, int k, int32_t* __restrict__ out, int h, int fid) {
  const int fw = fid >> 5, lane = fid & 31;
  const int n = s.h_n, m = s.h_m;
  const int64_t row = s.h_row, L = s.h_len;
  int32_t* o = out + row * static_cast<int64_t>(k);
  for (int p = m + fid; p < k; p += kFinishThreads) o[p] = -1;
  if (n > 0) {
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u, imax = 0u;
    for (int e = fid; e < n; e += kFinishThreads) {
      const uint32_t key = s.hkey[e];
      kmin = min(kmin, key);
      kmax = max(kmax, key);
      imax = max(imax, s.hidx[e]);
    }
    kmin = __reduce_min_sync(kFull, kmin);
    kmax = __reduce_max_sync(kFull, kmax);
    imax = __reduce_max_sync(kFull, imax);
    if (lane == 0) {
      s.nred[0][fw] = kmin;
      s.nred[1][fw] = kmax;
      s.nred[2][fw] = imax;
    }
    bar_finish();
#pragma unroll
    for (int ww = 0; ww < kFinishWarps; ++ww) {
      kmin = min(kmin, s.nred[0][ww]);
      kmax = max(kmax, s.nred[1][ww]);
      imax = max(imax, s.nred[2][ww]);
    }
    uint64_t cmax = (static_cast<uint64_t>(kmax - kmin) << 32) | imax;
    int sh = bucket_shift(cmax);
    auto comp = [&](uint32_t key, uint32_t idx) -> uint64_t {
      return (static_cast<uint64_t>(kmax - key) << 32) | idx;
    };
    uint4* bc4 = reinterpret_cast<uint4*>(&s.bcnt[fid * kScanPer]);
    const uint32_t mm1 = static_cast<uint32_t>(m - 1);
    uint32_t big = 0;
    for (int pass = 0;; ++pass) {
#pragma unroll
      for (int i = 0; i < kScanPer / 4; ++i) bc4[i] = make_uint4(0u, 0u, 0u, 0u);
      bar_finish();
      for (int e = fid; e < n; e += kFinishThreads) {
        const uint64_t c = comp(s.hkey[e], s.hidx[e]);
        if (c <= cmax) atomicAdd(&s.bcnt[static_cast<uint32_t>(c >> sh)], 1u);
      }
      bar_finish();
      // exclusive scan: thread fid owns counters [32 fid, 32 fid + 32)
      uint32_t c[kScanPer], sum = 0;
#pragma unroll
      for (int i = 0; i < kScanPer / 4; ++i) {
        const uint4 q = bc4[i];
        c[4 * i + 0] = q.x;
        c[4 * i + 1] = q.y;
        c[4 * i + 2] = q.z;
        c[4 * i + 3] = q.w;
        sum += q.x + q.y + q.z + q.w;
      }
      uint32_t incl = sum;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += t;
      }
      if (lane == 31) s.nred[3][fw] = incl;
      bar_finish();
      uint32_t run = incl - sum;
      for (int ww = 0; ww < fw; ++ww) run += s.nred[3][ww];
#pragma unroll
      for (int i = 0; i < kScanPer / 4; ++i) {
        uint4 q;
        q.x = run;
        run += c[4 * i + 0];
        q.y = run;
        run += c[4 * i + 1];
        q.z = run;
        run += c[4 * i + 2];
        q.w = run;
        run += c[4 * i + 3];
        bc4[i] = q;
      }
      // the bucket holding rank m-1 (exactly one thread finds it)
      run = incl - sum;
      for (int ww = 0; ww < fw; ++ww) run += s.nred[3][ww];
#pragma unroll
      for (int i = 0; i < kScanPer; ++i) {
        if (run <= mm1 && mm1 < run + c[i]) s.bc[4] = static_cast<uint32_t>(fid * kScanPer + i);
        run += c[i];
      }
      bar_finish();
      const uint32_t bm = s.bc[4];
      big = 0;  // largest bucket at or before bm
#pragma unroll
      for (int i = 0; i < kScanPer; ++i)
        if (static_cast<uint32_t>(fid * kScanPer + i) <= bm) big = max(big, c[i]);
      big = __reduce_max_sync(kFull, big);
      if (lane == 0) s.nred[4][fw] = big;
      bar_finish();
#pragma unroll
      for (int ww = 0; ww < kFinishWarps; ++ww) big = max(big, s.nred[4][ww]);
      if (big <= static_cast<uint32_t>(kSmallBucket) || sh == 0 || pass == kSortPasses - 1) break;
      cmax = ((static_cast<uint64_t>(bm) + 1u) << sh) - 1u;
      sh = bucket_shift(cmax);
      bar_finish();  // bc[4] and nred[4] are rewritten by the next pass
    }
    if (big > static_cast<uint32_t>(kBigBucket)) {
      // many candidates share a bucket (values on a coarse grid): counting
      // ranks inside it would be quadratic, so sort everything instead
      finish_sorted(s, n, m, k, o, fid);
    } else {
      for (int e = fid; e < n; e += kFinishThreads) {
        const uint64_t cc = comp(s.hkey[e], s.hidx[e]);
        if (cc > cmax) continue;
        const uint32_t p = atomicAdd(&s.bcnt[static_cast<uint32_t>(cc >> sh)], 1u);
        s.perm[p] = static_cast<uint16_t>(e);
      }
      bar_finish();  // bcnt[b] is now the end of bucket b (= start of b + 1)
      const int a = k >= 4 ? (3 * k) / 4 - 1 : 0;
      for (int e = fid; e < n; e += kFinishThreads) {
        const uint32_t key = s.hkey[e], idx = s.hidx[e];
        const uint64_t cc = comp(key, idx);
        if (cc > cmax) continue;
        const uint32_t b = static_cast<uint32_t>(cc >> sh);
        const uint32_t s0 = b ? s.bcnt[b - 1] : 0u, s1 = s.bcnt[b];
        if (s0 >= static_cast<uint32_t>(m)) continue;
        uint32_t r = s0;
        for (uint32_t q = s0; q < s1; ++q) {
          const uint32_t j = s.perm[q];
          const uint32_t kj = s.hkey[j], ij = s.hidx[j];
          r += kj > key || (kj == key && ij < idx);
        }
        if (r < static_cast<uint32_t>(m)) {
          s.ostage[r] = static_cast<int32_t>(idx);
          if (r == static_cast<uint32_t>(k - 1)) s.rec[0] = key;
          if (r == static_cast<uint32_t>(a)) s.rec[1] = key;
        }
      }
      bar_finish();
      for (int p = fid; p < m; p += kFinishThreads) o[p] = s.ostage[p];
    }
  }
  if (fid == 0) {
    bool ok = false;
    float e = 0.f;
    if (n > 0 && m == k) {
      const uint32_t kt = s.rec[0], ka = s.rec[1];
      const float vt = from_key(kt), va = from_key(ka);
      e = vt - 0.5f * (va - vt);
      ok = kt != kNanKey && ka != kNanKey && isfinite(e);
    }
    s.est[h & 1] = e;
    s.est_len[h & 1] = L;
    s.est_ok[h & 1] = ok ? 1 : 0;
  }
}

__device__ void finish_loop(Smem& s, int64_t num_rows, int k, int32_t* __restrict__ out, int fid) {
  const int lane = fid & 31;
  int h = 0;
  for (int64_t row = blockIdx.x; row < num_rows; row += gridDim.x, ++h) {
    mbar_wait_sleep(&s.hfull, h & 1);
    finish_one(s, k, out, h, fid);
    bar_finish();  // every read of the handover is done, the estimate written
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.hempty);
  }
}

// ---------------------------------------------------------- producer warp
__device__ void produce_loop(Smem& s, const float* logits, int64_t row_stride, const int32_t* lengths,
                             int64_t num_rows) {
  int slot = 0;         // ring slot of the next stage
  uint32_t phase = 0u;  // parity of the slot's current fill
  for (int64_t row = blockIdx.x; row < num_rows; row += gridDim.x) {
    const int64_t L = clamp_len(lengths, row, row_stride);
    const RowSpan sp = row_span(logits + row * row_stride, L);
    for (int st = 0; st < sp.nst; ++st) {
      mbar_wait_sleep(&s.empty[slot], phase ^ 1u);
      const uint32_t bytes = st + 1 == sp.nst ? sp.last_bytes : kStageBytes;
      fence_proxy_async();
      mbar_arrive_expect_tx(&s.full[slot], bytes);
      bulk_g2s(&s.ring[slot][0], sp.src + static_cast<uint64_t>(st) * kStageBytes, bytes, &s.full[slot]);
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
    }
  }
}

}  // namespace rows

// Many rows: grid = min(num_rows, SMs), one CTA per SM, rows strided by grid.
__global__ void __launch_bounds__(rows::kThreads, 1)
    topk_rows_kernel(const float* __restrict__ logits, int64_t row_stride, const int32_t* __restrict__ lengths,
                     int64_t num_rows, int k, int32_t* __restrict__ out) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  rows::Smem& s = *reinterpret_cast<rows::Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < rows::kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], rows::kFilterWarps);
    }
    mbar_init(&s.hfull, rows::kFilterWarps);
    mbar_init(&s.hempty, rows::kFinishWarps);
    for (int i = 0; i < 2; ++i) {
      s.est_ok[i] = 0;
      s.est[i] = 0.f;
      s.est_len[i] = 0;
    }
    s.own_key = 0u;
    s.own_len = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (warp < rows::kFilterWarps) {
    rows::filter_loop(s, logits, row_stride, lengths, num_rows, k, tid);
  } else if (warp < rows::kProducerWarp) {
    rows::finish_loop(s, num_rows, k, out, tid - rows::kFilterThreads);
  } else if (lane == 0) {
    rows::produce_loop(s, logits, row_stride, lengths, num_rows);
  }
}
