// The top-k kernel: one persistent CTA per SM over many rows, or a
// thread-block cluster per row when rows are few and long.
//
// Many-row mode (cluster size 1, 480 threads, three warp roles):
//   producer (1 warp, one lane)  : cp.async.bulk copies of the CTA's rows, in
//                                  8192-element stages, into a 96 KB shared
//                                  ring (full / empty mbarriers).
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
//   finisher (6 warps; 7 for     : ranks the handed-over candidates by (key
//   16-bit logits)                 descending, index ascending) with bucket
//                                  passes over a composite key (an LSD radix
//                                  sort when a bucket stays crowded with equal
//                                  keys), then writes the first m indices and
//                                  -1 padding while the filter warps already
//                                  stream the next row.
//
// A row starts with a speculative threshold: from the row the finisher
// completed two rows earlier (half the gap between that row's 3k/4-th and
// k-th largest below its k-th), else from the threshold that passed enough of
// the CTA's previous row, else from a sample of the row itself. If fewer than
// m values pass it, the filter warps re-read the row from global memory with
// no threshold; the result is exact either way, only the time changes.
//
// Cluster mode (a cluster of C CTAs per row, 384 threads: filter warps and a
// producer warpgroup, no finisher warps): rank r streams the contiguous chunk r of
// the row exactly as a row is streamed above, keeping a superset of the
// chunk's top min(m, chunk). The ranks then merge through distributed shared
// memory (SGLang PR #34167 code excerpt, TopKCluster::forward: per-rank
// counts, cluster barriers between phases, rank-ordered write offsets):
// counts and key bounds are published, cluster-wide histogram rounds narrow a
// threshold until the survivors fit the leader's buffer, and every rank writes
// its survivors into the leader's shared memory at rank-ordered offsets (a
// tied threshold value is shared out in rank order, which is index order).
// The leader's filter warps then rank and write the row like the finisher.
// DSMEM addresses are 32-bit shared::cluster addresses used only with
// ld/st.shared::cluster (the SGLang page traces a miscompile to merging them
// with CTA pointers).
//
// The selection follows the pages' histogram / cumulative-sum / threshold /
// gt-eq split (SGLang PR #34167 code excerpt, the radix top-k kernel), made
// exact: ties at the threshold go to the lowest indices (a second radix select
// over the indices of the tied keys) instead of a capped tie list.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace dsa {
namespace rows {

constexpr int kFilterWarps = 8;
constexpr int kFilterThreads = kFilterWarps * 32;  // 256
// Finisher warps of the many-row kernel, by element type. With 16-bit logits
// the ranking (values tied on a coarse grid, sorted) bounds a row, so it takes
// the spare warp too; with fp32 the finisher keeps up with six, and a
// seventh only takes issue slots from the streaming filter warps.
template <class T>
__host__ __device__ constexpr int finish_warps() { return sizeof(T) == 4 ? 6 : 7; }
constexpr int kFinishWarpsMax = 7;
constexpr int kNredWarps = kFilterWarps + 6;  // warps whose reductions sit in Smem::nred
template <class T>
__host__ __device__ constexpr int finish_threads() { return finish_warps<T>() * 32; }  // 192 or 224
template <class T>
__host__ __device__ constexpr int joint_threads() { return kFilterThreads + finish_threads<T>(); }  // both ranking a CTA's last row
template <class T>
__host__ __device__ constexpr int producer_warp() { return kFilterWarps + finish_warps<T>(); }
constexpr int kThreads = 16 * 32;                       // 512: many-row mode (filter, finisher, producer warps)
constexpr int kClusterWarp = kFilterWarps;              // cluster mode: the producer warp
constexpr int kClusterThreads = 12 * 32;                // 384: cluster mode (3 warpgroups; warps 9-11 only mirror barriers)
constexpr int kGroups = 8;                              // groups of 4 values per lane and stage
constexpr int kVals = 4 * kGroups;                      // 32 values per lane and stage
constexpr int kWarpElems = 32 * kVals;                  // 1024 per warp and stage
constexpr int kStageElems = kFilterWarps * kWarpElems;  // 8192
constexpr int kRingBytes = 3 * 32768;                   // 96 KB ring
constexpr int kMaxStages = 6;
constexpr int64_t kShortStride = 8192 - 8;                // rows of at most this many elements are one stage
constexpr int kFiltCap = 8192;                          // candidate buffer entries
constexpr int kTrigger = kFiltCap / 2;                  // compact after a stage that leaves more
constexpr int kHandCap = 4096;                          // handed-over (or gathered) candidates, at most
constexpr int kPerThread = (kFiltCap + kFilterThreads - 1) / kFilterThreads;  // entries per filter thread
constexpr int kRounds = 4;                              // radix rounds of 8 bits
constexpr int kKeepLimit = 2560;                        // approximate compaction keeps at most this many
constexpr int kSampleRunsPerWarp = 4;                   // runs of 128 each filter warp samples
constexpr int kSampleChunks = kFilterWarps * kSampleRunsPerWarp;  // runs sampled for a row's first threshold
constexpr int kSampleVals = kSampleChunks * 128;        // 4096 sampled values
constexpr int64_t kSampleMinLen = 2 * kSampleVals;      // shorter rows start with no threshold
constexpr int kBigBucket = 64;                          // finisher: larger buckets are sorted instead
constexpr int kSmallBucket = 16;                        // finisher: largest bucket ranked by direct counting
constexpr int kSortPasses = 3;                          // finisher: bucket count passes, at most
constexpr int kBucketMax = 4096;                        // finisher bucket counters
constexpr uint32_t kUnsorted = DSA_FLAG_UNSORTED;

template <class T>
__host__ __device__ constexpr int stages_of() {
  return kRingBytes / (kStageElems * static_cast<int>(sizeof(T)));
}

static_assert(kVals <= 32, "a lane's survivors of one stage form a 32-bit mask");
static_assert(kFiltCap - kTrigger >= kStageElems / 2, "half a stage fits after a compaction");
static_assert(kFilterWarps % 2 == 0 && kKeepLimit + kStageElems / 2 <= kFiltCap, "split halves fit after a compaction");
static_assert(kHandCap >= kMaxK && kTrigger >= kMaxK, "buffers must hold k entries");
static_assert(stages_of<float>() == 3 && stages_of<__half>() == 6 && stages_of<__half>() <= kMaxStages, "ring");

// Call parameters (the C ABI's arguments).
struct Params {
  const void* logits;
  int64_t row_stride;  // elements
  const int32_t* lengths;
  int64_t num_rows;
  int32_t k;
  uint32_t flags;        // DSA_FLAG_*
  const int32_t* table;  // optional index table: out = table[row * table_stride + idx]
  int64_t table_stride;
  int32_t* out;
};

struct __align__(128) Smem {
  unsigned char ring[kRingBytes];  // stages of kStageElems elements
  uint32_t fkey[kFiltCap];         // filter candidates
  uint32_t fidx[kFiltCap];
  uint32_t hkey[kHandCap];  // handed over to the finishers (cluster mode: gathered at the leader)
  uint32_t hidx[kHandCap];
  uint32_t bcnt[kBucketMax];  // finisher bucket counters / ends (cluster mode: merge histograms first)
  uint16_t perm[kHandCap];    // finisher: candidates grouped by bucket
  int32_t ostage[kMaxK];      // finisher: the row's output, written out coalesced
  uint32_t hist[256];         // filter radix histogram
  uint4 red[2][(kFilterWarps + 3) / 4];  // per-warp survivor counts, by stage parity
  uint32_t fred[4][kFilterWarps];
  uint32_t nred[5][kNredWarps];  // finisher per-warp reductions (6 to 14 warps; a 15th: nred_x)
  uint32_t bc[8];
  uint32_t small[32];
  uint32_t rec[2];  // finisher: keys at ranks k-1 and 3k/4-1
  uint32_t pub[8];  // cluster mode: published to the other ranks
  uint32_t spub[4];  // cluster mode: [0..2] this rank's sample count and key bounds, read by the others; [3] the merge's key-difference bits
  // handover (filter -> finisher)
  int64_t h_row, h_len;
  int32_t h_n, h_m;
  // speculative threshold (finisher -> filter), by handover parity
  int64_t est_len[2];
  float est[2];
  int32_t est_ok[2];
  // the filter warps' own estimate: an earlier row of length own_len passed at
  // least k values at or above own_key (own_len 0: none yet)
  uint32_t own_key;
  int32_t own_len;
  float row_t0;        // the current row's initial threshold
  WaitCtl wait;        // abort flag and time limit of every pipeline wait
  uint32_t abort_seen; // the abort flag as thread 0 read it before an item's last filter barrier
  uint32_t abort_any;  // cluster mode: some rank gave up (read by the leader)
  uint32_t final_bar;  // cluster mode: number of cluster barriers of the merge (0: not yet known)
  uint32_t joint;      // many-row mode: the CTA's last row is ranked by filter and finisher warps together
  uint32_t merge_bars; // cluster mode: cluster barriers of earlier merge attempts
  uint32_t merge_retry;
  unsigned long long full[kMaxStages], empty[kMaxStages];
  unsigned long long hfull, hempty;
  // the 15th warp's per-warp reductions (a joint ranking with seven finisher
  // warps), kept apart so that every other field has the offset it has with
  // six: the block's layout measurably changes the streaming loop's speed
  uint32_t nred_x[5];
};
static_assert(sizeof(Smem) <= 232448, "shared memory budget of one CTA per SM");

// The CTA's shared-memory block. Functions that are not inlined take it from
// here, not as an argument: through a reference argument every access would
// be a generic one (slower than a shared-memory access, atomics most of all).
__device__ __forceinline__ Smem& cta_smem() {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  return *reinterpret_cast<Smem*>(smem_raw);
}
static_assert(2 * 256 + 256 <= kBucketMax, "merge histograms alias the bucket counters");

__device__ __forceinline__ void bar_filter() { asm volatile("bar.sync 1, %0;" ::"n"(kFilterThreads) : "memory"); }
// Named barrier that also returns whether any participating thread passed
// true: every thread of the role takes the same branch afterwards.
template <int kBar, int kCount>
__device__ __forceinline__ bool bar_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(kBar), "n"(kCount)
      : "memory");
  return r != 0u;
}
__device__ __forceinline__ bool bar_filter_any(bool pred) { return bar_any<1, kFilterThreads>(pred); }

// Smallest float threshold t with (!(x < t)) == (key(x) > T) for every non-NaN x.
// T at or above +inf's key has no such float: +inf is returned, which also
// keeps +inf itself (a superset, harmless: the final ranking is exact).
__device__ __forceinline__ float above(uint32_t T) {
  return T < kInfKey ? from_key(T + 1u) : __int_as_float(0x7f800000);
}

// The 16-byte aligned byte span covering item entries [0, L) of an item that
// starts at element pointer `row`.
struct RowSpan {
  const char* src;
  int64_t j0;           // item index of the span's first element (-7..0)
  int nst;              // stages
  uint32_t last_bytes;  // bytes of the last stage
};

template <class T>
__device__ __forceinline__ RowSpan row_span(const T* row, int64_t L) {
  constexpr uint32_t kStageBytes = kStageElems * sizeof(T);
  RowSpan sp;
  const uintptr_t a = reinterpret_cast<uintptr_t>(row);
  const uintptr_t as = a & ~static_cast<uintptr_t>(15);
  sp.src = reinterpret_cast<const char*>(as);
  sp.j0 = -static_cast<int64_t>((a - as) / sizeof(T));
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
// Position of value j (0..31) of a lane inside its stage: group j/4 of four
// consecutive elements at warp*kWarpElems + (j/4)*128 + lane*4 (conflict-free
// 128-bit (fp32) or 64-bit (16-bit types) shared loads).
__device__ __forceinline__ int val_offset(int w, int lane, int j) {
  return w * kWarpElems + (j >> 2) * 128 + lane * 4 + (j & 3);
}

__device__ __forceinline__ uint32_t pass_mask(const float (&v)[kVals], float t) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < kVals; ++j) m |= static_cast<uint32_t>(!(v[j] < t)) << j;
  return m;
}

// Stage-local offsets [lo, hi) of a stage whose first element has item index
// sj0 that hold item indices in [0, L).
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

// 256-bin histogram of the 8-bit digit at bit sh of v(e), over the entries
// [0, n) with pred(e) and v(e) in [lo, hi] (hist zeroed, filter threads).
// One shared atomic per entry: merging the lanes of a digit first (match.any
// or a vote per digit bit) costs more than the contended atomics it saves,
// even for values on a few levels.
template <class V, class P>
__device__ __forceinline__ void digit_histogram(uint32_t* hist, int n, V v, P pred, uint32_t lo, uint32_t hi, int sh,
                                                int tid) {
#pragma unroll 4
  for (int e = tid; e < n; e += kFilterThreads) {
    if (!pred(e)) continue;
    const uint32_t x = v(e);
    if (x >= lo && x <= hi) atomicAdd(&hist[(x >> sh) & 255u], 1u);
  }
}

// need-th largest of v(e) over the candidates with pred(e) (1 <= need <= their
// number). Radix rounds over 8-bit windows below the highest bit where the
// bounds differ; a bucket of <= 32 values is finished by one warp. Each thread
// adds a run of equal digits with one atomic.
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
    {
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
    }
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
struct FIdx {
  const Smem* s;
  __device__ uint32_t operator()(int e) const { return s->fidx[e]; }
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

// Stores the candidates with key > A and, when kTies, those with key == A and
// index <= I at positions off.. of the shared::cluster addresses rkey / ridx
// (the copy to a cluster's leader, another buffer). Two rolled passes over the
// candidates, count then store, instead of holding 32 entries per thread in
// registers: it runs once per launch, so its code size is its cost. Returns
// the kept count (uniform).
template <bool kTies>
__device__ uint32_t keep_remote(Smem& s, int n, uint32_t A, uint32_t I, int tid, uint32_t rkey, uint32_t ridx,
                                uint32_t off) {
  const int w = tid >> 5, lane = tid & 31;
  auto kept = [&](int e) -> bool {
    const uint32_t kk = s.fkey[e];
    return kk > A || (kTies && kk == A && s.fidx[e] <= I);
  };
  uint32_t nk = 0;
  for (int e = tid; e < n; e += kFilterThreads) nk += kept(e) ? 1u : 0u;
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
  for (int e = tid; e < n; e += kFilterThreads) {
    if (kept(e)) {
      dsmem_st(rkey + 4u * (off + pos), s.fkey[e]);
      dsmem_st(ridx + 4u * (off + pos), s.fidx[e]);
      ++pos;
    }
  }
  bar_filter();
  return total;
}

// Keeps the candidates with key > A and, when kTies, those with key == A and
// index <= I, in place and in any order. Every filter thread reads its entries
// (into registers) before any is written. Returns the kept count (uniform).
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

// Index cut among the candidates with key == T: the need-th smallest index
// (1 <= need <= neq, their number; indices are distinct).
__device__ __forceinline__ uint32_t tie_cut(Smem& s, int n, uint32_t T, uint32_t need, uint32_t neq, int tid) {
  // when the tied entries' indices form one dense range (a run of one repeated
  // value, such as a tail of -inf), the need-th smallest is min + need - 1
  uint32_t lo, hi;
  filter_minmax(s, n, FIdx{&s}, FKeyIs{&s, T}, lo, hi, tid);
  if (hi - lo + 1u == neq) return lo + need - 1u;
  return ~filter_kth(s, n, need, FNotIdx{&s}, FKeyIs{&s, T}, tid);
}

// Counts of candidates [0, n) with key > T and key == T (uniform).
__device__ void count_gt_eq(Smem& s, int n, uint32_t T, uint32_t& ngt, uint32_t& neq, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t g = 0, q = 0;
  for (int e = tid; e < n; e += kFilterThreads) {
    const uint32_t key = s.fkey[e];
    g += key > T;
    q += key == T;
  }
  g = __reduce_add_sync(kFull, g);
  q = __reduce_add_sync(kFull, q);
  if (lane == 0) {
    s.fred[2][w] = g;
    s.fred[3][w] = q;
  }
  bar_filter();
  ngt = __reduce_add_sync(kFull, lane < kFilterWarps ? s.fred[2][lane] : 0u);
  neq = __reduce_add_sync(kFull, lane < kFilterWarps ? s.fred[3][lane] : 0u);
  bar_filter();
}

// Exact: keeps the top m of candidates [0, n) by (key descending, index
// ascending), n > m >= 1. Returns the m-th largest key.
__device__ __noinline__ uint32_t compact_exact(int n, int m, int tid) {
  Smem& s = cta_smem();
  bar_filter();  // every append is visible
  const uint32_t T = filter_kth(s, n, static_cast<uint32_t>(m), FKey{&s}, FAll{}, tid);
  uint32_t ngt, neq;
  count_gt_eq(s, n, T, ngt, neq, tid);
  const uint32_t need = static_cast<uint32_t>(m) - ngt;  // entries equal to T that stay
  uint32_t I = 0xFFFFFFFFu;                               // largest index of a kept tie
  if (neq > need) I = tie_cut(s, n, T, need, neq, tid);
  keep_pass<true>(s, n, T, I, tid);
  return T;
}

// Approximate: narrows the radix bucket holding the m-th largest key until
// every key at or above the bucket's lower end fits in kKeepLimit entries,
// then keeps exactly those (a superset of the top m). Returns ok = 0, having
// changed nothing, when that needs more than kRounds rounds or the bucket is
// one tied key with too many entries: the exact pass must run.
struct FastCut {
  uint32_t ok, lo, kept;
};

__device__ __noinline__ FastCut compact_fast(int n, int m, int tid) {
  Smem& s = cta_smem();
  uint32_t kept = 0;
  const int w = tid >> 5, lane = tid & 31;
  bar_filter();  // every append is visible
  uint32_t lo, hi;
  filter_minmax(s, n, FKey{&s}, FAll{}, lo, hi, tid);
  uint32_t need = static_cast<uint32_t>(m), above_lo = 0;
  bool ok = false;
  for (int round = 0; round < kRounds && lo != hi; ++round) {
    const int sh = window_shift(lo, hi);
    for (int i = tid; i < 256; i += kFilterThreads) s.hist[i] = 0u;
    if (tid == 0) s.bc[0] = 0xFFFFFFFFu;
    bar_filter();
    digit_histogram(s.hist, n, FKey{&s}, FAll{}, lo, hi, sh, tid);
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
    above_lo += above_b;
    need -= above_b;
    narrow(lo, hi, sh, bsel);
    if (above_lo + in_b <= static_cast<uint32_t>(kKeepLimit)) {
      ok = true;
      kept = above_lo + in_b;
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
  bool compacted;     // the item was compacted at least once
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
  const FastCut c = compact_fast(static_cast<int>(f.cnt), m, tid);
  if (c.ok) {
    f.cnt = c.kept;
    f.t = c.lo > kInfKey ? __int_as_float(0x7f800000) : from_key(c.lo);
    f.last_key = c.lo;
    f.bounded = true;
    f.strict = false;
    tighten(f, m);
  } else {
    const uint32_t T = compact_exact(static_cast<int>(f.cnt), m, tid);
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
template <class T, bool kRing>
__device__ __forceinline__ void put_survivors(Smem& s, const T* src, uint32_t msk, uint32_t idx0, uint32_t pos, int w,
                                              int lane) {
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
    if (a1) x1 = kRing ? Elem<T>::f(src[o1]) : Elem<T>::one_ldg(src + o1);
    if (a2) x2 = kRing ? Elem<T>::f(src[o2]) : Elem<T>::one_ldg(src + o2);
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
// two halves, compacting first whenever a half would not fit. A half with
// more than the free space implies more than kTrigger >= m entries held, so
// the compaction applies; afterwards a half (<= kStageElems / 2) fits. Masks
// taken before a compaction are supersets of the current ones, which is
// harmless: the final ranking is exact.
// (Rare paths take and return the filter state by value so that it never has
// an address and stays in registers in the hot loop. This one and the re-read
// below are inlined: a real call inside the row loop made the compiler keep
// loop state in local memory, reloaded on every stage.)
template <class T, bool kRing>
__device__ __forceinline__ Filter take_stage_split(Smem& s, Filter f, const uint32_t* red, const T* src, uint32_t msk,
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
    if (w / kHalf == half) put_survivors<T, kRing>(s, src, msk, idx0, f.cnt + before, w, lane);
    f.cnt += tot;
    bar_filter();  // this half's entries are visible to a following compaction
  }
  return f;
}

// Takes one stage after the filter barrier that completed its per-warp counts.
template <class T, bool kRing>
__device__ __forceinline__ void take_stage(Smem& s, Filter& f, const uint4* red, const T* src, uint32_t msk,
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
    put_survivors<T, kRing>(s, src, msk, idx0, f.cnt + before, w, lane);
    f.cnt += tot;
  } else {
    f = take_stage_split<T, kRing>(s, f, reinterpret_cast<const uint32_t*>(red), src, msk, idx0, m, tid);
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

// The speculative threshold let fewer than m values through: stream the item
// again from global memory with no threshold (one filter barrier per stage).
template <class T>
__device__ __forceinline__ Filter refilter_from_global(Smem& s, Filter f, RowSpan sp, int64_t L, uint32_t base, int m,
                                                       int tid) {
  constexpr uint32_t kStageBytes = kStageElems * sizeof(T);
  const int w = tid >> 5, lane = tid & 31;
  f.cnt = 0;
  f.t = __int_as_float(0xff800000);  // -inf: keep everything
  f.compacted = false;
  f.strict = false;
  f.bounded = false;
  for (int st = 0; st < sp.nst; ++st) {
    const T* src = reinterpret_cast<const T*>(sp.src + static_cast<uint64_t>(st) * kStageBytes);
    const uint32_t avail = st + 1 == sp.nst ? sp.last_bytes : kStageBytes;
    const int64_t sj0 = sp.j0 + static_cast<int64_t>(st) * kStageElems;
    float v[kVals];
#pragma unroll
    for (int q = 0; q < kGroups; ++q) {
      const int off = w * kWarpElems + q * 128 + lane * 4;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (static_cast<uint32_t>(sizeof(T)) * static_cast<uint32_t>(off + 4) <= avail) Elem<T>::four_ldg(src + off, x);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[4 * q + i] = x[i];
    }
    const uint32_t msk = stage_mask(v, f.t, st == 0 || st + 1 == sp.nst, sj0, L, w, lane);
    publish(&s.red[f.par][0], msk, w, lane);
    bar_filter();
    take_stage<T, false>(s, f, &s.red[f.par][0], src, msk, base + static_cast<uint32_t>(sj0), m, tid);
    f.par ^= 1;
    if (f.cnt > static_cast<uint32_t>(kTrigger)) compact_any(s, f, m, tid);
    tighten(f, m);
  }
  bar_filter();
  return f;
}

// The need-th largest of the nvals sampled keys in fkey, to within
// one bin of a second histogram round (1 <= need <= the number sampled; every
// sampled key lies in [lo, hi]). Round one counts 1024 bins over a 10-bit
// slice of [lo, hi] below its highest differing bit and finds, from the top,
// the bin holding the need-th key; round two does the same inside that bin.
// The result is the smallest sampled key in the final bin: at least `need`
// sampled keys are at or above it, and at most the rest of that bin besides
// (for fp32 logits a second-round bin spans about 1e-3 of the value and holds
// about one sampled key; for values on a coarse grid it is one value, the
// exact answer).
// Counters live in fidx, unused until the item streams. Two plain-atomic
// passes instead of a radix select's three or four rounds with their
// barriers.
__device__ __forceinline__ uint32_t sample_kth(Smem& s, int nvals, uint32_t need, uint32_t lo, uint32_t hi, int tid) {
  constexpr int kBits = 10, kBins = 1 << kBits, kPer = kBins / kFilterThreads;  // 4 bins per thread
  const int w = tid >> 5, lane = tid & 31;
  uint32_t* hist = s.fidx;
  const uint32_t span = hi - lo;
  if (span == 0u) return lo;
  const int bits = 32 - __clz(span);
  int sh = bits > kBits ? bits - kBits : 0;  // (key - lo) >> sh < kBins
  uint32_t base = lo, top = hi;
  for (int round = 0; round < 2; ++round) {
    uint4* h4 = reinterpret_cast<uint4*>(hist + kPer * tid);
#pragma unroll
    for (int i = 0; i < kPer / 4; ++i) h4[i] = make_uint4(0u, 0u, 0u, 0u);
    bar_filter();
    for (int e = tid; e < nvals; e += kFilterThreads) {
      const uint32_t x = s.fkey[e];
      if (x >= base && x <= top) atomicAdd(&hist[(x - base) >> sh], 1u);
    }
    bar_filter();
    // from the top: thread tid owns bins kBins - 1 - (kPer tid + j), j = 0..kPer-1
    const uint4* r4 = reinterpret_cast<const uint4*>(hist + kBins - kPer * (tid + 1));
    uint32_t c[kPer], sum = 0u;
#pragma unroll
    for (int i = 0; i < kPer / 4; ++i) {
      const uint4 q = r4[i];  // bins ascending; c[] descending
      c[kPer - 1 - 4 * i] = q.x;
      c[kPer - 2 - 4 * i] = q.y;
      c[kPer - 3 - 4 * i] = q.z;
      c[kPer - 4 - 4 * i] = q.w;
      sum += q.x + q.y + q.z + q.w;
    }
    uint32_t incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t t = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += t;
    }
    if (lane == 31) s.fred[2][w] = incl;
    bar_filter();
    uint32_t run = incl - sum;
    for (int ww = 0; ww < w; ++ww) run += s.fred[2][ww];
    if (run < need && need <= run + sum) {  // exactly one thread
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if (run < need && need <= run + c[j]) {
          s.bc[0] = static_cast<uint32_t>(kBins - 1 - (kPer * tid + j));
          s.bc[1] = run;
        }
        run += c[j];
      }
    }
    bar_filter();
    const uint32_t b = s.bc[0];
    need -= s.bc[1];
    base += b << sh;
    top = min(top, base + ((1u << sh) - 1u));
    if (round == 1 || sh == 0) break;
    sh = sh > kBits ? sh - kBits : 0;
    bar_filter();  // bc and the counters are rewritten by the next round
  }
  // the smallest sampled key in the final bin: a key that occurs (a value
  // grid's level, so that the filter's strict bound can later exclude its
  // further copies), with as many keys at or above it as the bin's edge
  uint32_t mn = 0xFFFFFFFFu;
  for (int e = tid; e < nvals; e += kFilterThreads) {
    const uint32_t x = s.fkey[e];
    if (x >= base && x <= top) mn = min(mn, x);
  }
  mn = __reduce_min_sync(kFull, mn);
  if (lane == 0) s.fred[3][w] = mn;
  bar_filter();
  return __reduce_min_sync(kFull, lane < kFilterWarps ? s.fred[3][lane] : 0xFFFFFFFFu);
}

// Loads kFilterWarps * kRunsPerWarp evenly spaced runs of 128 values (aligned
// 16-byte blocks inside the item) into fkey as keys, 0 for a position outside
// [0, L) (below every key), and returns their smallest and largest key in
// every filter thread.
template <class T, int kRunsPerWarp>
__device__ __forceinline__ void sample_keys(Smem& s, const T* row, int64_t L, int tid, uint32_t& mn, uint32_t& mx) {
  constexpr int kChunks = kFilterWarps * kRunsPerWarp;
  const int w = tid >> 5, lane = tid & 31;
  const uintptr_t a = reinterpret_cast<uintptr_t>(row);
  const uintptr_t as = a & ~static_cast<uintptr_t>(15);
  const int64_t j0 = -static_cast<int64_t>((a - as) / sizeof(T));  // item index of the aligned base
  const int64_t span = L - j0;                                      // elements from the aligned base to the end
  mn = 0xFFFFFFFFu;
  mx = 0u;
#pragma unroll
  for (int q = 0; q < kRunsPerWarp; ++q) {
    const int64_t c = w * kRunsPerWarp + q;
    const int64_t b = ((span - 128) * c / (kChunks - 1)) & ~static_cast<int64_t>(3);
    float xv[4];
    Elem<T>::four_ldg(reinterpret_cast<const T*>(as) + b + 4 * lane, xv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t j = j0 + b + 4 * lane + i;
      const uint32_t key = (j >= 0 && j < L) ? to_key(xv[i]) : 0u;  // 0: below every key
      s.fkey[c * 128 + lane * 4 + i] = key;
      mn = min(mn, key);
      mx = max(mx, key);
    }
  }
  mn = __reduce_min_sync(kFull, mn);
  mx = __reduce_max_sync(kFull, mx);
  if (lane == 0) {
    s.fred[0][w] = mn;
    s.fred[1][w] = mx;
  }
  bar_filter();
  mn = __reduce_min_sync(kFull, lane < kFilterWarps ? s.fred[0][lane] : 0xFFFFFFFFu);
  mx = __reduce_max_sync(kFull, lane < kFilterWarps ? s.fred[1][lane] : 0u);
}

// A threshold for an item with no estimate, from a sample of kSampleVals
// values in kSampleChunks evenly spaced runs of 128 (aligned 16-byte blocks
// inside the item): the value with as many sampled values above it as 1.25
// times the share of m in the sample, plus 12. On a 128K-value row with k =
// 2048 that lets about 2.9K values through, some three standard deviations of
// the sample's count above m: a re-read is rare, and a looser margin costs
// more in candidate writes and compactions than it saves. With `few` (each
// CTA has at most two rows, so most rows sample) half as many values are
// sampled: the sample's cost then counts for more than the looser threshold;
// with many rows per CTA only a CTA's first row samples, and the rows after it
// start from thresholds carried from it. Returns -inf when the sample gives
// none.
template <class T>
__device__ __noinline__ float sample_threshold(const T* row, int64_t L, int m, int tid, bool few) {
  Smem& s = cta_smem();
  uint32_t mn, mx;
  int nvals;
  if (few) {
    sample_keys<T, kSampleRunsPerWarp / 2>(s, row, L, tid, mn, mx);
    nvals = kSampleVals / 2;
  } else {
    sample_keys<T, kSampleRunsPerWarp>(s, row, L, tid, mn, mx);
    nvals = kSampleVals;
  }
  const double share = static_cast<double>(nvals) * m / static_cast<double>(L);
  const uint32_t need = min(static_cast<uint32_t>(nvals - 8), static_cast<uint32_t>(1.25 * share) + 12u);
  const uint32_t T0 = sample_kth(s, nvals, need, mn, mx, tid);
  bar_filter();  // fkey, fidx, fred and bc are free again
  return (T0 == 0u || T0 >= kInfKey) ? __int_as_float(0xff800000) : from_key(T0);
}

// Consumer position in the ring.
struct RingPos {
  int slot;        // ring slot of the next stage
  uint32_t phase;  // its full-barrier phase parity
  uint32_t par;    // parity of the per-stage counts in s.red
};

// Streams one item (a row, or a rank's chunk of a row: L entries whose stored
// indices are base + item index) through the ring into the candidate buffer,
// starting from threshold f.t. A stage whose wait gave up counts as empty:
// after a timeout every wait of the CTA fails at once, so the loop runs out
// quickly through the same barriers as always, and the caller learns of it
// from the CTA's abort flag (a consensus at the next row or merge).
template <class T>
__device__ __forceinline__ void stream_item(Smem& s, Filter& f, RingPos& rp, const RowSpan& sp, int32_t L, uint32_t base,
                                            int m, int tid) {
  constexpr int kStages = stages_of<T>();
  const int w = tid >> 5, lane = tid & 31;
  int32_t sj0 = static_cast<int32_t>(sp.j0);  // item index of the stage's first element (< L <= INT32_MAX)
  for (int st = 0; st < sp.nst; ++st, sj0 += kStageElems) {
    const bool ok = mbar_wait(&s.full[rp.slot], rp.phase, &s.wait);
    // the pass mask, group by group as the values are loaded (values of a
    // stage that never came are unused)
    uint32_t msk = 0;
    {
      const T* rg = reinterpret_cast<const T*>(s.ring) + rp.slot * kStageElems + w * kWarpElems + lane * 4;
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        float x[4];
        Elem<T>::four(rg + q * 128, x);
#pragma unroll
        for (int i = 0; i < 4; ++i) msk |= static_cast<uint32_t>(!(x[i] < f.t)) << (4 * q + i);
      }
      if (st == 0 || st + 1 == sp.nst) {
        int lo, hi;
        stage_bounds(sj0, L, lo, hi);
        msk &= range_mask(w, lane, lo, hi);
      }
      if (!ok) msk = 0u;
    }
    publish(&s.red[rp.par][0], msk, w, lane);
    bar_filter();  // every warp's count of this stage is published
    const T* ring = reinterpret_cast<const T*>(s.ring) + rp.slot * kStageElems;
    take_stage<T, true>(s, f, &s.red[rp.par][0], ring, msk, base + static_cast<uint32_t>(sj0), m, tid);
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[rp.slot]);
    if (f.cnt > static_cast<uint32_t>(kTrigger)) compact_any(s, f, m, tid);
    tighten(f, m);
    rp.par ^= 1u;
    if (++rp.slot == kStages) {
      rp.slot = 0;
      rp.phase ^= 1u;
    }
  }
  // a snapshot of the abort flag, the same for every filter thread after the
  // barrier (the flag itself may be raised by another role at any time)
  if (tid == 0) s.abort_seen = *reinterpret_cast<volatile uint32_t*>(&s.wait.abort);
  bar_filter();  // every append is visible
}

// An item of one stage with no threshold yet (a short row): every value in
// [0, L) is a candidate, so the stage is copied into the candidate buffer in
// index order, coalesced, with no pass masks or survivor exchange. Out of
// line and outside the stage loop, so the streaming loop's code is untouched.
struct OpenItem {
  RingPos rp;    // the ring position after the stage
  uint32_t cnt;  // candidates taken (0 if the stage's wait gave up)
};

template <class T>
__device__ __noinline__ OpenItem stream_open(RingPos rp, int64_t j0, int32_t L, uint32_t base, int tid) {
  Smem& s = cta_smem();
  constexpr int kStages = stages_of<T>();
  const int lane = tid & 31;
  const bool ok = mbar_wait(&s.full[rp.slot], rp.phase, &s.wait);
  const T* ring = reinterpret_cast<const T*>(s.ring) + rp.slot * kStageElems - j0;  // ring[e]: item index e
  const int n = ok ? L : 0;
  for (int e = tid; e < n; e += kFilterThreads) {
    s.fkey[e] = to_key(Elem<T>::f(ring[e]));
    s.fidx[e] = base + static_cast<uint32_t>(e);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&s.empty[rp.slot]);
  rp.par ^= 1u;
  if (++rp.slot == kStages) {
    rp.slot = 0;
    rp.phase ^= 1u;
  }
  if (tid == 0) s.abort_seen = *reinterpret_cast<volatile uint32_t*>(&s.wait.abort);
  bar_filter();  // every append is visible
  return OpenItem{rp, static_cast<uint32_t>(n)};
}

// ---------------------------------------------------------- finisher
// Bounds on a candidate set known before its ranking starts: kmin <= every
// key <= kmax, every index <= imax, and kdiff has every bit in which two of
// the keys may differ.
struct KeyBounds {
  uint32_t kmin, kmax, imax, kdiff;
};

// Ranks candidates hkey/hidx [0, n) by the composite C = (kmax - key) << 32 |
// index (ascending C = key descending, index ascending; all C distinct) and
// writes the first m to the output row. Buckets are 12-bit slices of C: count,
// scan, then find the bucket holding rank m-1. While a bucket at or before it
// is large, the range shrinks to the buckets up to it (everything after has
// rank >= m) and the count repeats. Then the candidates are grouped by bucket
// and each one's rank is its bucket's start plus the number of bucket members
// ahead of it. In set mode (DSA_FLAG_UNSORTED) only the bucket holding rank
// m-1 is ranked; the rest of the top m is written in bucket order.
// NT threads (192: the finisher warps; 256: the filter warps of a cluster's
// leader) synchronise on named barrier BAR.
template <int NT, int BAR, bool kFromFilter = false>
struct Finisher {
  static constexpr int kWarps = NT / 32;
  // the candidates: the handover buffer, or (kFromFilter: a CTA's last row)
  // the filter's own buffer, left in place
  __device__ __forceinline__ static uint32_t* cand_key(Smem& s) { return kFromFilter ? s.fkey : s.hkey; }
  __device__ __forceinline__ static uint32_t* cand_idx(Smem& s) { return kFromFilter ? s.fidx : s.hidx; }
  static constexpr int kBuckets = kBucketMax / (4 * NT) * (4 * NT);  // 3840, 4096 or 3584
  static constexpr int kScanPer = kBuckets / NT;  // counters per thread
  static_assert(kBuckets <= kBucketMax && kBuckets >= 2048 && kScanPer % 4 == 0 &&
                    kWarps <= kFilterWarps + kFinishWarpsMax,
                "bucket counters split evenly over the threads; bucket_shift narrows a slice by one bit at most");

  __device__ __forceinline__ static void bar() { asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory"); }

  // per-warp reduction slot i of warp w
  __device__ __forceinline__ static uint32_t& nred(Smem& s, int i, int w) {
    if constexpr (kWarps > kNredWarps) {
      return w < kNredWarps ? s.nred[i][w] : s.nred_x[i];
    } else {
      return s.nred[i][w];
    }
  }

  __device__ __forceinline__ static int bucket_shift(uint64_t cmax) {
    const int bits = cmax ? 64 - __clzll(static_cast<long long>(cmax)) : 0;
    int sh = bits > 12 ? bits - 12 : 0;  // cmax >> sh < 4096
    if ((cmax >> sh) >= static_cast<uint64_t>(kBuckets)) ++sh;
    return sh;
  }

  // Ranks, position-parallel (used when the finisher runs alone, where its
  // latency is the kernel's tail): each warp takes 32 consecutive positions
  // of the bucket order (one per lane) up to the end of the bucket holding
  // rank m-1. A candidate's rank is its bucket's start plus the bucket members
  // that beat it; members in the same 32-position window come from the
  // neighbouring lanes by shuffles (only as far as the widest bucket of the
  // window), the few beyond the window from shared memory. In set mode only
  // the bucket holding rank m-1 is ranked; earlier positions stay as they lie.
  template <class Bucket>
  __device__ __forceinline__ static void rank_by_windows(Smem& s, int n, int m, int k, int a, uint32_t bm,
                                                         bool set_mode, Bucket bucket_of, int fid) {
    const int fw = fid >> 5, lane = fid & 31;
    const uint32_t qend = s.bcnt[bm];  // positions past this have rank >= m
    const uint32_t cut0 = bm ? s.bcnt[bm - 1] : 0u;
    for (uint32_t q0 = static_cast<uint32_t>(fw) * 32u; q0 < qend; q0 += kWarps * 32u) {
      const uint32_t q = q0 + lane;
      const bool v = q < qend;
      const uint32_t e = v ? s.perm[q] : 0u;
      const uint32_t key = v ? cand_key(s)[e] : 0u, idx = v ? cand_idx(s)[e] : 0xFFFFFFFFu;
      uint32_t s0 = q, s1 = q + 1;  // invalid lanes: a bucket of their own
      if (v) {
        uint32_t b;
        bucket_of(key, idx, b);
        s0 = b ? s.bcnt[b - 1] : 0u;
        s1 = s.bcnt[b];
      }
      uint32_t r = 0;
      const bool need = v && !(set_mode && s1 <= cut0) && s0 < static_cast<uint32_t>(m) && s1 - s0 > 1u;
      const uint32_t span = __reduce_max_sync(kFull, need ? s1 - s0 : 1u);
      for (uint32_t d = 1; d < span && d < 32u; ++d) {
        const uint32_t ku = __shfl_down_sync(kFull, key, d), iu = __shfl_down_sync(kFull, idx, d);
        const uint32_t kd = __shfl_up_sync(kFull, key, d), id = __shfl_up_sync(kFull, idx, d);
        if (need) {
          if (lane + d < 32u && q + d < s1) r += ku > key || (ku == key && iu < idx);
          if (lane >= d && q - d >= s0) r += kd > key || (kd == key && id < idx);
        }
      }
      if (need && (s0 < q0 || s1 > q0 + 32u)) {  // bucket members outside the window
        for (uint32_t q2 = s0; q2 < s1; ++q2) {
          if (q2 >= q0 && q2 < q0 + 32u) continue;
          const uint32_t j = s.perm[q2];
          const uint32_t kj = cand_key(s)[j], ij = cand_idx(s)[j];
          r += kj > key || (kj == key && ij < idx);
        }
      }
      if (v) {
        const uint32_t pos = (set_mode && s1 <= cut0) ? q : s0 + r;
        if (pos < static_cast<uint32_t>(m)) {
          s.ostage[pos] = static_cast<int32_t>(idx);
          if (pos == static_cast<uint32_t>(k - 1)) s.rec[0] = key;
          if (pos == static_cast<uint32_t>(a)) s.rec[1] = key;
        }
      }
    }
  }

  // Writes o[0 .. m) from the staged indices; the optional table maps a
  // row-local index to the caller's value (-1 passes through). With a table,
  // each thread first
  // issues eight independent table loads, then stores: the gathers overlap
  // instead of waiting one by one.
  __device__ __forceinline__ static void write_out(const int32_t* staged, int32_t* o, int m, int64_t row,
                                                   const Params& p, int fid) {
    if (p.table == nullptr) {
      for (int q = fid; q < m; q += NT) o[q] = staged[q];
      return;
    }
    const int32_t* trow = p.table + row * p.table_stride;
    for (int q0 = fid; q0 < m; q0 += 8 * NT) {
      int32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int q = q0 + u * NT;
        const int32_t idx = q < m ? staged[q] : -1;
        v[u] = idx >= 0 ? __ldg(trow + idx) : -1;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (q0 + u * NT < m) o[q0 + u * NT] = v[u];
    }
  }

  // One stable LSD pass per digit of up to eight of the bits `vary` of the
  // composite C = (kmax - key) << 32 | index, lowest bits first, moving the
  // permutation from *pa to *pb and swapping them. Each warp owns a contiguous range of the
  // current order. Counting needs no order: every lane adds one to its
  // warp's counter for its digit (16-bit counters, two to a word). The
  // scatter walks the warp's chunks of 32 in order; the lanes holding one
  // digit find one another through a per-warp lane-mask word per digit
  // (atomicOr, read back, cleared by the group's first lane), and take
  // consecutive places after that digit's running position. (One vote per
  // digit bit, or match.any, costs several times more here.) The masks are
  // zero on entry and on return.
  // Scratch of the sort passes: the bucket counters; with more than eight
  // warps, the handover buffer (hkey and hidx, contiguous) when the candidates
  // stay in the filter's buffer, else the filter's buffer.
  __device__ __forceinline__ static uint32_t* sort_scratch(Smem& s) {
    return kWarps > kFilterWarps ? (kFromFilter ? s.hkey : s.fkey) : s.bcnt;
  }
  __device__ __forceinline__ static void radix_passes(Smem& s, int n, uint32_t kmax, uint64_t vary,
                                                      uint16_t*& pa, uint16_t*& pb, int fid) {
    constexpr int kBins = 256;
    static_assert(kWarps * kBins + kWarps * kBins / 2 + kBins <= (kWarps > kFilterWarps ? 2 * kHandCap : kBucketMax) &&
                      kHandCap < 65536,
                  "lane masks, 16-bit digit counters and digit starts fit the sort scratch");
    const int fw = fid >> 5, lane = fid & 31;
    uint32_t* scr = sort_scratch(s);
    uint32_t* mw = scr + fw * kBins;  // this warp's lane masks
    uint32_t* cwords = scr + kWarps * kBins;
    uint32_t* cw = cwords + fw * (kBins / 2);                 // this warp's counters, as words
    uint16_t* ch = reinterpret_cast<uint16_t*>(cwords);       // [kWarps][kBins] counters
    uint16_t* mine = ch + fw * kBins;
    uint32_t* dbase = cwords + kWarps * (kBins / 2);          // [kBins] digit starts
    const int per = ((n + kWarps - 1) / kWarps + 31) & ~31;  // items per warp, whole chunks
    const int i0 = fw * per, i1 = min(n, i0 + per);
    const uint32_t lt = lanemask_lt();
    uint64_t rest = vary;
    while (rest != 0u) {
      // this pass's digit: the next eight (or fewer) bits of C that vary,
      // lowest first, across both halves (bits that are the same in every
      // candidate do not order them)
      uint64_t dm = 0u;
      int pos[8], nb = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pos[i] = 0;
        if (rest != 0u) {
          pos[i] = __ffsll(static_cast<long long>(rest)) - 1;
          dm |= 1ull << pos[i];
          rest &= rest - 1u;
          ++nb;
        }
      }
      const int p0 = pos[0];
      const bool run = ((dm >> p0) & ((dm >> p0) + 1u)) == 0u;  // the bits are contiguous
      auto digit = [&](uint32_t e) -> uint32_t {
        const uint64_t x = (static_cast<uint64_t>(kmax - cand_key(s)[e]) << 32) | cand_idx(s)[e];
        if (run) return static_cast<uint32_t>((x >> p0) & (dm >> p0));
        uint32_t d = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (i < nb) d |= static_cast<uint32_t>((x >> pos[i]) & 1u) << i;
        return d;
      };
      for (int d = lane; d < kBins / 2; d += 32) cw[d] = 0u;
      __syncwarp();
#pragma unroll 4
      for (int c0 = i0; c0 < i1; c0 += 32) {
        const int i = c0 + lane;
        if (i < i1) {
          const uint32_t d = digit(pa[i]);
          atomicAdd(&cw[d >> 1], 1u << (16u * (d & 1u)));
        }
      }
      bar();
      // digit totals; their exclusive scan (warp 0); each warp's start per digit
      for (int d = fid; d < kBins; d += NT) {
        uint32_t t = 0;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) t += ch[ww * kBins + d];
        dbase[d] = t;
      }
      bar();
      if (fw == 0) {
        constexpr int kPer = kBins / 32;
        uint32_t c[kPer], sum = 0;
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
          c[t] = dbase[kPer * lane + t];
          sum += c[t];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
          const uint32_t y = __shfl_up_sync(kFull, incl, o2);
          if (lane >= o2) incl += y;
        }
        uint32_t run = incl - sum;
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
          dbase[kPer * lane + t] = run;
          run += c[t];
        }
      }
      bar();
      for (int d = fid; d < kBins; d += NT) {
        uint32_t run = dbase[d];
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
          const uint32_t t = ch[ww * kBins + d];
          ch[ww * kBins + d] = static_cast<uint16_t>(run);
          run += t;
        }
      }
      bar();
      // scatter in order; the next chunk's item and digit are loaded ahead
      bool vn = i0 + lane < i1;
      uint32_t en = vn ? pa[i0 + lane] : 0u;
      uint32_t dn = vn ? digit(en) : 0u;
      for (int c0 = i0; c0 < i1; c0 += 32) {
        const bool v = vn;
        const uint32_t e = en, d = dn;
        vn = c0 + 32 + lane < i1;
        if (vn) {
          en = pa[c0 + 32 + lane];
          dn = digit(en);
        }
        if (v) atomicOr(&mw[d], 1u << lane);
        __syncwarp();
        const uint32_t peers = v ? mw[d] : 0u;
        const uint32_t base = v ? mine[d] : 0u;
        if (v) pb[base + __popc(peers & lt)] = static_cast<uint16_t>(e);
        __syncwarp();
        if (v && (peers & lt) == 0u) {
          mw[d] = 0u;
          mine[d] = static_cast<uint16_t>(base + __popc(peers));
        }
        __syncwarp();
      }
      bar();
      uint16_t* t = pa;
      pa = pb;
      pb = t;
    }
  }

  // Candidates with C <= cut (every rank below m among them) ordered by the
  // composite C = (kmax - key) << 32 | index (key descending, index
  // ascending) with a stable LSD radix sort of a 16-bit permutation, then the
  // first m written. Used when buckets stay crowded with equal keys (values
  // on a coarse grid, such as fp8 or bf16), where counting ranks inside a
  // bucket would be quadratic. The 8-bit digits are laid over the bits of C
  // that differ between the sorted candidates, across both halves (a 128K
  // row's 17 index bits and a bf16 grid's nine key bits take four passes).
  // Ends with a barrier.
  __device__ __noinline__ static void finish_sorted(int n, int m, int k, uint32_t kmax, uint64_t cut, int64_t row,
                                                    const Params p, int fid) {
    Smem& s = cta_smem();
    const int fw = fid >> 5, lane = fid & 31;
    int32_t* o = p.out + row * static_cast<int64_t>(k);
    uint16_t* pa = s.perm;
    uint16_t* pb = reinterpret_cast<uint16_t*>(s.ostage);  // 2 x kMaxK bytes = kHandCap entries
    uint32_t* scr = sort_scratch(s);
    for (int i = fid; i < kWarps * 256; i += NT) scr[i] = 0u;  // the radix passes' lane masks
    if (fid == 0) s.bc[6] = 0u;
    bar();
    // the candidates to sort, and the bits of C that vary among them (from
    // the OR and AND of its two halves)
    uint32_t or_hi = 0u, and_hi = 0xFFFFFFFFu, or_lo = 0u, and_lo = 0xFFFFFFFFu;
    const uint32_t lt = lanemask_lt();
    for (int e0 = 0; e0 < n; e0 += NT) {  // warp-uniform trip count
      const int e = e0 + fid;
      bool keep = false;
      uint32_t hi = 0u, lo = 0u;
      if (e < n) {
        hi = kmax - cand_key(s)[e];
        lo = cand_idx(s)[e];
        keep = ((static_cast<uint64_t>(hi) << 32) | lo) <= cut;
      }
      const uint32_t b = __ballot_sync(kFull, keep);
      uint32_t base = 0u;
      if (lane == 0 && b) base = atomicAdd(&s.bc[6], static_cast<uint32_t>(__popc(b)));
      base = __shfl_sync(kFull, base, 0);
      if (keep) {
        pa[base + __popc(b & lt)] = static_cast<uint16_t>(e);
        or_hi |= hi;
        and_hi &= hi;
        or_lo |= lo;
        and_lo &= lo;
      }
    }
    or_hi = __reduce_or_sync(kFull, or_hi);
    and_hi = __reduce_and_sync(kFull, and_hi);
    or_lo = __reduce_or_sync(kFull, or_lo);
    and_lo = __reduce_and_sync(kFull, and_lo);
    if (lane == 0) {
      nred(s, 0, fw) = or_hi;
      nred(s, 1, fw) = and_hi;
      nred(s, 2, fw) = or_lo;
      nred(s, 3, fw) = and_lo;
    }
    bar();
    const int ns = static_cast<int>(s.bc[6]);
    uint32_t vhi = 0u, vlo = 0u;
    {
      uint32_t a0 = 0u, a1 = 0xFFFFFFFFu, b0 = 0u, b1 = 0xFFFFFFFFu;
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        a0 |= nred(s, 0, ww);
        a1 &= nred(s, 1, ww);
        b0 |= nred(s, 2, ww);
        b1 &= nred(s, 3, ww);
      }
      vhi = a0 & ~a1;
      vlo = b0 & ~b1;
    }
    // one digit sequence over the varying bits of the whole composite (a digit
    // may take the index's last bits and the key's first)
    radix_passes(s, ns, kmax, (static_cast<uint64_t>(vhi) << 32) | vlo, pa, pb, fid);
    const int a = k >= 4 ? (3 * k) / 4 - 1 : 0;
    if (fid == 0) {
      if (m == k) s.rec[0] = cand_key(s)[pa[k - 1]];
      if (a < m) s.rec[1] = cand_key(s)[pa[a]];
    }
    // the sorted order's first m indices (the permutation buffer may be the
    // output stage, so it is read, not staged)
    if (p.table == nullptr) {
      for (int q = fid; q < m; q += NT) o[q] = static_cast<int32_t>(cand_idx(s)[pa[q]]);
    } else {
      const int32_t* trow = p.table + row * p.table_stride;
      for (int q = fid; q < m; q += NT) o[q] = __ldg(trow + cand_idx(s)[pa[q]]);
    }
    bar();
  }

  // Ranks n candidates and writes the row: m indices, then -1 up to k.
  // `alone`: nothing else runs on the SM meanwhile (a CTA's last row, a
  // cluster's leader).
  // (Inlined into the finisher warps' loop; a call there cost a few percent.)
  // kb: NULL, or bounds the caller already holds; then the pass that finds
  // them is skipped (looser bounds than the pass would find only change which
  // exact method is picked below)
  __device__ __forceinline__ static void finish(Smem& s, int n, int m, int k, int64_t row, const Params& p, int fid,
                                                bool alone, const KeyBounds* kb = nullptr) {
    const int fw = fid >> 5, lane = fid & 31;
    int32_t* o = p.out + row * static_cast<int64_t>(k);
    for (int q = m + fid; q < k; q += NT) o[q] = -1;
    if (n <= 0) return;
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u, imax = 0u, kdiff = 0u;
    if (kb != nullptr) {
      kmin = kb->kmin;
      kmax = kb->kmax;
      imax = kb->imax;
      kdiff = kb->kdiff;
    } else {
      const uint32_t key0 = cand_key(s)[0];
      for (int e = fid; e < n; e += NT) {
        const uint32_t key = cand_key(s)[e];
        kmin = min(kmin, key);
        kmax = max(kmax, key);
        kdiff |= key ^ key0;
        imax = max(imax, cand_idx(s)[e]);
      }
      kmin = __reduce_min_sync(kFull, kmin);
      kmax = __reduce_max_sync(kFull, kmax);
      imax = __reduce_max_sync(kFull, imax);
      kdiff = __reduce_or_sync(kFull, kdiff);
      if (lane == 0) {
        nred(s, 0, fw) = kmin;
        nred(s, 1, fw) = kmax;
        nred(s, 2, fw) = imax;
        nred(s, 3, fw) = kdiff;
      }
      bar();
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        kmin = min(kmin, nred(s, 0, ww));
        kmax = max(kmax, nred(s, 1, ww));
        imax = max(imax, nred(s, 2, ww));
        kdiff |= nred(s, 3, ww);
      }
    }
    // every two keys differ by a multiple of 2^grid (keys on a value grid,
    // such as fp8 or bf16 values, have zero low bits): buckets no wider than
    // that hold one key each, and finer passes cannot split them
    const int grid = kdiff ? __ffs(kdiff) - 1 : 32;
    uint64_t cmax = (static_cast<uint64_t>(kmax - kmin) << 32) | imax;
    int sh = bucket_shift(cmax);
    auto comp = [&](uint32_t key, uint32_t idx) -> uint64_t {
      return (static_cast<uint64_t>(kmax - key) << 32) | idx;
    };
    // A row ranked alone (its latency is the kernel's tail) takes a first
    // pass that buckets linearly in the value when the keys are off a coarse
    // grid and their range is finite: smooth logits then rarely need a second
    // pass, where 12-bit slices of a key range spanning both signs
    // crowd most values into a few buckets. Still exact: the bucket is a
    // monotone function of the key (correctly rounded steps), and the members
    // of one bucket are ranked by comparison. A first pass that leaves a
    // bucket crowded hands over to the slices of the composite.
    const float vtop = from_key(kmax), vlow = from_key(kmin);
    float scale = 0.f;
    bool lin = alone && grid < 8 && vtop > vlow && isfinite(vtop) && isfinite(vlow);
    if (lin) {
      scale = static_cast<float>(kBuckets - 1) / (vtop - vlow);
      lin = isfinite(scale) && scale > 0.f;
    }
    // bucket b of a candidate; false: past the range counted (after bm)
    auto bucket_of = [&](uint32_t key, uint32_t idx, uint32_t& b) -> bool {
      if (lin) {
        const float d = (vtop - from_key(key)) * scale;
        b = d < static_cast<float>(kBuckets - 1) ? static_cast<uint32_t>(d) : static_cast<uint32_t>(kBuckets - 1);
        return true;
      }
      const uint64_t c = comp(key, idx);
      b = static_cast<uint32_t>(c >> sh);
      return c <= cmax;
    };
    uint4* bc4 = reinterpret_cast<uint4*>(&s.bcnt[fid * kScanPer]);
    const uint32_t mm1 = static_cast<uint32_t>(m - 1);
    uint32_t big = 0;
    for (int pass = 0;; ++pass) {
#pragma unroll
      for (int i = 0; i < kScanPer / 4; ++i) bc4[i] = make_uint4(0u, 0u, 0u, 0u);
      bar();
      for (int e = fid; e < n; e += NT) {
        uint32_t b;
        if (bucket_of(cand_key(s)[e], cand_idx(s)[e], b)) atomicAdd(&s.bcnt[b], 1u);
      }
      bar();
      // exclusive scan: thread fid owns counters [kScanPer fid, kScanPer (fid + 1))
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
      if (lane == 31) nred(s, 3, fw) = incl;
      bar();
      uint32_t run = incl - sum;
      for (int ww = 0; ww < fw; ++ww) run += nred(s, 3, ww);
      const uint32_t run0 = run;
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
      run = run0;
#pragma unroll
      for (int i = 0; i < kScanPer; ++i) {
        if (run <= mm1 && mm1 < run + c[i]) s.bc[4] = static_cast<uint32_t>(fid * kScanPer + i);
        run += c[i];
      }
      bar();
      const uint32_t bm = s.bc[4];
      big = 0;  // largest bucket at or before bm
#pragma unroll
      for (int i = 0; i < kScanPer; ++i)
        if (static_cast<uint32_t>(fid * kScanPer + i) <= bm) big = max(big, c[i]);
      big = __reduce_max_sync(kFull, big);
      if (lane == 0) nred(s, 4, fw) = big;
      bar();
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) big = max(big, nred(s, 4, ww));
      // a bucket still crowded past the counting limit after a second, finer
      // pass holds values on a coarse grid (equal keys), which finer slices of
      // the same composite range do not split: sort instead (the first pass
      // alone can be coarse when the keys span both signs)
      if (big <= static_cast<uint32_t>(kSmallBucket)) break;
      if (lin) {  // crowded after the value-linear pass: the composite slices from the start
        lin = false;
        pass = -1;
        bar();  // bc[4] and nred[4] are rewritten by the next pass
        continue;
      }
      if ((big > static_cast<uint32_t>(kBigBucket) && (pass >= 1 || sh <= 32 + grid)) || sh == 0 ||
          pass == kSortPasses - 1)
        break;
      cmax = ((static_cast<uint64_t>(bm) + 1u) << sh) - 1u;
      sh = bucket_shift(cmax);
      bar();  // bc[4] and nred[4] are rewritten by the next pass
    }
    if (big > static_cast<uint32_t>(kBigBucket)) {
      // many candidates share a bucket (values on a coarse grid): counting
      // ranks inside it would be quadratic, so sort instead, everything up to
      // the end of the bucket holding rank m-1
      finish_sorted(n, m, k, kmax, ((static_cast<uint64_t>(s.bc[4]) + 1u) << sh) - 1u, row, p, fid);
      return;
    }
    for (int e = fid; e < n; e += NT) {
      uint32_t b;
      if (!bucket_of(cand_key(s)[e], cand_idx(s)[e], b)) continue;
      const uint32_t q = atomicAdd(&s.bcnt[b], 1u);
      s.perm[q] = static_cast<uint16_t>(e);
    }
    bar();  // bcnt[b] is now the end of bucket b (= start of b + 1)
    const int a = k >= 4 ? (3 * k) / 4 - 1 : 0;
    const uint32_t bm = s.bc[4];
    const bool set_mode = (p.flags & kUnsorted) != 0u;
    if (alone && n > 2 * m) {
      // nothing overlaps this row, and most candidates rank past m: ranking
      // only the positions before m is fastest (the per-candidate loop below
      // takes the fewest issue slots, which counts while rows still stream)
      rank_by_windows(s, n, m, k, a, bm, set_mode, bucket_of, fid);
    } else if (set_mode) {
      // set mode: positions before the bucket holding rank m-1 are taken as
      // they lie (bucket order); only that bucket's members are ranked
      const uint32_t s0 = bm ? s.bcnt[bm - 1] : 0u, s1 = s.bcnt[bm];
      for (uint32_t q = fid; q < s0; q += NT) {
        const uint32_t e = s.perm[q];
        s.ostage[q] = static_cast<int32_t>(cand_idx(s)[e]);
        if (q == static_cast<uint32_t>(a)) s.rec[1] = cand_key(s)[e];
      }
      for (uint32_t q = s0 + fid; q < s1; q += NT) {
        const uint32_t e = s.perm[q];
        const uint32_t key = cand_key(s)[e], idx = cand_idx(s)[e];
        uint32_t r = s0;
        for (uint32_t q2 = s0; q2 < s1; ++q2) {
          const uint32_t j = s.perm[q2];
          const uint32_t kj = cand_key(s)[j], ij = cand_idx(s)[j];
          r += kj > key || (kj == key && ij < idx);
        }
        if (r < static_cast<uint32_t>(m)) {
          s.ostage[r] = static_cast<int32_t>(idx);
          if (r == static_cast<uint32_t>(k - 1)) s.rec[0] = key;
          if (r == static_cast<uint32_t>(a)) s.rec[1] = key;
        }
      }
    } else {
      // each candidate: its bucket's start plus the bucket members ahead of it
      for (int e = fid; e < n; e += NT) {
        const uint32_t key = cand_key(s)[e], idx = cand_idx(s)[e];
        uint32_t b;
        if (!bucket_of(key, idx, b)) continue;
        const uint32_t s0 = b ? s.bcnt[b - 1] : 0u, s1 = s.bcnt[b];
        if (s0 >= static_cast<uint32_t>(m)) continue;
        uint32_t r = s0;
        for (uint32_t q = s0; q < s1; ++q) {
          const uint32_t j = s.perm[q];
          const uint32_t kj = cand_key(s)[j], ij = cand_idx(s)[j];
          r += kj > key || (kj == key && ij < idx);
        }
        if (r < static_cast<uint32_t>(m)) {
          s.ostage[r] = static_cast<int32_t>(idx);
          if (r == static_cast<uint32_t>(k - 1)) s.rec[0] = key;
          if (r == static_cast<uint32_t>(a)) s.rec[1] = key;
        }
      }
    }
    bar();
    write_out(s.ostage, o, m, row, p, fid);
  }
};

template <class T>
using RowFinisher = Finisher<finish_threads<T>(), 2>;
// the filter warps' own ranking of a cluster leader's row
using LeaderFinisher = Finisher<kFilterThreads, 1>;
// a CTA's last row, ranked by the filter and finisher warps together
template <class T>
using JointFinisher = Finisher<joint_threads<T>(), 3, true>;

// Where the filter and finisher warps meet after their row loops. Both roles reach it on every path (a wait that gave up ends a
// loop early; no loop ends without passing here), so the hardware barrier
// always completes, and the flag the filter warps wrote before it (s.joint)
// decides for both whether they rank the row together.
template <class T>
__device__ __forceinline__ void joint_rendezvous() {
  asm volatile("bar.sync 3, %0;" ::"n"(joint_threads<T>()) : "memory");
}

// The joint ranking, out of line (inlined into the row loops, its registers
// would be allocated with theirs).
template <class T>
__device__ __noinline__ void joint_finish(const Params p, int tid) {
  Smem& s = cta_smem();
  JointFinisher<T>::finish(s, s.h_n, s.h_m, p.k, s.h_row, p, tid, true);
}



// kShort: the launch's row stride fits one stage (every row is one item of
// one stage), and rows with no threshold take the stage whole (stream_open).
// A separate kernel instance, so longer rows run unchanged code.
template <class T, bool kShort>
__device__ void filter_loop(Smem& s, const Params& p, int tid) {
  const int lane = tid & 31;
  const T* logits = static_cast<const T*>(p.logits);
  const int k = p.k;
  RingPos rp{0, 0u, 0u};
  Filter f;
  f.par = 0;
  int h = 0;
  int64_t row = blockIdx.x;
  int32_t L_next = row < p.num_rows ? static_cast<int32_t>(clamp_len(p.lengths, row, p.row_stride)) : 0;
  for (; row < p.num_rows; row += gridDim.x, ++h) {
    if (s.abort_seen) break;  // a wait gave up during the previous row: the filter warps leave together
    const int32_t L = L_next;  // lengths are int32, so is every clamped length
    if (row + gridDim.x < p.num_rows)
      L_next = static_cast<int32_t>(clamp_len(p.lengths, row + gridDim.x, p.row_stride));
    const int m = static_cast<int>(min64(k, L));
    const T* rowp = logits + row * p.row_stride;
    const RowSpan sp = row_span(rowp, L);
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
      const float ts = sample_threshold(rowp, L, m, tid, p.num_rows <= 2 * static_cast<int64_t>(gridDim.x));
      if (ts > __int_as_float(0xff800000)) {
        spec = true;
        f.t = ts;
      }
    }
    if (tid == 0) s.row_t0 = f.t;  // the row's initial threshold (read by thread 0 at the row's end)
    f.cnt = 0;
    f.compacted = false;
    f.strict = false;
    f.bounded = false;
    if (kShort && sp.nst == 1 && !spec) {
      const OpenItem o = stream_open<T>(rp, sp.j0, L, 0u, tid);
      rp = o.rp;
      f.cnt = o.cnt;
      tighten(f, m);
    } else {
      stream_item<T>(s, f, rp, sp, L, 0u, m, tid);
    }
    const bool reread = spec && !f.compacted && f.cnt < static_cast<uint32_t>(m) && !s.abort_seen;
    if (reread) {
      if (tid == 0) atomicOr(&g_status, kStatusReread);
      f = refilter_from_global<T>(s, f, sp, L, 0u, m, tid);
    }
    if (f.cnt > static_cast<uint32_t>(kHandCap)) compact_any(s, f, m, tid);
    if (tid == 0 && m == k) {
      // carried to the CTA's next row: a speculative threshold that passed at
      // least m values of this row (it needed no re-read), else the bound the
      // filter ended with. A compaction's cut is a poor carry: it can sit
      // just under this row's m-th value and above a similar row's.
      if (spec && !reread) {
        s.own_key = to_key(s.row_t0);
        s.own_len = L;
      } else if (f.bounded) {
        s.own_key = f.last_key;
        s.own_len = L;
      }
    }
    bar_filter();  // the own estimate is read at the next row's start; every append is visible
    if (row + gridDim.x >= p.num_rows) {
      // the CTA's last row: the finisher warps stop after the row before it
      // and nothing else is left to stream, so both roles rank this one
      // together after the rendezvous, from the filter's buffer (more
      // threads, no handover copy)
      if (tid == 0) {
        s.h_row = row;
        s.h_n = static_cast<int32_t>(f.cnt);
        s.h_m = m;
        s.joint = 1u;
      }
      break;
    }
    // hand over: wait until the finishers released the previous handover (a
    // wait that gave up hands over regardless; the row's output is undefined)
    mbar_wait_sleep(&s.hempty, (h & 1) ^ 1, &s.wait);
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
  joint_rendezvous<T>();
  if (s.joint) joint_finish<T>(p, tid);
}


// The estimate the filter starts a later row from: the k-th value minus half
// the gap to the 3k/4-th, and at least one step (two for 16-bit values) of
// the element type's value grid below the k-th (a coarse grid, such as bf16
// logits, often puts both ranks on one value; an estimate equal to the k-th
// value then lets too few values of a similar row through and forces a
// re-read).
template <class T>
__device__ __forceinline__ float row_estimate(float vt, float va) {
  constexpr int kMantissa = sizeof(T) == 4 ? 23 : (Elem<T>::kCode == DSA_DTYPE_BF16 ? 7 : 10);
  const float step = fabsf(vt) * (1.0f / static_cast<float>(1 << kMantissa));
  return vt - fmaxf(0.5f * (va - vt), (sizeof(T) == 4 ? 1.0f : 2.0f) * step);
}

template <class T>
__device__ void finish_loop(Smem& s, const Params& p, int fid) {
  const int lane = fid & 31;
  const int k = p.k;
  int h = 0;
  // rows up to, not including, the CTA's last (which the filter warps rank,
  // alone or with these warps)
  for (int64_t row = blockIdx.x; row + gridDim.x < p.num_rows; row += gridDim.x, ++h) {
    const bool ok = mbar_wait_sleep(&s.hfull, h & 1, &s.wait);
    if (bar_any<2, finish_threads<T>()>(!ok)) break;  // the filter warps left: nothing more comes
    const int n = s.h_n, m = s.h_m;
    const int64_t L = s.h_len;
    RowFinisher<T>::finish(s, n, m, k, s.h_row, p, fid, false);
    if (fid == 0) {
      bool est_ok = false;
      float e = 0.f;
      if (n > 0 && m == k) {
        const uint32_t kt = s.rec[0], ka = s.rec[1];
        const float vt = from_key(kt), va = from_key(ka);
        e = row_estimate<T>(vt, va);
        est_ok = kt != kNanKey && ka != kNanKey && isfinite(e);
      }
      s.est[h & 1] = e;
      s.est_len[h & 1] = L;
      s.est_ok[h & 1] = est_ok ? 1 : 0;
    }
    RowFinisher<T>::bar();  // every read of the handover is done, the estimate written
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.hempty);
  }
  joint_rendezvous<T>();
  if (s.joint) joint_finish<T>(p, kFilterThreads + fid);
}

// ---------------------------------------------------------- producer
// Issues stages [st0, st1) of an item into the ring. Returns false when a wait
// gave up.
template <class T>
__device__ __forceinline__ bool produce_stages(Smem& s, const RowSpan& sp, int st0, int st1, int& slot, uint32_t& phase,
                                               long long& gi, long long skip, uint32_t& armed, uint32_t& arm_par) {
  constexpr int kStages = stages_of<T>();
  constexpr uint32_t kStageBytes = kStageElems * sizeof(T);
  for (int st = st0; st < st1; ++st, ++gi) {
    if (!mbar_wait_sleep(&s.empty[slot], phase ^ 1u, &s.wait)) return false;
    if (gi != skip) {
      const uint32_t bytes = st + 1 == sp.nst ? sp.last_bytes : kStageBytes;
      fence_proxy_async();
      mbar_arrive_expect_tx(&s.full[slot], bytes);
      bulk_g2s(s.ring + static_cast<uint32_t>(slot) * kStageBytes, sp.src + static_cast<uint64_t>(st) * kStageBytes,
               bytes, &s.full[slot]);
      armed |= 1u << slot;
      arm_par = (arm_par & ~(1u << slot)) | (phase << slot);
    }
    if (++slot == kStages) {
      slot = 0;
      phase ^= 1u;
    }
  }
  return true;
}

// Issues one item's stages into the ring. Returns false when a wait gave up.
template <class T>
__device__ __forceinline__ bool produce_span(Smem& s, const RowSpan& sp, int& slot, uint32_t& phase, long long& gi,
                                             long long skip, uint32_t& armed, uint32_t& arm_par) {
  return produce_stages<T>(s, sp, 0, sp.nst, slot, phase, gi, skip, armed, arm_par);
}

// Before returning, on the normal path and after an abort alike, the producer
// waits until the last copy it issued into each slot has landed, so the CTA
// never exits with a bulk copy still writing into its shared memory.
__device__ __forceinline__ void producer_drain(Smem& s, uint32_t armed, uint32_t arm_par) {
  for (int i = 0; i < kMaxStages; ++i)
    if ((armed >> i) & 1u) mbar_drain(&s.full[i], (arm_par >> i) & 1u, &s.wait);
}

template <class T>
__device__ void produce_loop(Smem& s, const Params& p) {
  const T* logits = static_cast<const T*>(p.logits);
  int slot = 0;
  uint32_t phase = 0u, armed = 0u, arm_par = 0u;
  const long long skip = g_skip_stage;  // test hook: a stage left unissued
  long long gi = 0;                     // stages this CTA has passed (issued or skipped)
  for (int64_t row = blockIdx.x; row < p.num_rows; row += gridDim.x) {
    const int64_t L = clamp_len(p.lengths, row, p.row_stride);
    if (!produce_span<T>(s, row_span(logits + row * p.row_stride, L), slot, phase, gi, skip, armed, arm_par)) break;
  }
  producer_drain(s, armed, arm_par);
}

// ---------------------------------------------------------- cluster mode
constexpr uint32_t kMergeRetry = 0xFFFFFFFFu;
constexpr int kMaxClusterSize = 16;  // the largest cluster the host plans
constexpr int kSampleBars = 3;       // cluster barriers of cluster_threshold, on every path

// Sum over the cluster's ranks of bin tid of the 256-bin histogram ph (the
// same shared-memory offset in every rank). The remote loads are all issued
// before any is summed: one at a time, each load's round trip would add up
// across the cluster.
__device__ __forceinline__ uint32_t cluster_bin_sum(const uint32_t* ph, uint32_t ncta, int tid) {
  const uint32_t a = smem_addr(&ph[tid]);
  uint32_t v[kMaxClusterSize];
#pragma unroll
  for (int r = 0; r < kMaxClusterSize; ++r) v[r] = static_cast<uint32_t>(r) < ncta ? dsmem_ld(dsmem_map(a, r)) : 0u;
  uint32_t g = 0;
#pragma unroll
  for (int r = 0; r < kMaxClusterSize; ++r) g += v[r];
  return g;
}

// One threshold for a whole cluster-split row, from every rank's sample: each
// rank with a chunk of at least kSampleMinLen samples 1024 of its values (one
// run of 128 per filter warp); the ranks publish their sample counts and key
// bounds, then two cluster-wide 256-bin histogram rounds narrow the bin that
// holds the need-th largest of all samples, need being the sample's share of
// m with the margin of the single-row threshold (1.25 x + 12). Keys at or
// above the final bin's lower edge number at least `need` among the samples;
// on a row of 900K values with m = 1024 the threshold lets about 1.9K values
// through in total, where a threshold from each rank's own sample must let
// m-plus-margin through in every rank (a rank's chunk may hold the whole top
// m). Every rank computes the same threshold from the same sums, which is
// what lets the merge check it: if the ranks together hold at least m values
// at or above it, those contain the row's top m.
// Returns -inf when the samples give no threshold above -inf (or one at or
// above +inf). Runs exactly kSampleBars cluster barriers on every path (the
// producer warpgroup runs as many). The histograms go in the merge's slots of
// bcnt, which the filter warps leave alone until the merge, whose first
// cluster barrier every rank reaches only after it has read them.
template <class T>
__device__ __noinline__ float cluster_threshold(const T* chunk, int64_t Lc, int64_t L, uint32_t m, uint32_t ncta,
                                                int tid) {
  Smem& s = cta_smem();
  const int w = tid >> 5, lane = tid & 31;
  constexpr uint32_t kRankVals = kFilterWarps * 128;
  uint32_t mn = 0xFFFFFFFFu, mx = 0u, ns = 0u;
  if (Lc >= kSampleMinLen) {
    sample_keys<T, 1>(s, chunk, Lc, tid, mn, mx);
    ns = kRankVals;
  }
  if (tid == 0) {
    s.spub[0] = ns;
    s.spub[1] = mn;
    s.spub[2] = mx;
  }
  cluster_barrier();
  if (w == 0) {
    uint32_t n = 0, lo_r = 0xFFFFFFFFu, hi_r = 0u;
    if (lane < static_cast<int>(ncta)) {
      const uint32_t a = dsmem_map(smem_addr(&s.spub[0]), lane);
      n = dsmem_ld(a);
      lo_r = dsmem_ld(a + 4);
      hi_r = dsmem_ld(a + 8);
    }
    n = __reduce_add_sync(kFull, n);
    lo_r = __reduce_min_sync(kFull, lo_r);
    hi_r = __reduce_max_sync(kFull, hi_r);
    if (lane == 0) {
      s.bc[2] = n;
      s.bc[3] = lo_r;
      s.bc[4] = hi_r;
    }
  }
  bar_filter();
  const uint32_t N = s.bc[2];
  uint32_t lo = s.bc[3], hi = s.bc[4];
  const double share = static_cast<double>(N) * m / static_cast<double>(L);
  uint32_t need = N > 16u ? min(N - 8u, static_cast<uint32_t>(1.25 * share) + 12u) : 0u;
  bool ok = need > 0u;  // the same in every rank (N, m and L are)
  uint32_t* ghist = s.bcnt + 512;
#pragma unroll 1
  for (int round = 0; round < kSampleBars - 1; ++round) {
    uint32_t* ph = s.bcnt + 256 * round;
    const bool live = ok && lo != hi;
    const int sh = live ? window_shift(lo, hi) : 0;
    ph[tid] = 0u;  // kFilterThreads == 256
    if (tid == 0) s.bc[0] = 0xFFFFFFFFu;
    bar_filter();
    if (live) digit_histogram(ph, static_cast<int>(ns), FKey{&s}, FAll{}, lo, hi, sh, tid);
    cluster_barrier();
    if (live) {
      ghist[tid] = cluster_bin_sum(ph, ncta, tid);
      bar_filter();
      if (w == 0) find_bucket_warp0(ghist, need, s.bc, lane);
      bar_filter();
      const uint32_t b = s.bc[0];
      if (b == 0xFFFFFFFFu) {  // the same sums in every rank: the same outcome
        ok = false;
      } else {
        need -= s.bc[1];
        narrow(lo, hi, sh, b);
      }
    }
    bar_filter();  // bc and ghist are rewritten by the next round
  }
  return (ok && lo > to_key(__int_as_float(0xff800000)) && lo < kInfKey) ? from_key(lo) : __int_as_float(0xff800000);
}

// After streaming, rank `rank` holds n_r candidates in fkey/fidx (none if a
// wait gave up): every value of its chunk at or above the row's threshold,
// or, once the rank compacted, a superset of its chunk's top min(m, chunk).
// The filter warps of every rank run the merge; at the leader (rank 0) the
// survivors end in hkey/hidx. Returns the number gathered there, or
// kMergeRetry when some rank's threshold was a guess (guessed) and the ranks
// together hold fewer than m: then every rank takes its chunk again with no
// threshold and merges once more. The producer warp mirrors every cluster
// barrier (s.final_bar tells it how many there are).
__device__ __noinline__ uint32_t cluster_merge(uint32_t n_r, uint32_t m, bool aborted, bool guessed, uint32_t rank,
                                               uint32_t ncta, int tid) {
  Smem& s = cta_smem();
  const int w = tid >> 5, lane = tid & 31;
  uint32_t nbar = s.merge_bars;
  uint32_t* phist = s.bcnt;        // [2][256], per rank, read by the others
  uint32_t* ghist = s.bcnt + 512;  // [256], cluster sums
  // ---- phase 1: publish (count, min key, max key, gave up, guessed, the
  // bits in which a key differs from the max) of this rank
  uint32_t mn, mx;
  filter_minmax(s, static_cast<int>(n_r), FKey{&s}, FAll{}, mn, mx, tid);
  uint32_t kd = 0u;
  for (int e = tid; e < static_cast<int>(n_r); e += kFilterThreads) kd |= s.fkey[e] ^ mx;
  kd = __reduce_or_sync(kFull, kd);
  if (lane == 0) s.fred[2][w] = kd;
  bar_filter();
  kd = __reduce_or_sync(kFull, lane < kFilterWarps ? s.fred[2][lane] : 0u);
  if (tid == 0) {
    s.pub[7] = kd;
    s.pub[0] = n_r;
    s.pub[1] = mn;
    s.pub[2] = mx;
    s.pub[3] = aborted ? 1u : 0u;
    s.pub[6] = guessed ? 1u : 0u;
  }
  cluster_barrier();
  ++nbar;
  if (w == 0) {
    uint32_t n = 0, lo_r = 0xFFFFFFFFu, hi_r = 0u, ab = 0u, op = 0u;
    if (lane < static_cast<int>(ncta)) {
      const uint32_t a = dsmem_map(smem_addr(&s.pub[0]), lane);
      n = dsmem_ld(a);
      lo_r = dsmem_ld(a + 4);
      hi_r = dsmem_ld(a + 8);
      ab = dsmem_ld(a + 12);
      op = dsmem_ld(a + 24);
      kd = dsmem_ld(a + 28);
    }
    const bool full_rank = lane < static_cast<int>(ncta) && n >= m;
    const uint32_t N = __reduce_add_sync(kFull, n);
    const uint32_t gmin = __reduce_min_sync(kFull, lo_r);
    const uint32_t gmax = __reduce_max_sync(kFull, hi_r);
    // a rank holding at least m entries at or above its min bounds the m-th key from below
    const uint32_t B = __reduce_max_sync(kFull, full_rank ? lo_r : 0u);
    const bool any_full = __ballot_sync(kFull, full_rank) != 0;
    const bool any_ab = __ballot_sync(kFull, ab != 0u) != 0;
    const bool any_guess = __ballot_sync(kFull, op != 0u) != 0;
    // bits in which two candidates of the cluster may differ (the leader's
    // ranking detects a value grid from them)
    const uint32_t kdall = __reduce_or_sync(kFull, n > 0u ? (kd | (hi_r ^ gmax)) : 0u);
    if (lane == 0) {
      s.bc[2] = N;
      s.bc[3] = any_full ? B : gmin;
      s.bc[4] = gmax;
      s.bc[5] = gmin;
      s.spub[3] = kdall;  // read below and by the leader's ranking
      s.abort_any = any_ab ? 1u : 0u;
      // fewer than m candidates under a guessed threshold: values below it
      // are needed, so every rank takes its chunk again with no threshold
      s.merge_retry = (any_guess && N < m && !any_ab) ? 1u : 0u;
    }
  }
  bar_filter();
  const uint32_t N = s.bc[2];
  uint32_t lo = s.bc[3], hi = s.bc[4];
  const uint32_t gmin = s.bc[5];
  const bool retry = s.merge_retry != 0u;
  bar_filter();
  if (retry) {
    cluster_barrier();  // every rank has read the published values before they change
    ++nbar;
    if (tid == 0) s.merge_bars = nbar;
    bar_filter();
    return kMergeRetry;
  }
  uint32_t need = m;
  bool exact = false;
  // Everything goes to the leader when it fits, unless the candidates sit on
  // a coarse value grid (keys differing only from bit 8 up, as bf16 values
  // do) and number more than m by an eighth: then at least one round narrows
  // them, usually to m plus one tied level (a leader ranking twice m tied
  // candidates costs more than the round; off a grid it costs less)
  const uint32_t kdg = s.spub[3];  // the key-difference bits, the same in every rank
  const bool coarse = kdg == 0u || __ffs(kdg) - 1 >= 8;
  if (N <= static_cast<uint32_t>(kHandCap) && (N <= m + (m >> 3) || !coarse)) {
    lo = gmin;
  } else {
    // ---- phase 2: cluster-wide histogram rounds until the survivors fit
    int hp = 0;
    for (int round = 0;; ++round) {
      if (lo == hi || round == kRounds + 1) {
        if (lo != hi && tid == 0) atomicOr(&g_status, kStatusSelectBroken);
        exact = true;
        break;
      }
      const int sh = window_shift(lo, hi);
      uint32_t* ph = phist + 256 * hp;
      ph[tid] = 0u;  // kFilterThreads == 256
      if (tid == 0) s.bc[0] = 0xFFFFFFFFu;
      bar_filter();
      digit_histogram(ph, static_cast<int>(n_r), FKey{&s}, FAll{}, lo, hi, sh, tid);
      cluster_barrier();
      ++nbar;
      ghist[tid] = cluster_bin_sum(ph, ncta, tid);  // every rank's count for this thread's bin
      bar_filter();
      if (w == 0) find_bucket_warp0(ghist, need, s.bc, lane);
      bar_filter();
      if (s.bc[0] == 0xFFFFFFFFu) {  // identical on every rank: the same sums
        if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
        exact = true;
        lo = hi;
        bar_filter();
        break;
      }
      const uint32_t b = s.bc[0], above_b = s.bc[1];
      need -= above_b;
      const uint32_t S = (m - need) + ghist[b];  // keys above the bucket + keys in it
      narrow(lo, hi, sh, b);
      bar_filter();
      hp ^= 1;
      if (S <= static_cast<uint32_t>(kHandCap)) break;
    }
  }
  if (tid == 0) s.final_bar = nbar + 2;  // phases 3 and 4 end with one cluster barrier each (counted from the first attempt)
  // ---- phase 3: publish this rank's survivor counts
  // exact: keep key > T plus a rank-ordered share of key == T; else keep key >= lo
  const uint32_t T = exact ? lo : lo - 1u;
  uint32_t g_r, q_r;
  count_gt_eq(s, static_cast<int>(n_r), T, g_r, q_r, tid);
  if (tid == 0) {
    s.pub[4] = g_r;
    s.pub[5] = exact ? q_r : 0u;
    s.bc[5] = lo;  // every key copied to the leader is >= lo (bc[4] still holds the max)
  }
  cluster_barrier();
  ++nbar;
  if (w == 0) {
    uint32_t g = 0, q = 0;
    if (lane < static_cast<int>(ncta)) {
      const uint32_t a = dsmem_map(smem_addr(&s.pub[4]), lane);
      g = dsmem_ld(a);
      q = dsmem_ld(a + 4);
    }
    // ranks hold contiguous, increasing index ranges: rank order is index order
    uint32_t q_incl = q;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(kFull, q_incl, o);
      if (lane >= o) q_incl += v;
    }
    const uint32_t q_excl = q_incl - q;
    const uint32_t keep_q = exact ? (need > q_excl ? min(q, need - q_excl) : 0u) : 0u;
    const uint32_t cnt = g + keep_q;
    uint32_t c_incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(kFull, c_incl, o);
      if (lane >= o) c_incl += v;
    }
    if (lane == static_cast<int>(rank)) {
      s.bc[6] = c_incl - cnt;  // my offset at the leader
      s.bc[7] = keep_q;
    }
    const uint32_t total = __shfl_sync(kFull, c_incl, 31);
    if (lane == 0) s.bc[2] = total;
  }
  bar_filter();
  const uint32_t my_off = s.bc[6], my_keep = s.bc[7], total = s.bc[2];
  bar_filter();
  // ---- phase 4: copy survivors into the leader at rank-ordered offsets
  const uint32_t rkey = dsmem_map(smem_addr(&s.hkey[0]), 0);
  const uint32_t ridx = dsmem_map(smem_addr(&s.hidx[0]), 0);
  if (exact && my_keep > 0u) {
    // this rank's share of the tied key: its my_keep lowest indices
    const uint32_t I = my_keep < q_r ? tie_cut(s, static_cast<int>(n_r), T, my_keep, q_r, tid) : 0xFFFFFFFFu;
    keep_remote<true>(s, static_cast<int>(n_r), T, I, tid, rkey, ridx, my_off);
  } else {
    keep_remote<false>(s, static_cast<int>(n_r), T, 0u, tid, rkey, ridx, my_off);
  }
  cluster_barrier();
  ++nbar;
  return total;
}

// The row and chunk of this CTA in cluster mode (the same computation in every
// role of every rank).
struct ClusterItem {
  uint32_t rank, ncta;
  int64_t row, L, c0, c1;
  uint32_t m;
};

__device__ __forceinline__ ClusterItem cluster_item(const Params& p) {
  ClusterItem it;
  it.rank = cluster_rank();
  it.ncta = cluster_size();
  it.row = cluster_index();
  it.L = clamp_len(p.lengths, it.row, p.row_stride);
  it.m = static_cast<uint32_t>(min64(p.k, it.L));
  int64_t chunk = (it.L + it.ncta - 1) / it.ncta;
  chunk = (chunk + 7) & ~static_cast<int64_t>(7);
  it.c0 = min64(it.L, static_cast<int64_t>(it.rank) * chunk);
  it.c1 = min64(it.L, it.c0 + chunk);
  return it;
}

// Cluster mode, warps kClusterWarp.. (one warpgroup): lane 0 of the first
// streams the chunk into the ring. The ring's first fill waits for nothing,
// so it is issued before the filter warps' sample exchange, whose
// kSampleBars cluster barriers every warp of the group takes too; then the
// rest of the chunk. Then every warp of the group mirrors the merge's
// cluster barriers (s.final_bar tells how many), leaving after the last.
template <class T>
__device__ __noinline__ void cluster_mirror(const Params p, int tid) {
  Smem& s = cta_smem();
  const int w = tid >> 5, lane = tid & 31;
  const ClusterItem it = cluster_item(p);
  if (it.m == 0) return;  // the same for every CTA of the cluster: no merge, no barrier
  const bool producer = w == kClusterWarp && lane == 0;
  const T* rowp = static_cast<const T*>(p.logits) + it.row * p.row_stride;
  const RowSpan sp = row_span(rowp + it.c0, it.c1 - it.c0);
  const int first = min(sp.nst, stages_of<T>());
  int slot = 0;
  uint32_t phase = 0u, armed = 0u, arm_par = 0u;
  long long gi = 0;
  bool live = true;
  if (producer) live = produce_stages<T>(s, sp, 0, first, slot, phase, gi, g_skip_stage, armed, arm_par);
  __syncwarp();
#pragma unroll 1
  for (int i = 0; i < kSampleBars; ++i) cluster_barrier();
  if (producer) {
    if (live) produce_stages<T>(s, sp, first, sp.nst, slot, phase, gi, g_skip_stage, armed, arm_par);
    producer_drain(s, armed, arm_par);
  }
  __syncwarp();
  for (uint32_t i = 1;; ++i) {
    cluster_barrier();
    const volatile uint32_t* fb = &s.final_bar;
    if (*fb == i) break;
  }
}

// Cluster mode, filter warps: this rank's chunk, then the merge; the leader
// ranks and writes the row.
template <class T>
__device__ __forceinline__ void cluster_filter(Smem& s, const Params& p, int tid) {
  const ClusterItem it = cluster_item(p);
  const int k = p.k;
  if (it.m == 0) {  // the same for every CTA of the cluster: no merge, no barrier
    if (it.rank == 0)
      for (int q = tid; q < k; q += kFilterThreads) p.out[it.row * static_cast<int64_t>(k) + q] = -1;
    return;
  }
  const T* rowp = static_cast<const T*>(p.logits) + it.row * p.row_stride;
  const int32_t Lc = static_cast<int32_t>(it.c1 - it.c0);
  const RowSpan sp = row_span(rowp + it.c0, Lc);
  const uint32_t m_r = min(it.m, static_cast<uint32_t>(Lc));
  Filter f;
  f.par = 0;
  // the row's threshold, the same in every rank (every rank takes part, a
  // rank with a short chunk sampling nothing)
  f.t = cluster_threshold<T>(rowp + it.c0, Lc, it.L, it.m, it.ncta, tid);
  // With no threshold from the samples the rank keeps only values above -inf:
  // a chunk of -inf (a row's padded tail) would otherwise fill the buffer with
  // ties and cut them by index while the other ranks wait at the merge.
  if (!(f.t > __int_as_float(0xff800000))) f.t = __int_as_float(0xff7fffff);  // -FLT_MAX: keep x unless x = -inf
  f.cnt = 0;
  f.compacted = false;
  f.strict = false;
  f.bounded = false;
  RingPos rp{0, 0u, 0u};
  stream_item<T>(s, f, rp, sp, Lc, static_cast<uint32_t>(it.c0), static_cast<int>(m_r), tid);
  const bool ok = !s.abort_seen;
  if (!ok) {
    f.cnt = 0;  // no candidates from this rank; it still takes part in the merge
  } else if (f.cnt > static_cast<uint32_t>(kHandCap)) {
    compact_any(s, f, static_cast<int>(m_r), tid);
  }
  // Either threshold is a guess: the merge checks that the ranks together
  // hold at least m values, or has every rank take its chunk again with none.
  uint32_t total = cluster_merge(f.cnt, it.m, !ok, true, it.rank, it.ncta, tid);
  if (total == kMergeRetry) {  // the same on every rank of the cluster
    if (tid == 0) atomicOr(&g_status, kStatusReread);
    f = refilter_from_global<T>(s, f, sp, Lc, static_cast<uint32_t>(it.c0), static_cast<int>(m_r), tid);
    if (f.cnt > static_cast<uint32_t>(kHandCap)) compact_any(s, f, static_cast<int>(m_r), tid);
    total = cluster_merge(f.cnt, it.m, !ok, false, it.rank, it.ncta, tid);
  }
  if (it.rank != 0) return;
  if (s.abort_any) {  // some rank gave up: no valid result for this row
    for (int q = tid; q < k; q += kFilterThreads) p.out[it.row * static_cast<int64_t>(k) + q] = -1;
    return;
  }
  const KeyBounds kb{s.bc[5], s.bc[4], static_cast<uint32_t>(it.L - 1), s.spub[3]};
  LeaderFinisher::finish(s, static_cast<int>(total), static_cast<int>(it.m), k, it.row, p, tid, true, &kb);
}

// Shared state of a fresh CTA (thread 0; a barrier follows).
__device__ __forceinline__ void init_cta(Smem& s, int finish_warps) {
  for (int i = 0; i < kMaxStages; ++i) {
    mbar_init(&s.full[i], 1);
    mbar_init(&s.empty[i], kFilterWarps);
  }
  mbar_init(&s.hfull, kFilterWarps);
  mbar_init(&s.hempty, finish_warps);
  for (int i = 0; i < 2; ++i) {
    s.est_ok[i] = 0;
    s.est[i] = 0.f;
    s.est_len[i] = 0;
  }
  s.own_key = 0u;
  s.own_len = 0;
  s.wait.abort = 0u;
  s.abort_seen = 0u;
  s.wait.limit_ns = g_wait_limit_ns;
  s.abort_any = 0u;
  s.final_bar = 0u;
  s.joint = 0u;
  s.merge_bars = 0u;
  s.merge_retry = 0u;
  fence_mbar_init();
}

}  // namespace rows

// Many rows: grid = min(num_rows, SMs), one CTA per SM, rows strided by the
// grid, 512 threads. kShort: every row fits one stage (see filter_loop). (A kernel of its own, apart from the cluster mode, so
// that each gets its own register allocation.)
template <class T, bool kShort>
__global__ void __launch_bounds__(rows::kThreads) topk_rows_kernel(const rows::Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  rows::Smem& s = *reinterpret_cast<rows::Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) rows::init_cta(s, rows::finish_warps<T>());
  __syncthreads();
  pdl_enter();  // every thread: inputs and outputs are touched only after this
  if (warp < rows::kFilterWarps) {
    rows::filter_loop<T, kShort>(s, p, tid);
  } else if (warp < rows::producer_warp<T>()) {
    rows::finish_loop<T>(s, p, tid - rows::kFilterThreads);
  } else if (warp == rows::producer_warp<T>() && lane == 0) {
    rows::produce_loop<T>(s, p);
  }
}

// A cluster per row: grid = num_rows * cluster size, 384 threads.
template <class T>
__global__ void __launch_bounds__(rows::kThreads) topk_cluster_kernel(const rows::Params p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  rows::Smem& s = *reinterpret_cast<rows::Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) rows::init_cta(s, 1);  // no finisher warps: the handover barrier is unused
  __syncthreads();
  pdl_enter();  // every thread: inputs and outputs are touched only after this
  if (warp < rows::kFilterWarps)
    rows::cluster_filter<T>(s, p, tid);
  else
    rows::cluster_mirror<T>(p, tid);
}

}  // namespace dsa
