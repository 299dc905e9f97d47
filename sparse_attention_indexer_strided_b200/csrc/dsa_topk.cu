// Strided indexer top-k for B200 (sm_100a).
//
// Operation (vLLM PR #42169 report, "实现拆解"; SGLang PR #34167 code
// excerpt): for each row r of fp32 logits at logits + r*row_stride, the k
// largest of the first L_r values, as row-local indices ordered by value
// descending and index ascending, padded with -1 past min(k, L_r).
//
// Design (one HBM pass, no global scratch), two kernels:
//   * Many rows (rows_path.cuh, topk_rows_kernel): one persistent CTA per SM
//     with a TMA producer warp, filter warps that stream each row against a
//     running threshold into a shared candidate buffer, and finisher warps
//     that rank the previous row's candidates while the next row streams.
//   * Few long rows (this file, topk_cluster_kernel): a thread-block cluster
//     splits a row into contiguous chunks. Each rank streams its chunk
//     through a TMA ring (one producer thread issues cp.async.bulk copies, no
//     multicast), keeps candidates above a running threshold in index order,
//     and compacts with a radix select (adaptive 8-bit windows over the key
//     range present) plus a stable keep that gives ties to the lowest index:
//     the pages' histogram / run_cumsum / threshold / gt-eq split, made exact
//     and deterministic. Long chunks start from a sampled threshold. Ranks
//     then merge through distributed shared memory: a cluster-wide histogram
//     over the candidates narrows the threshold, ranks publish counts, and
//     each rank writes its survivors into the leader's shared memory at
//     rank-ordered offsets (so index order, hence the tie rule, is kept). The
//     leader sorts the winners (stable LSD radix) and writes the row with -1
//     padding. Cluster barriers separate the phases; every CTA reaches every
//     barrier.
//
// Coding rules taken from the SGLang PR #34167 discussion: a distributed
// shared-memory address is only ever a 32-bit shared::cluster address used
// with ld/st.shared::cluster, never merged with a CTA-local pointer; k is a
// runtime value; kernel attributes are set per kernel per device.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "dsa_topk.h"

#define DSA_EXPORT extern "C" __attribute__((visibility("default")))

namespace dsa {

constexpr int kNumConsumerWarps = 8;                           // every warp consumes
constexpr int kConsumerThreads = kNumConsumerWarps * 32;       // 256
constexpr int kThreads = kConsumerThreads;
constexpr int kBlocksPerSM = 2;                                // one CTA selects/sorts while the other streams
constexpr int kStageElems = kNumConsumerWarps * 512;           // 16 KB per stage
constexpr uint32_t kStageBytes = kStageElems * 4;
constexpr int kStages = 3;                                     // 48 KB ring
constexpr int kWarpStageElems = kStageElems / kNumConsumerWarps;  // 512 = 4 groups x 32 lanes x float4
constexpr int kMaxK = DSA_TOPK_MAX_K;
constexpr int kCap = kMaxK + kStageElems;                      // candidate buffer entries
constexpr int kGatherOff = kMaxK;                              // cluster gather region
constexpr int kGatherCap = kCap - kGatherOff;
constexpr int kSortCountOff = 2 * kMaxK;                       // sort counters alias free space
constexpr int kMaxEntriesPerThread = (kCap + kConsumerThreads - 1) / kConsumerThreads;
constexpr int kStage2 = 192;  // per-warp staging entries for one stage's survivors
constexpr int kSortItemsPerWarp = kMaxK / kNumConsumerWarps;   // 256
constexpr int kSortSlots = kSortItemsPerWarp / 32;              // 8 per lane
constexpr uint32_t kNanKey = 0xFFC00000u;  // key of the canonical quiet NaN
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr unsigned long long kWaitLimitNs = 500000000ull;     // 0.5 s per pipeline wait
constexpr int kMaxRadixRounds = 4;  // 32-bit keys, >= 8 bits resolved per round

// Sticky status bits (g_status).
constexpr unsigned kStatusWaitTimeout = 1u;   // a pipeline wait gave up
constexpr unsigned kStatusSelectBroken = 2u;  // a radix round lost its invariant

static_assert(kSortCountOff + kNumConsumerWarps * 256 <= kCap, "sort counters must fit");
static_assert(kGatherCap >= kMaxK, "gather region must hold k entries");
static_assert(kCap - kMaxK >= kStageElems, "a stage must fit after a compaction");
static_assert(kWarpStageElems == 4 * 32 * 4, "a warp covers 4 float4 groups per stage");
static_assert(kConsumerThreads >= 256, "digit-parallel steps use one thread per 8-bit digit");

// Stream filter: kAcceptAll keeps every valid entry; kAbove keeps key > T (T is
// the exact k-th key of what was seen); kAtLeast keeps key >= T (T is a lower
// estimate taken from the previous row); kRejectAll keeps nothing (T is NaN).
enum Mode : int { kAcceptAll = 0, kAbove = 1, kAtLeast = 2, kRejectAll = 3 };

// A work item is the slice [c0, c1) of one row. Its bytes are fetched as the
// 16-byte aligned span that covers them; entries outside [c0, c1) are masked.
struct Span {
  const char* src;   // 16-byte aligned start
  int64_t j0;        // row-local index of the first float of the span
  uint64_t bytes;    // span length, multiple of 16
  int nst;           // stages
};

struct __align__(128) Smem {
  float ring[kStages][kStageElems];
  uint32_t ckey[kCap];
  uint32_t cidx[kCap];
  uint32_t hist[256];
  uint32_t phist[2][256];  // published to the cluster
  uint32_t ghist[256];
  uint32_t wtot[2][kNumConsumerWarps];
  uint32_t red[6][kNumConsumerWarps];
  uint32_t pub[8];  // published to the cluster
  uint32_t bc[8];
  uint32_t skip[4];
  uint32_t small[32];
  uint32_t stg_key[kNumConsumerWarps][kStage2];
  uint32_t stg_idx[kNumConsumerWarps][kStage2];
  unsigned long long full[kStages];
};
static_assert(sizeof(Smem) <= 232448 / kBlocksPerSM - 1024, "shared memory budget per CTA");

__device__ unsigned int g_status;  // sticky status bits, see kStatus*

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Orders this thread's earlier generic-proxy shared-memory accesses (made
// visible by a preceding barrier) before a following TMA write.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait: returns false (and records the status bit) after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_status, kStatusWaitTimeout);
      return false;
    }
  }
}
// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about hint_ns pass, instead of spinning on the barrier.
__device__ __forceinline__ bool mbar_try_wait_hint(unsigned long long* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Bounded wait for waits that are often long (a role idling until another
// catches up): sleeps in the barrier instead of spinning.
__device__ __forceinline__ bool mbar_wait_sleep(unsigned long long* bar, uint32_t parity) {
  if (mbar_try_wait_hint(bar, parity, 2000u)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_status, kStatusWaitTimeout);
      return false;
    }
  }
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void bar_consumers() { __syncthreads(); }
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}
// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t dsmem_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void dsmem_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// ------------------------------------------------------------- key mapping
// Order-preserving map fp32 -> uint32: larger key = larger value; every NaN
// maps to the key of +qNaN (above +inf); -0.0 maps to +0.0's key.
__device__ __forceinline__ uint32_t to_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (x != x) u = 0x7fc00000u;
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Inverse of to_key for non-NaN keys.
__device__ __forceinline__ float from_key(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// ------------------------------------------------------------ row geometry
__device__ __forceinline__ Span make_span(const float* row, int64_t c0, int64_t c1) {
  Span sp;
  if (c1 <= c0) {
    sp.src = reinterpret_cast<const char*>(row);
    sp.j0 = c0;
    sp.bytes = 0;
    sp.nst = 0;
    return sp;
  }
  const uintptr_t a = reinterpret_cast<uintptr_t>(row + c0);
  const uintptr_t e = reinterpret_cast<uintptr_t>(row + c1);
  const uintptr_t as = a & ~static_cast<uintptr_t>(15);
  const uintptr_t ee = (e + 15) & ~static_cast<uintptr_t>(15);
  sp.src = reinterpret_cast<const char*>(as);
  sp.j0 = c0 - static_cast<int64_t>((a - as) >> 2);
  sp.bytes = ee - as;
  sp.nst = static_cast<int>((sp.bytes + kStageBytes - 1) / kStageBytes);
  return sp;
}

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ int64_t clamp_len(const int32_t* lengths, int64_t row, int64_t row_stride) {
  int64_t L = lengths[row];
  if (L < 0) L = 0;
  if (L > row_stride) L = row_stride;
  return L;
}

// Producer cursor, advanced by thread 0 only. It walks the same sequence of
// (work item, stage) pairs as the consumers, kStages stages ahead of them: a
// stage is issued into the ring slot that the consumers released at the
// barrier that ended the stage kStages before it.

struct Producer {
  int64_t row;          // current work item
  const char* src;      // its 16-byte aligned span start
  uint32_t nst, t;      // its stage count, next stage to issue
  uint32_t last_bytes;  // bytes of its last stage
  uint32_t g;           // stages issued so far (slot = g % kStages)
};

struct ItemSource {
  const float* logits;
  const int32_t* lengths;
  int64_t row_stride, row_end, row_step;
  int64_t c0, c1;  // slice of the row; c1 < 0: the whole valid row
};

__device__ __forceinline__ void producer_set_item(Producer& p, const ItemSource& is) {
  p.t = 0;
  p.nst = 0;
  if (p.row >= is.row_end) return;
  const int64_t L = clamp_len(is.lengths, p.row, is.row_stride);
  const int64_t c1 = is.c1 < 0 ? L : min64(is.c1, L);
  const Span sp = make_span(is.logits + p.row * is.row_stride, min64(is.c0, c1), c1);
  p.src = sp.src;
  p.nst = static_cast<uint32_t>(sp.nst);
  p.last_bytes = sp.nst ? static_cast<uint32_t>(sp.bytes - static_cast<uint64_t>(sp.nst - 1) * kStageBytes) : 0u;
}

__device__ __forceinline__ uint32_t stage_bytes(const Producer& p, uint32_t t) {
  return t + 1 == p.nst ? p.last_bytes : kStageBytes;
}

// Issue the next stage, if any remains.
__device__ __forceinline__ void producer_issue(Smem& s, Producer& p, const ItemSource& is) {
  while (p.t >= p.nst) {
    if (p.row >= is.row_end) return;
    p.row += is.row_step;
    producer_set_item(p, is);
  }
  const int slot = static_cast<int>(p.g % kStages);
  const uint32_t bytes = stage_bytes(p, p.t);
  const char* src = p.src + static_cast<uint64_t>(p.t) * kStageBytes;
  fence_proxy_async();
  mbar_arrive_expect_tx(&s.full[slot], bytes);
  bulk_g2s(&s.ring[slot][0], src, bytes, &s.full[slot]);
  ++p.t;
  ++p.g;
}

// ------------------------------------------------------ block-level helpers
struct MinMax {
  uint32_t mn, mx;
};

// min / max key over entries [base, base+n) (all consumer threads).
__device__ MinMax block_minmax(Smem& s, int base, int n, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int e = tid; e < n; e += kConsumerThreads) {
    const uint32_t key = s.ckey[base + e];
    mn = min(mn, key);
    mx = max(mx, key);
  }
  mn = __reduce_min_sync(kFull, mn);
  mx = __reduce_max_sync(kFull, mx);
  if (lane == 0) {
    s.red[0][w] = mn;
    s.red[1][w] = mx;
  }
  bar_consumers();
  const uint32_t a = lane < kNumConsumerWarps ? s.red[0][lane] : 0xFFFFFFFFu;
  const uint32_t b = lane < kNumConsumerWarps ? s.red[1][lane] : 0u;
  MinMax r;
  r.mn = __reduce_min_sync(kFull, a);
  r.mx = __reduce_max_sync(kFull, b);
  bar_consumers();  // red[0..1] may be rewritten by the next call
  return r;
}

// Bucket search over a 256-bin histogram in descending digit order: finds b
// with (#keys in bins > b) < need <= (#keys in bins >= b). Warp 0 writes
// bc[0] = b, bc[1] = #keys in bins > b. Caller synchronises.
__device__ __forceinline__ void find_bucket_warp0(const uint32_t* hist, uint32_t need, uint32_t* bc, int lane) {
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    c[t] = hist[255 - 8 * lane - t];
    sum += c[t];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t excl = incl - sum;
  if (excl < need && need <= incl) {
    uint32_t acc = excl;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (acc + c[t] >= need) {
        bc[0] = 255u - 8u * lane - t;
        bc[1] = acc;
        break;
      }
      acc += c[t];
    }
  }
}

// Narrow [lo, hi] to bucket b of the window starting at bit sh.
__device__ __forceinline__ void narrow(uint32_t& lo, uint32_t& hi, int sh, uint32_t b) {
  const uint32_t keep_hi = (sh + 8 >= 32) ? 0u : ~((1u << (sh + 8)) - 1u);
  const uint32_t blo = (lo & keep_hi) | (b << sh);
  const uint32_t bhi = blo | ((1u << sh) - 1u);
  lo = max(lo, blo);
  hi = min(hi, bhi);
}

// Window for the next radix step: 8 bits ending at the highest differing bit.
__device__ __forceinline__ int window_shift(uint32_t lo, uint32_t hi) {
  const int h = 31 - __clz(lo ^ hi);
  return h >= 7 ? h - 7 : 0;
}

// Histogram of keys in [lo, hi] over entries [base, base+n) into hist[256]
// (already zeroed). Each thread walks its strided entries and adds a run of
// equal digits with one atomic, so heavily tied keys cost few atomics.
__device__ __forceinline__ void histogram(const Smem& s, uint32_t* hist, int base, int n, uint32_t lo, uint32_t hi,
                                          int sh, int tid) {
  uint32_t cur = 0xFFFFFFFFu, run = 0;
  for (int e = tid; e < n; e += kConsumerThreads) {
    const uint32_t key = s.ckey[base + e];
    if (key < lo || key > hi) continue;
    const uint32_t d = (key >> sh) & 255u;
    if (d != cur) {
      if (run) atomicAdd(&hist[cur], run);
      cur = d;
      run = 0;
    }
    ++run;
  }
  if (run) atomicAdd(&hist[cur], run);
}

// Exact need-th largest key among the <= 32 keys in [lo, hi] (warp 0). Every
// lane holds one key (or 0, below any real key); returns the largest key x with
// #{keys >= x} >= need.
__device__ __forceinline__ uint32_t small_kth(uint32_t mine, uint32_t need) {
  uint32_t ge = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) ge += __shfl_sync(kFull, mine, j) >= mine;
  return __reduce_max_sync(kFull, (mine != 0u && ge >= need) ? mine : 0u);
}

// Stable selection of entries [base, base+n): keep key > T, plus the first
// need_eq entries with key == T (buffer order = index order). Kept entries go,
// in order, to dst positions 0.. . Local mode compacts in place at `base`;
// remote mode stores to the shared::cluster addresses rkey/ridx (+4*(off+pos)).
template <bool kRemote>
__device__ void stable_keep(Smem& s, int base, int n, uint32_t T, uint32_t need_eq, uint32_t rkey, uint32_t ridx,
                            uint32_t off, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  const int per_warp = ((n + kConsumerThreads - 1) / kConsumerThreads) * 32;
  const int E = per_warp >> 5;
  const int wbeg = w * per_warp;
  uint32_t kk[kMaxEntriesPerThread], ii[kMaxEntriesPerThread];
  uint32_t ngt = 0, neq = 0;
#pragma unroll
  for (int it = 0; it < kMaxEntriesPerThread; ++it) {
    if (it < E) {
      const int e = wbeg + it * 32 + lane;
      const bool v = e < n;
      kk[it] = v ? s.ckey[base + e] : 0u;  // key 0 never occurs: below any T
      ii[it] = v ? s.cidx[base + e] : 0u;
      ngt += __popc(__ballot_sync(kFull, kk[it] > T));
      neq += __popc(__ballot_sync(kFull, kk[it] == T));
    }
  }
  if (lane == 0) {
    s.red[2][w] = ngt;
    s.red[3][w] = neq;
  }
  bar_consumers();
  const uint32_t a = lane < kNumConsumerWarps ? s.red[2][lane] : 0u;
  const uint32_t b = lane < kNumConsumerWarps ? s.red[3][lane] : 0u;
  uint32_t gt_before = __reduce_add_sync(kFull, lane < w ? a : 0u);
  uint32_t eq_before = __reduce_add_sync(kFull, lane < w ? b : 0u);
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int it = 0; it < kMaxEntriesPerThread; ++it) {
    if (it < E) {
      const bool g = kk[it] > T, q = kk[it] == T;
      const uint32_t gb = __ballot_sync(kFull, g), eb = __ballot_sync(kFull, q);
      const uint32_t my_gt = gt_before + __popc(gb & lt);
      const uint32_t my_eq = eq_before + __popc(eb & lt);
      if (g || (q && my_eq < need_eq)) {
        const uint32_t pos = my_gt + min(my_eq, need_eq);
        if (kRemote) {
          dsmem_st(rkey + 4u * (off + pos), kk[it]);
          dsmem_st(ridx + 4u * (off + pos), ii[it]);
        } else {
          s.ckey[base + pos] = kk[it];
          s.cidx[base + pos] = ii[it];
        }
      }
      gt_before += __popc(gb);
      eq_before += __popc(eb);
    }
  }
  bar_consumers();
}

// Counts of keys > T and == T over entries [0, n) (block-wide, consumers).
__device__ void count_gt_eq(Smem& s, int base, int n, uint32_t T, uint32_t& ngt, uint32_t& neq, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  uint32_t g = 0, q = 0;
  for (int e = tid; e < n; e += kConsumerThreads) {
    const uint32_t key = s.ckey[base + e];
    g += key > T;
    q += key == T;
  }
  g = __reduce_add_sync(kFull, g);
  q = __reduce_add_sync(kFull, q);
  if (lane == 0) {
    s.red[4][w] = g;
    s.red[5][w] = q;
  }
  bar_consumers();
  ngt = __reduce_add_sync(kFull, lane < kNumConsumerWarps ? s.red[4][lane] : 0u);
  neq = __reduce_add_sync(kFull, lane < kNumConsumerWarps ? s.red[5][lane] : 0u);
  bar_consumers();
}

// Exact selection: entries [base, base+n), n > k. Keeps the k largest keys in
// place, in index order, ties to the lowest index. Returns the k-th largest key.
// Radix rounds narrow [lo, hi] (8-bit windows below the highest bit where lo
// and hi differ); once the bucket holding the k-th key has <= 32 entries, warp 0
// finishes it directly.
__device__ __noinline__ uint32_t select_topk(Smem& s, int base, int n, int k, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  const MinMax r = block_minmax(s, base, n, tid);
  uint32_t lo = r.mn, hi = r.mx, need = static_cast<uint32_t>(k);
  for (int round = 0; lo != hi; ++round) {
    if (round == kMaxRadixRounds) {  // unreachable for a consistent histogram
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    const int sh = window_shift(lo, hi);
    if (tid < 256) s.hist[tid] = 0u;
    if (tid == 0) {
      s.bc[0] = 0xFFFFFFFFu;
      s.bc[2] = 0u;
    }
    __syncthreads();
    histogram(s, s.hist, base, n, lo, hi, sh, tid);
    __syncthreads();
    if (w == 0) find_bucket_warp0(s.hist, need, s.bc, lane);
    __syncthreads();
    const uint32_t b = s.bc[0], above_b = s.bc[1];
    if (b == 0xFFFFFFFFu) {  // no bucket holds the need-th key
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    const uint32_t in_bucket = s.hist[b];
    need -= above_b;
    narrow(lo, hi, sh, b);
    if (in_bucket <= 32u && lo != hi) {
      // gather the bucket's keys (order irrelevant) and finish in one warp
      for (int e = tid; e < n; e += kConsumerThreads) {
        const uint32_t key = s.ckey[base + e];
        if (key >= lo && key <= hi) s.small[atomicAdd(&s.bc[2], 1u)] = key;
      }
      __syncthreads();
      if (w == 0) {
        const uint32_t mine = lane < static_cast<int>(in_bucket) ? s.small[lane] : 0u;
        const uint32_t t = small_kth(mine, need);
        const uint32_t above = __popc(__ballot_sync(kFull, mine > t));
        if (lane == 0) {
          s.bc[3] = t;
          s.bc[4] = need - above;
        }
      }
      __syncthreads();
      lo = hi = s.bc[3];
      need = s.bc[4];
    }
    __syncthreads();  // bc / hist / small reused by the next round
  }
  stable_keep<false>(s, base, n, lo, need, 0u, 0u, 0u, tid);
  return lo;
}

// Stable LSD radix sort of entries [src, src+m) (m <= kMaxK) by key
// descending, using [alt, alt+m) as the other buffer. Ties keep buffer order.
// Returns the base that holds the sorted entries. Bytes of the key above the
// highest bit where the smallest and largest keys differ are equal for every
// entry, so only the passes below it run. Within a warp, lanes holding the
// same digit are found with eight ballots (one per digit bit).
__device__ __noinline__ int sort_desc(Smem& s, int src, int alt, int m, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  if (m <= 1) return src;
  // bits that differ between some two keys: a byte with none is equal in every
  // key, and its stable pass would be the identity (the low bytes of values on
  // a coarse grid, such as fp8, are)
  uint32_t any1 = 0u, all1 = 0xFFFFFFFFu;
  for (int e = tid; e < m; e += kConsumerThreads) {
    const uint32_t key = s.ckey[src + e];
    any1 |= key;
    all1 &= key;
  }
  any1 = __reduce_or_sync(kFull, any1);
  all1 = __reduce_and_sync(kFull, all1);
  if (lane == 0) {
    s.red[2][w] = any1;
    s.red[3][w] = all1;
  }
  __syncthreads();
  any1 = 0u;
  all1 = 0xFFFFFFFFu;
#pragma unroll
  for (int ww = 0; ww < kNumConsumerWarps; ++ww) {
    any1 |= s.red[2][ww];
    all1 &= s.red[3][ww];
  }
  const uint32_t varying = any1 & ~all1;
  __syncthreads();  // red[2..3] may be rewritten by a later call
  if (varying == 0u) return src;
  uint32_t* wcnt = s.ckey + kSortCountOff;  // [warp][256]
  const uint32_t lt = lanemask_lt();
  for (int pass = 0; pass < 4; ++pass) {
    const int sh = pass * 8;
    if (((varying >> sh) & 255u) == 0u) continue;  // the same byte in every key
#pragma unroll
    for (int i = 0; i < 8; ++i) wcnt[w * 256 + i * 32 + lane] = 0u;
    __syncwarp();
    uint32_t dig[kSortSlots], lp[kSortSlots];
#pragma unroll
    for (int it = 0; it < kSortSlots; ++it) {
      const int item = w * kSortItemsPerWarp + it * 32 + lane;
      const bool v = item < m;
      const uint32_t d = v ? ((~s.ckey[src + item]) >> sh) & 255u : 0u;
      uint32_t peers = __ballot_sync(kFull, v);
#pragma unroll
      for (int bit = 0; bit < 8; ++bit) {
        const uint32_t bb = __ballot_sync(kFull, (d >> bit) & 1u);
        peers &= ((d >> bit) & 1u) ? bb : ~bb;
      }
      const uint32_t c = v ? wcnt[w * 256 + d] : 0u;
      __syncwarp();
      if (v && (peers & lt) == 0u) wcnt[w * 256 + d] = c + __popc(peers);
      __syncwarp();
      dig[it] = d;
      lp[it] = c + __popc(peers & lt);
    }
    __syncthreads();
    // digit-major, warp-minor exclusive prefix: thread t < 256 owns digit t
    uint32_t tot = 0, incl = 0, c[kNumConsumerWarps];
    if (tid < 256) {
#pragma unroll
      for (int ww = 0; ww < kNumConsumerWarps; ++ww) c[ww] = wcnt[ww * 256 + tid];
#pragma unroll
      for (int ww = 0; ww < kNumConsumerWarps; ++ww) {
        const uint32_t x = c[ww];
        c[ww] = tot;
        tot += x;
      }
      incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) s.red[4][w] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t dbase = incl - tot;
      for (int ww = 0; ww < w; ++ww) dbase += s.red[4][ww];
#pragma unroll
      for (int ww = 0; ww < kNumConsumerWarps; ++ww) wcnt[ww * 256 + tid] = c[ww] + dbase;
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < kSortSlots; ++it) {
      const int item = w * kSortItemsPerWarp + it * 32 + lane;
      if (item < m) {
        const uint32_t dst = wcnt[w * 256 + dig[it]] + lp[it];
        s.ckey[alt + dst] = s.ckey[src + item];
        s.cidx[alt + dst] = s.cidx[src + item];
      }
    }
    __syncthreads();
    const int t = src;
    src = alt;
    alt = t;
  }
  return src;
}

__device__ __forceinline__ void write_row(const Smem& s, int R, int m, int k, int32_t* out_row, int tid) {
  for (int j = tid; j < k; j += kConsumerThreads)
    out_row[j] = j < m ? static_cast<int32_t>(s.cidx[R + j]) : -1;
}

// ------------------------------------------------------------ stream phase
struct StreamState {
  uint32_t count;  // candidates held (uniform across threads)
  int mode;
  float thr;       // threshold value for kAbove / kAtLeast
  int par;         // wtot double-buffer parity
};

__device__ __forceinline__ void set_exact_threshold(StreamState& st, uint32_t T) {
  if (T == kNanKey) {
    st.mode = kRejectAll;
  } else {
    st.mode = kAbove;
    st.thr = from_key(T);
  }
}

// The 16 values a thread looks at in one stage: group j is the float4 at
// stage offset warp*512 + j*128 + lane*4 (coalesced, conflict-free reads).
struct Lane16 {
  float x[4][4];
};

__device__ __forceinline__ int lane_offset(int w, int lane, int j) { return w * kWarpStageElems + j * 128 + lane * 4; }

// v.x[b >> 2][b & 3] for a runtime b in [0, 16), as a select tree (keeps the
// values in registers).
__device__ __forceinline__ float pick16(const Lane16& v, int b) {
  float q[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = (b & 1) ? v.x[j][1] : v.x[j][0];
    const float hi = (b & 1) ? v.x[j][3] : v.x[j][2];
    q[j] = (b & 2) ? hi : lo;
  }
  const float lo = (b & 4) ? q[1] : q[0];
  const float hi = (b & 4) ? q[3] : q[2];
  return (b & 8) ? hi : lo;
}

// Filter one stage's values (in registers; `src` points at the same stage in
// shared or global memory), then append the survivors to the candidate buffer
// in index order. Index order inside a warp is (group, lane, component); one
// warp scan over byte-packed per-group counts gives every survivor its rank r
// in the warp. Before the stage barrier, lane r gathers the r-th survivor into
// the warp's staging area (so lanes work on one survivor each instead of
// looping over their own); after the barrier the staged entries are copied to
// the candidate buffer behind the warps before it. `prod` (thread 0 only, may
// be null) issues the next ring stage right after that barrier, which ends
// every read of this stage's slot.
__device__ __forceinline__ void consume_values(Smem& s, StreamState& st, const Lane16& v, const float* src,
                                               int64_t jbase, int64_t c0, int64_t c1, int k, int tid, Producer* prod,
                                               const ItemSource* is) {
  const int w = tid >> 5, lane = tid & 31;
  const int64_t lo64 = c0 - jbase, hi64 = c1 - jbase;
  const int lo = static_cast<int>(lo64 < 0 ? 0 : (lo64 > kStageElems ? kStageElems : lo64));
  const int hi = static_cast<int>(hi64 < 0 ? 0 : (hi64 > kStageElems ? kStageElems : hi64));
  const bool filtering = st.mode == kAbove || st.mode == kAtLeast;
  uint32_t F = 0;  // bit 4j+c: value x[j][c] survives
  if (st.mode == kAbove) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) F |= static_cast<uint32_t>(!(v.x[j][c] <= st.thr)) << (4 * j + c);
  } else if (st.mode == kAtLeast) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) F |= static_cast<uint32_t>(!(v.x[j][c] < st.thr)) << (4 * j + c);
  }
  if (filtering && (lo > 0 || hi < kStageElems)) {
    // entries outside [c0, c1) (span head/tail, short last stage) never survive
    uint32_t valid = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int o = lane_offset(w, lane, j) + c;
        valid |= static_cast<uint32_t>(o >= lo && o < hi) << (4 * j + c);
      }
    F &= valid;
  }
  uint32_t excl = 0, tj[4] = {0, 0, 0, 0}, wt = 0;
  if (filtering && __any_sync(kFull, F != 0u)) {
    // per-group popcounts, one byte each (SWAR, no XU-pipe popc)
    const uint32_t c2 = F - ((F >> 1) & 0x5555u);
    const uint32_t c4 = (c2 & 0x3333u) + ((c2 >> 2) & 0x3333u);
    const uint32_t packed = (c4 & 0xFu) | ((c4 & 0xF0u) << 4) | ((c4 & 0xF00u) << 8) | ((c4 & 0xF000u) << 12);
    uint32_t incl = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += t;  // each byte stays <= 128
    }
    excl = incl - packed;
    const uint32_t tot = __shfl_sync(kFull, incl, 31);
#pragma unroll
    for (int j = 0; j < 4; ++j) tj[j] = (tot >> (8 * j)) & 0xFFu;
    wt = tj[0] + tj[1] + tj[2] + tj[3];
    if (wt <= static_cast<uint32_t>(kStage2)) {
      // gather: lane r fetches the warp's r-th survivor (group-major order)
      const uint32_t t0 = tj[0], t1 = t0 + tj[1], t2 = t1 + tj[2];
      for (uint32_t r0 = 0; r0 < wt; r0 += 32) {
        const uint32_t r = r0 + lane;
        const int j = (r >= t0) + (r >= t1) + (r >= t2);
        const uint32_t rj = r - (j == 0 ? 0u : (j == 1 ? t0 : (j == 2 ? t1 : t2)));
        const int sj = 8 * j;
        int l = 0;  // largest lane whose group-j exclusive prefix is <= rj
#pragma unroll
        for (int step = 16; step; step >>= 1) {
          const uint32_t e = __shfl_sync(kFull, excl, l + step);
          if (((e >> sj) & 0xFFu) <= rj) l += step;
        }
        const uint32_t el = (__shfl_sync(kFull, excl, l) >> sj) & 0xFFu;
        uint32_t f = (__shfl_sync(kFull, F, l) >> (4 * j)) & 0xFu;
        const uint32_t q = rj - el;  // q-th set bit of lane l's group-j nibble
        if (q > 0) f &= f - 1u;
        if (q > 1) f &= f - 1u;
        if (q > 2) f &= f - 1u;
        const int off = lane_offset(w, l, j) + (__ffs(f) - 1);
        if (r < wt) {
          s.stg_key[w][r] = to_key(src[off]);
          s.stg_idx[w][r] = static_cast<uint32_t>(jbase + off);
        }
      }
    }
  }
  if (lane == 0) s.wtot[st.par][w] = wt;
  __syncthreads();
  if (prod) producer_issue(s, *prod, *is);
  uint32_t pre = 0, tot = 0;
  if (filtering) {
    const uint32_t wv = lane < kNumConsumerWarps ? s.wtot[st.par][lane] : 0u;
    pre = __reduce_add_sync(kFull, lane < w ? wv : 0u);
    tot = __reduce_add_sync(kFull, wv);
  } else if (st.mode == kAcceptAll) {
    tot = static_cast<uint32_t>(hi > lo ? hi - lo : 0);
  }
  st.par ^= 1;
  if (tot == 0) return;
  if (st.count + tot > static_cast<uint32_t>(kCap)) {
    // Make room. This stage's survivors passed the old threshold; appending
    // them after the compaction keeps the buffer a superset of the winners.
    const uint32_t T = select_topk(s, 0, static_cast<int>(st.count), k, tid);
    st.count = static_cast<uint32_t>(k);
    set_exact_threshold(st, T);
  }
  if (!filtering) {
    // every entry in [lo, hi) survives: its rank is its offset
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int o = lane_offset(w, lane, j) + c;
        if (o >= lo && o < hi) {
          const uint32_t p = st.count + static_cast<uint32_t>(o - lo);
          s.ckey[p] = to_key(v.x[j][c]);
          s.cidx[p] = static_cast<uint32_t>(jbase + o);
        }
      }
  } else if (wt <= static_cast<uint32_t>(kStage2)) {
    const uint32_t base = st.count + pre;
    for (uint32_t r = lane; r < wt; r += 32) {
      s.ckey[base + r] = s.stg_key[w][r];
      s.cidx[base + r] = s.stg_idx[w][r];
    }
  } else if (F) {
    // more survivors than the staging area holds: each lane writes its own
    const uint32_t base = st.count + pre;
    const uint32_t g0 = base + (excl & 0xFFu);
    const uint32_t g1 = base + tj[0] + ((excl >> 8) & 0xFFu);
    const uint32_t g2 = base + tj[0] + tj[1] + ((excl >> 16) & 0xFFu);
    const uint32_t g3 = base + tj[0] + tj[1] + tj[2] + (excl >> 24);
    const int64_t jl = jbase + w * kWarpStageElems + lane * 4;
    uint32_t rest = F, run = 0, gcur = 0;
    int jcur = -1;
    while (rest) {
      const int b = __ffs(rest) - 1;
      rest &= rest - 1u;
      const int j = b >> 2;
      if (j != jcur) {
        jcur = j;
        run = 0;
        gcur = j == 0 ? g0 : (j == 1 ? g1 : (j == 2 ? g2 : g3));
      }
      const uint32_t p = gcur + run++;
      s.ckey[p] = to_key(pick16(v, b));
      s.cidx[p] = static_cast<uint32_t>(jl + j * 128 + (b & 3));
    }
  }
  st.count += tot;
  if (st.mode == kAcceptAll && st.count >= 2u * static_cast<uint32_t>(k)) {
    // Seen at least 2k entries: fix an exact threshold early; fewer entries
    // survive the filter afterwards than if the buffer were left to fill.
    __syncthreads();
    const uint32_t T = select_topk(s, 0, static_cast<int>(st.count), k, tid);
    st.count = static_cast<uint32_t>(k);
    set_exact_threshold(st, T);
  }
}

// Consumer side of the ring: g = stages consumed so far.
__device__ __forceinline__ void load_stage(const Smem& s, uint32_t g, Lane16& v, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  const float* src = &s.ring[g % kStages][0];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 q = *reinterpret_cast<const float4*>(src + lane_offset(w, lane, j));
    v.x[j][0] = q.x;
    v.x[j][1] = q.y;
    v.x[j][2] = q.z;
    v.x[j][3] = q.w;
  }
}

// Stream one work item through the ring. On return the buffer holds the
// item's top min(k, #valid) entries in index order when the filter never
// dropped a winner, which is always the case unless the starting mode was
// kAtLeast; then the caller checks `count >= k` (see stream_row).
__device__ __forceinline__ uint32_t stream_ring(Smem& s, const Span& sp, int64_t c0, int64_t c1, int k, uint32_t& g,
                                                int& par, int mode0, float thr0, bool& compacted, int tid,
                                                Producer* prod, const ItemSource* is) {
  StreamState st;
  st.count = 0;
  st.mode = mode0;
  st.thr = thr0;
  st.par = par;
  for (int t = 0; t < sp.nst; ++t) {
    mbar_wait(&s.full[g % kStages], (g / kStages) & 1u);
    Lane16 v;
    load_stage(s, g, v, tid);
    consume_values(s, st, v, &s.ring[g % kStages][0], sp.j0 + static_cast<int64_t>(t) * kStageElems, c0, c1, k, tid,
                   prod, is);
    ++g;
  }
  __syncthreads();  // the last stage's appends land before anyone reads the buffer
  compacted = st.mode != mode0;
  par = st.par;
  return st.count;
}

// Same as stream_ring, reading the span straight from global memory (used to
// redo a row whose speculative threshold turned out too high).
__device__ __noinline__ uint32_t stream_global(Smem& s, const Span& sp, int64_t c0, int64_t c1, int k, int& par, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  StreamState st;
  st.count = 0;
  st.mode = kAcceptAll;
  st.thr = 0.f;
  st.par = par;
  for (int t = 0; t < sp.nst; ++t) {
    Lane16 v;
    const uint64_t sbase = static_cast<uint64_t>(t) * kStageBytes;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint64_t off = sbase + 4u * static_cast<uint64_t>(lane_offset(w, lane, j));
      float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
      if (off + 16 <= sp.bytes) q = __ldg(reinterpret_cast<const float4*>(sp.src + off));
      v.x[j][0] = q.x;
      v.x[j][1] = q.y;
      v.x[j][2] = q.z;
      v.x[j][3] = q.w;
    }
    consume_values(s, st, v, reinterpret_cast<const float*>(sp.src + sbase),
                   sp.j0 + static_cast<int64_t>(t) * kStageElems, c0, c1, k, tid, nullptr, nullptr);
  }
  __syncthreads();
  par = st.par;
  return st.count;
}

// need-th largest key among candidates [0, n) (consumer threads; 1 <= need
// <= n): the radix rounds of select_topk without the compaction.
__device__ __noinline__ uint32_t kth_key(Smem& s, int n, uint32_t need, int tid) {
  const int w = tid >> 5, lane = tid & 31;
  const MinMax r = block_minmax(s, 0, n, tid);
  uint32_t lo = r.mn, hi = r.mx;
  for (int round = 0; lo != hi; ++round) {
    if (round == kMaxRadixRounds) {
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    const int sh = window_shift(lo, hi);
    if (tid < 256) s.hist[tid] = 0u;
    if (tid == 0) {
      s.bc[0] = 0xFFFFFFFFu;
      s.bc[2] = 0u;
    }
    __syncthreads();
    histogram(s, s.hist, 0, n, lo, hi, sh, tid);
    __syncthreads();
    if (w == 0) find_bucket_warp0(s.hist, need, s.bc, lane);
    __syncthreads();
    const uint32_t b = s.bc[0], above_b = s.bc[1];
    if (b == 0xFFFFFFFFu) {
      if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
      break;
    }
    const uint32_t in_bucket = s.hist[b];
    need -= above_b;
    narrow(lo, hi, sh, b);
    if (in_bucket <= 32u && lo != hi) {
      for (int e = tid; e < n; e += kConsumerThreads) {
        const uint32_t key = s.ckey[e];
        if (key >= lo && key <= hi) {
          const uint32_t slot = atomicAdd(&s.bc[2], 1u);
          if (slot < 32u) s.small[slot] = key;
        }
      }
      __syncthreads();
      if (w == 0) {
        const uint32_t t = small_kth(lane < static_cast<int>(in_bucket) ? s.small[lane] : 0u, need);
        if (lane == 0) s.bc[3] = t;
      }
      __syncthreads();
      lo = hi = s.bc[3];
    }
    __syncthreads();
  }
  return lo;
}

// A starting threshold for a cluster rank's chunk [c0, c1) of a row: the
// chunk is sampled as kStageElems values in 32 evenly spaced runs of 128
// (aligned 16-byte blocks inside the chunk), and the threshold is the value
// with 1.5 times the chunk's share of m_r sampled values above it, plus 16.
// Returns -inf when the sample gives none.
__device__ __noinline__ float chunk_threshold(Smem& s, const float* row, int64_t c0, int64_t c1, uint32_t m_r,
                                              int tid) {
  const int w = tid >> 5, lane = tid & 31;
  const uintptr_t a = reinterpret_cast<uintptr_t>(row + c0);
  const uintptr_t as = a & ~static_cast<uintptr_t>(15);
  const int64_t j0 = c0 - static_cast<int64_t>((a - as) >> 2);  // row index of the aligned base
  const int64_t span = c1 - j0;                                   // floats from there to the chunk end
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t run = w * 4 + q;  // 0..31
    const int64_t b = ((span - 128) * run / 31) & ~static_cast<int64_t>(3);
    const float4 x = __ldg(reinterpret_cast<const float4*>(as) + (b >> 2) + lane);
    const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t j = j0 + b + 4 * lane + i;
      s.ckey[w * 512 + q * 128 + lane * 4 + i] = (j >= c0 && j < c1) ? to_key(xv[i]) : 0u;  // 0: below every key
    }
  }
  __syncthreads();
  const double share = static_cast<double>(kStageElems) * m_r / static_cast<double>(c1 - c0);
  const uint32_t need = min(static_cast<uint32_t>(kStageElems - 8), static_cast<uint32_t>(1.5 * share) + 16u);
  const uint32_t T = kth_key(s, kStageElems, need, tid);
  return (T == 0u || T >= 0xFF800000u) ? __int_as_float(0xff800000) : from_key(T);
}

__device__ __forceinline__ void init_pipeline(Smem& s) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&s.full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
}

// --------------------------------------------------------------- kernels
// Few long rows: a cluster of CTAs per row (grid = num_rows * cluster size).
// kSample: ranks whose chunk holds at least kSampleChunk values start from a
// sampled threshold; the host picks the instantiation from row_stride and the
// cluster size (which bound every chunk), so short chunks run the plain one.
constexpr int64_t kSampleChunk = 8 * kStageElems;

template <bool kSample>
__global__ void __launch_bounds__(kThreads, kBlocksPerSM)
    topk_cluster_kernel(const float* __restrict__ logits, int64_t row_stride, const int32_t* __restrict__ lengths,
                        int64_t num_rows, int k, int32_t* __restrict__ out) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  init_pipeline(s);
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank();
  const uint32_t ncta = cluster_size();
  const int64_t row = cluster_index();
  // every CTA of the cluster takes the same branch (row is per cluster)
  if (row >= num_rows) return;
  const int64_t L = clamp_len(lengths, row, row_stride);
  int64_t chunk = (L + ncta - 1) / ncta;
  chunk = (chunk + 3) & ~static_cast<int64_t>(3);
  const int64_t c0 = min64(L, static_cast<int64_t>(rank) * chunk);
  const int64_t c1 = min64(L, c0 + chunk);
  const float* row_ptr = logits + row * row_stride;
  const Span sp = make_span(row_ptr, c0, c1);
  const int w = tid >> 5, lane = tid & 31;
  const uint32_t m = static_cast<uint32_t>(min64(k, L));
  if (m == 0) {  // L == 0 for every rank alike: nothing streamed, no merge
    if (rank == 0) write_row(s, 0, 0, k, out + row * static_cast<int64_t>(k), tid);
    return;
  }
  const ItemSource is{logits, lengths, row_stride, row + 1, 1, c0, c1};  // this one row only
  Producer prod;
  if (tid == 0) {
    prod.row = row;
    prod.g = 0;
    producer_set_item(prod, is);
    for (int i = 0; i < kStages; ++i) producer_issue(s, prod, is);
  }
  // a sampled starting threshold for long chunks (the ring is already filling)
  const uint32_t m_r = static_cast<uint32_t>(min64(k, c1 - c0));
  int mode0 = kAcceptAll;
  float thr0 = 0.f;
  if (kSample && c1 - c0 >= kSampleChunk && m_r > 0) {
    const float t = chunk_threshold(s, row_ptr, c0, c1, m_r, tid);
    if (t > __int_as_float(0xff800000)) {
      mode0 = kAtLeast;
      thr0 = t;
    }
  }
  uint32_t g = 0;
  int par = 0;
  bool compacted = false;
  uint32_t n_r = stream_ring(s, sp, c0, c1, k, g, par, mode0, thr0, compacted, tid, tid == 0 ? &prod : nullptr,
                             &is);
  if (kSample && mode0 == kAtLeast && !compacted && n_r < m_r) {
    // the sample's threshold let fewer than this rank's top-m_r through: redo exactly
    n_r = stream_global(s, sp, c0, c1, k, par, tid);
  }
  if (n_r > static_cast<uint32_t>(k)) {
    select_topk(s, 0, static_cast<int>(n_r), k, tid);
    n_r = static_cast<uint32_t>(k);
  }

  // ---- merge phase 1: publish (count, min key, max key) of this rank
  const MinMax mm = block_minmax(s, 0, static_cast<int>(n_r), tid);
  if (tid == 0) {
    s.pub[0] = n_r;
    s.pub[1] = mm.mn;
    s.pub[2] = mm.mx;
  }
  cluster_barrier();
  if (w == 0) {
    uint32_t n = 0, mn = 0xFFFFFFFFu, mx = 0u;
    if (lane < static_cast<int>(ncta)) {
      const uint32_t a = dsmem_map(smem_addr(&s.pub[0]), lane);
      n = dsmem_ld(a);
      mn = dsmem_ld(a + 4);
      mx = dsmem_ld(a + 8);
    }
    const bool full_rank = lane < static_cast<int>(ncta) && n == static_cast<uint32_t>(k);
    const uint32_t N = __reduce_add_sync(kFull, n);
    const uint32_t gmin = __reduce_min_sync(kFull, mn);
    const uint32_t gmax = __reduce_max_sync(kFull, mx);
    // a rank holding k entries >= its min bounds the global k-th key from below
    const uint32_t B = __reduce_max_sync(kFull, full_rank ? mn : 0u);
    const bool any_full = __ballot_sync(kFull, full_rank) != 0;
    if (lane == 0) {
      s.bc[2] = N;
      s.bc[3] = any_full ? B : gmin;
      s.bc[4] = gmax;
      s.bc[5] = gmin;
    }
  }
  bar_consumers();
  const uint32_t N = s.bc[2];
  uint32_t lo = s.bc[3], hi = s.bc[4];
  const uint32_t gmin = s.bc[5];
  bar_consumers();
  uint32_t need = m, S = N;
  bool exact = false;
  if (N <= static_cast<uint32_t>(kGatherCap)) {
    lo = gmin;  // everything fits at the leader
  } else {
    // ---- merge phase 2: cluster-wide histogram rounds until the survivors fit
    int hp = 0;
    for (int round = 0;; ++round) {
      if (lo == hi || round == kMaxRadixRounds + 1) {
        if (lo != hi && tid == 0) atomicOr(&g_status, kStatusSelectBroken);
        exact = true;
        break;
      }
      const int sh = window_shift(lo, hi);
      if (tid < 256) s.phist[hp][tid] = 0u;
      if (tid == 0) s.bc[0] = 0xFFFFFFFFu;
      bar_consumers();
      histogram(s, s.phist[hp], 0, static_cast<int>(n_r), lo, hi, sh, tid);
      cluster_barrier();
      if (tid < 256) {
        const uint32_t a = smem_addr(&s.phist[hp][tid]);
        uint32_t g = 0;
        for (uint32_t r = 0; r < ncta; ++r) g += dsmem_ld(dsmem_map(a, r));
        s.ghist[tid] = g;
      }
      bar_consumers();
      if (w == 0) find_bucket_warp0(s.ghist, need, s.bc, lane);
      bar_consumers();
      if (s.bc[0] == 0xFFFFFFFFu) {  // identical on every rank: the same sums
        if (tid == 0) atomicOr(&g_status, kStatusSelectBroken);
        exact = true;
        lo = hi;
        bar_consumers();
        break;
      }
      const uint32_t b = s.bc[0], above_b = s.bc[1];
      need -= above_b;
      S = (m - need) + s.ghist[b];  // keys above the bucket + keys in it
      narrow(lo, hi, sh, b);
      bar_consumers();
      hp ^= 1;
      if (S <= static_cast<uint32_t>(kGatherCap)) break;
    }
  }
  // ---- merge phase 3: publish this rank's survivor counts
  // exact: keep key > T plus a rank-ordered share of key == T; else keep key >= lo
  const uint32_t T = exact ? lo : lo - 1u;
  uint32_t g_r, q_r;
  count_gt_eq(s, 0, static_cast<int>(n_r), T, g_r, q_r, tid);
  if (tid == 0) {
    s.pub[4] = g_r;
    s.pub[5] = exact ? q_r : 0u;
  }
  cluster_barrier();
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
  bar_consumers();
  const uint32_t my_off = s.bc[6], my_keep = s.bc[7], total = s.bc[2];
  // ---- merge phase 4: copy survivors, in index order, into the leader
  const uint32_t rkey = dsmem_map(smem_addr(&s.ckey[kGatherOff]), 0);
  const uint32_t ridx = dsmem_map(smem_addr(&s.cidx[kGatherOff]), 0);
  stable_keep<true>(s, 0, static_cast<int>(n_r), T, exact ? my_keep : 0u, rkey, ridx, my_off, tid);
  cluster_barrier();
  if (rank != 0) return;
  // ---- leader: exact top-m of the gathered survivors, sort, write
  if (total > m) select_topk(s, kGatherOff, static_cast<int>(total), static_cast<int>(m), tid);
  const int R = sort_desc(s, kGatherOff, 0, static_cast<int>(m), tid);
  write_row(s, R, static_cast<int>(m), k, out + row * static_cast<int64_t>(k), tid);
}

#include "rows_path.cuh"

// ------------------------------------------------------------------ host
struct DeviceInfo {
  int sms = 0;
  int major = 0, minor = 0;
  int max_cluster = 0;  // largest supported cluster (16 or 8), 0 if none
  bool ready = false;
};

constexpr int kMaxDevices = 64;
static DeviceInfo g_dev[kMaxDevices];
static std::mutex g_dev_mu;

static int device_setup(int dev, DeviceInfo* out) {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return DSA_ERR_NO_DEVICE;
    if (p.major != 10) return DSA_ERR_NO_DEVICE;
    d.sms = p.multiProcessorCount;
    d.major = p.major;
    d.minor = p.minor;
    const int smem = static_cast<int>(sizeof(Smem));
    if (cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sizeof(rows::Smem))) != cudaSuccess ||
        cudaFuncSetAttribute(topk_cluster_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(topk_cluster_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
      cudaGetLastError();
      return DSA_ERR_CONFIG;
    }
    d.max_cluster = 0;
    for (int cs : {16, 8}) {
      if (cs > 8 &&
          (cudaFuncSetAttribute(topk_cluster_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
               cudaSuccess ||
           cudaFuncSetAttribute(topk_cluster_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
               cudaSuccess)) {
        cudaGetLastError();
        continue;
      }
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nclusters = 0;
      if (cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel<false>, &cfg) == cudaSuccess &&
          nclusters > 0) {
        d.max_cluster = cs;
        break;
      }
      cudaGetLastError();
    }
    d.ready = true;
  }
  *out = d;
  return DSA_OK;
}

// Launch plan from host-known sizes only.
static void plan(const DeviceInfo& d, int64_t num_rows, int64_t row_stride, int* cs_out, int64_t* grid_out) {
  constexpr int64_t kMinChunk = 16384;  // elements per rank worth a cluster merge
  int cs = 1;
  const int64_t row_slots = d.sms;                                         // one many-row CTA per SM
  const int64_t cluster_slots = static_cast<int64_t>(d.sms) * kBlocksPerSM;  // cluster CTAs per GPU
  if (num_rows < row_slots && d.max_cluster > 1) {
    int64_t want = cluster_slots / (num_rows > 0 ? num_rows : 1);
    while (cs * 2 <= want && cs * 2 <= d.max_cluster && row_stride / (cs * 2) >= kMinChunk) cs *= 2;
  }
  *cs_out = cs;
  if (cs == 1)
    *grid_out = num_rows < row_slots ? num_rows : row_slots;
  else
    *grid_out = num_rows * cs;
}

static int check_args(const void* logits, int64_t row_stride, const void* lengths, int64_t num_rows, int32_t k,
                      const void* out) {
  if (k < 1 || k > kMaxK) return DSA_ERR_BAD_K;
  if (row_stride < 1) return DSA_ERR_BAD_STRIDE;
  if (num_rows < 0) return DSA_ERR_BAD_ROWS;
  if (num_rows > 0 && row_stride > INT64_MAX / num_rows) return DSA_ERR_OVERFLOW;
  if (num_rows > 0 && num_rows > INT64_MAX / k) return DSA_ERR_OVERFLOW;
  if (num_rows == 0) return DSA_OK;
  if (!logits || !lengths || !out) return DSA_ERR_NULL_POINTER;
  if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(lengths) |
       reinterpret_cast<uintptr_t>(out)) &
      3u)
    return DSA_ERR_MISALIGNED;
  return DSA_OK;
}

static int current_device(DeviceInfo* info) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return DSA_ERR_NO_DEVICE;
  }
  return device_setup(dev, info);
}

static int launch(const DeviceInfo& d, const float* logits, int64_t row_stride, const int32_t* lengths,
                  int64_t num_rows, int32_t k, int32_t* out, cudaStream_t stream) {
  int cs;
  int64_t grid;
  plan(d, num_rows, row_stride, &cs, &grid);
  if (grid > 0x7fffffff) return DSA_ERR_OVERFLOW;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(Smem);
  cfg.stream = stream;
  cudaError_t e;
  if (cs == 1) {
    cfg.blockDim = dim3(rows::kThreads, 1, 1);
    cfg.dynamicSmemBytes = sizeof(rows::Smem);
    e = cudaLaunchKernelEx(&cfg, topk_rows_kernel, logits, row_stride, lengths, num_rows, static_cast<int>(k), out);
  } else {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the longest possible chunk decides whether any rank samples
    const int64_t max_chunk = (row_stride + cs - 1) / cs;
    if (max_chunk >= kSampleChunk)
      e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<true>, logits, row_stride, lengths, num_rows,
                             static_cast<int>(k), out);
    else
      e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<false>, logits, row_stride, lengths, num_rows,
                             static_cast<int>(k), out);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_LAUNCH;
  }
  return DSA_OK;
}

}  // namespace dsa

DSA_EXPORT int dsa_topk(const float* logits, int64_t row_stride, const int32_t* lengths, int64_t num_rows,
                        int32_t k, int32_t* out_idx, dsa_stream_t stream) {
  int rc = dsa::check_args(logits, row_stride, lengths, num_rows, k, out_idx);
  if (rc != DSA_OK || num_rows == 0) return rc;
  dsa::DeviceInfo d;
  rc = dsa::current_device(&d);
  if (rc != DSA_OK) return rc;
  return dsa::launch(d, logits, row_stride, lengths, num_rows, k, out_idx, stream);
}

DSA_EXPORT int dsa_topk_host(const float* h_logits, int64_t row_stride, const int32_t* h_lengths, int64_t num_rows,
                             int32_t k, int32_t* h_out, float* d_logits, int32_t* d_lengths, int32_t* d_out,
                             dsa_stream_t stream) {
  int rc = dsa::check_args(h_logits, row_stride, h_lengths, num_rows, k, h_out);
  if (rc != DSA_OK || num_rows == 0) return rc;
  rc = dsa::check_args(d_logits, row_stride, d_lengths, num_rows, k, d_out);
  if (rc != DSA_OK) return rc;
  dsa::DeviceInfo d;
  rc = dsa::current_device(&d);
  if (rc != DSA_OK) return rc;
  const size_t in_bytes = static_cast<size_t>(num_rows) * static_cast<size_t>(row_stride) * sizeof(float);
  if (cudaMemcpyAsync(d_logits, h_logits, in_bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemcpyAsync(d_lengths, h_lengths, static_cast<size_t>(num_rows) * sizeof(int32_t),
                      cudaMemcpyHostToDevice, stream) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_LAUNCH;
  }
  rc = dsa::launch(d, d_logits, row_stride, d_lengths, num_rows, k, d_out, stream);
  if (rc != DSA_OK) return rc;
  if (cudaMemcpyAsync(h_out, d_out, static_cast<size_t>(num_rows) * k * sizeof(int32_t), cudaMemcpyDeviceToHost,
                      stream) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_LAUNCH;
  }
  return DSA_OK;
}

DSA_EXPORT int dsa_topk_plan(int64_t num_rows, int64_t row_stride, int32_t k, int32_t* cluster_size, int32_t* grid) {
  if (k < 1 || k > dsa::kMaxK) return DSA_ERR_BAD_K;
  if (row_stride < 1) return DSA_ERR_BAD_STRIDE;
  if (num_rows < 0) return DSA_ERR_BAD_ROWS;
  dsa::DeviceInfo d;
  const int rc = dsa::current_device(&d);
  if (rc != DSA_OK) return rc;
  int cs;
  int64_t g;
  dsa::plan(d, num_rows, row_stride, &cs, &g);
  if (cluster_size) *cluster_size = cs;
  if (grid) *grid = static_cast<int32_t>(g > 0x7fffffff ? 0x7fffffff : g);
  return DSA_OK;
}

DSA_EXPORT int dsa_topk_device_status(uint32_t* status, int clear) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpyFromSymbol(&v, dsa::g_status, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_LAUNCH;
  }
  if (status) *status = v;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(dsa::g_status, &z, sizeof(z)) != cudaSuccess) {
      cudaGetLastError();
      return DSA_ERR_LAUNCH;
    }
  }
  return DSA_OK;
}

DSA_EXPORT const char* dsa_topk_strerror(int code) {
  switch (code) {
    case DSA_OK: return "success";
    case DSA_ERR_NULL_POINTER: return "a required pointer is NULL";
    case DSA_ERR_BAD_K: return "k must be in [1, 2048]";
    case DSA_ERR_BAD_STRIDE: return "row_stride must be >= 1";
    case DSA_ERR_BAD_ROWS: return "num_rows must be >= 0";
    case DSA_ERR_OVERFLOW: return "sizes overflow int64 / the launch grid";
    case DSA_ERR_MISALIGNED: return "a pointer is not 4-byte aligned";
    case DSA_ERR_NO_DEVICE: return "no current CUDA device of compute capability 10.x (sm_100)";
    case DSA_ERR_LAUNCH: return "the CUDA runtime rejected a launch or copy";
    case DSA_ERR_CONFIG: return "kernel attribute set-up failed on this device";
    default: return "unknown dsa_topk error code";
  }
}

DSA_EXPORT int dsa_topk_version(void) { return 100; }
