// Device helpers shared by the top-k kernel: status flags and test hooks,
// bounded mbarrier waits, bulk copies, cluster / distributed-shared-memory
// access, the order-preserving key map and the radix-select building blocks
// (digit histogram search, bound narrowing, the small exact finish).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_topk.h"

namespace dsa {

constexpr int kMaxK = DSA_TOPK_MAX_K;
constexpr uint32_t kNanKey = 0xFFC00000u;  // key of the canonical quiet NaN
constexpr uint32_t kInfKey = 0xFF800000u;  // key of +inf
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr unsigned long long kWaitLimitNs = 500000000ull;  // 0.5 s per pipeline wait

// Sticky status bits (g_status).
constexpr unsigned kStatusWaitTimeout = 1u;   // a pipeline wait gave up (error)
constexpr unsigned kStatusSelectBroken = 2u;  // a radix round lost its invariant (error)
constexpr unsigned kStatusReread = 4u;        // a speculative threshold was redone from global memory (info)

__device__ unsigned int g_status;  // sticky status bits, see kStatus*
// Test hooks (dsa_topk_set_test_hooks): the time limit of every pipeline wait,
// and a stage that each CTA's producer leaves unissued (-1: none), so that a
// test can make a wait run out without faulting anything.
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;
__device__ long long g_skip_stage = -1;

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
// Per-CTA wait control in shared memory: the abort flag raised by the first
// wait that gives up, and the time limit of every wait (copied from
// g_wait_limit_ns once at kernel start, so that a wait's slow path never
// stalls on a global load before it looks at its barrier again).
struct WaitCtl {
  uint32_t abort;
  uint32_t pad;
  unsigned long long limit_ns;
};

// Bounded wait. Returns false after the limit (recording the status bit and
// raising the CTA's abort flag), or at once when another thread of the CTA has
// raised that flag: the first wait that gives up ends every later one.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity, WaitCtl* ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile uint32_t*>(&ctl->abort)) return false;
    if (global_ns() - t0 > ctl->limit_ns) {
      atomicOr(&g_status, kStatusWaitTimeout);
      *reinterpret_cast<volatile uint32_t*>(&ctl->abort) = 1u;
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
__device__ __forceinline__ bool mbar_wait_sleep(unsigned long long* bar, uint32_t parity, WaitCtl* ctl) {
  if (mbar_try_wait_hint(bar, parity, 2000u)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (*reinterpret_cast<volatile uint32_t*>(&ctl->abort)) return false;
    if (global_ns() - t0 > ctl->limit_ns) {
      atomicOr(&g_status, kStatusWaitTimeout);
      *reinterpret_cast<volatile uint32_t*>(&ctl->abort) = 1u;
      return false;
    }
  }
}
// Drain: waits (bounded, ignoring the abort flag) until an issued bulk copy
// has landed, so that no copy is still writing into shared memory when the
// CTA exits. Copies from valid global memory always complete.
__device__ __forceinline__ void mbar_drain(unsigned long long* bar, uint32_t parity, const WaitCtl* ctl) {
  if (mbar_try_wait(bar, parity)) return;
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > ctl->limit_ns) {
      atomicOr(&g_status, kStatusWaitTimeout);
      return;
    }
  }
}
// Programmatic dependent launch: wait until the grids this launch depends on
// have completed and their writes are visible (a no-op without the launch
// attribute), then let the next launch in the stream be scheduled; its CTAs
// wait in their own griddepcontrol.wait until this grid completes.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
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
// Cluster barrier in the form any subset of a warp may execute (the aligned
// form below needs the whole warp at the same instruction).
__device__ __forceinline__ void cluster_barrier_any() {
  asm volatile(
      "barrier.cluster.arrive.release;\n\t"
      "barrier.cluster.wait.acquire;" ::
          : "memory");
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

// ------------------------------------------------------------ element types
// Logits come as fp32, bf16 or fp16. Every value is widened to fp32 (exact)
// before it is keyed, so all three share the key order above.
template <class T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kCode = DSA_DTYPE_F32;
  __device__ __forceinline__ static float f(float x) { return x; }
  // four consecutive elements at a 16-byte aligned address
  __device__ __forceinline__ static void four(const float* p, float (&x)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
  }
  __device__ __forceinline__ static void four_ldg(const float* p, float (&x)[4]) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
  }
  __device__ __forceinline__ static float one_ldg(const float* p) { return __ldg(p); }
};
template <class T, class T2, float2 (*kTo2)(T2), float (*kTo1)(T)>
struct Elem16 {
  __device__ __forceinline__ static float f(T x) { return kTo1(x); }
  // four consecutive elements at an 8-byte aligned address
  __device__ __forceinline__ static void four(const T* p, float (&x)[4]) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    unpack(q, x);
  }
  __device__ __forceinline__ static void four_ldg(const T* p, float (&x)[4]) {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
    unpack(q, x);
  }
  __device__ __forceinline__ static float one_ldg(const T* p) {
    return kTo1(__ushort_as_bf_or_h(__ldg(reinterpret_cast<const unsigned short*>(p))));
  }
  __device__ __forceinline__ static void unpack(uint2 q, float (&x)[4]) {
    const float2 a = kTo2(*reinterpret_cast<const T2*>(&q.x)), b = kTo2(*reinterpret_cast<const T2*>(&q.y));
    x[0] = a.x, x[1] = a.y, x[2] = b.x, x[3] = b.y;
  }
  __device__ __forceinline__ static T __ushort_as_bf_or_h(unsigned short u) { return *reinterpret_cast<T*>(&u); }
};
__device__ __forceinline__ float2 bf2_to_f2(__nv_bfloat162 v) { return __bfloat1622float2(v); }
__device__ __forceinline__ float bf_to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float2 h2_to_f2(__half2 v) { return __half22float2(v); }
__device__ __forceinline__ float h_to_f(__half v) { return __half2float(v); }
template <>
struct Elem<__nv_bfloat16> : Elem16<__nv_bfloat16, __nv_bfloat162, bf2_to_f2, bf_to_f> {
  static constexpr int kCode = DSA_DTYPE_BF16;
};
template <>
struct Elem<__half> : Elem16<__half, __half2, h2_to_f2, h_to_f> {
  static constexpr int kCode = DSA_DTYPE_F16;
};

// ------------------------------------------------------------ row geometry

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ int64_t clamp_len(const int32_t* lengths, int64_t row, int64_t row_stride) {
  int64_t L = lengths[row];
  if (L < 0) L = 0;
  if (L > row_stride) L = row_stride;
  return L;
}

// --------------------------------------------------- radix-select pieces

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

// Exact need-th largest key among the <= 32 keys in [lo, hi] (warp 0). Every
// lane holds one key (or 0, below any real key); returns the largest key x with
// #{keys >= x} >= need.
__device__ __forceinline__ uint32_t small_kth(uint32_t mine, uint32_t need) {
  uint32_t ge = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) ge += __shfl_sync(kFull, mine, j) >= mine;
  return __reduce_max_sync(kFull, (mine != 0u && ge >= need) ? mine : 0u);
}

}  // namespace dsa
