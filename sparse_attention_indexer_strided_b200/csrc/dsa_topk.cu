// Strided indexer top-k for B200 (sm_100a): host side and the C ABI.
//
// Operation (vLLM PR #42169 report, "实现拆解"; SGLang PR #34167 code
// excerpt): for each row r of logits at logits + r*row_stride, the k largest
// of the first L_r values, as row-local indices ordered by value descending
// and index ascending, padded with -1 past min(k, L_r).
//
// One kernel (topk_kernel.cuh), instantiated for fp32, bf16 and fp16 logits,
// with two launch shapes chosen here from host-known sizes only:
//   * many rows: one persistent CTA per SM (grid = min(rows, SMs)), rows
//     strided over the grid;
//   * few long rows: a thread-block cluster per row (grid = rows x cluster
//     size), when the whole grid fits on the GPU at once.
// The library allocates nothing: all working storage is shared memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "dsa_topk.h"
#include "topk_kernel.cuh"

#define DSA_EXPORT extern "C" __attribute__((visibility("default")))

namespace dsa {

struct DeviceInfo {
  int sms = 0;
  // CTAs of a cluster launch of size 2, 4, 8, 16 that can be resident at once
  // (index log2 of the size; 0: that size does not launch on this device)
  int cluster_ctas[5] = {0, 0, 0, 0, 0};
  bool ready = false;
};

constexpr int kMaxDevices = 64;
static DeviceInfo g_dev[kMaxDevices];
static std::mutex g_dev_mu;

template <class T>
static bool set_kernel_attributes() {
  const int smem = static_cast<int>(sizeof(rows::Smem));
  if (cudaFuncSetAttribute(topk_rows_kernel<T, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(topk_rows_kernel<T, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(topk_cluster_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cudaFuncSetAttribute(topk_cluster_kernel<T>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    cudaGetLastError();  // then only portable sizes (<= 8) launch
  return true;
}

static int device_setup(int dev, DeviceInfo* out) {
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) {
      cudaGetLastError();
      return DSA_ERR_NO_DEVICE;
    }
    // the library carries sm_100a code only, which runs on compute capability
    // 10.0 alone; the attribute query fails when no image loads on this device
    cudaFuncAttributes fa;
    if (p.major != 10 || p.minor != 0 || cudaFuncGetAttributes(&fa, topk_rows_kernel<float, false>) != cudaSuccess) {
      cudaGetLastError();
      return DSA_ERR_NO_DEVICE;
    }
    d.sms = p.multiProcessorCount;
    if (!set_kernel_attributes<float>() || !set_kernel_attributes<__nv_bfloat16>() ||
        !set_kernel_attributes<__half>())
      return DSA_ERR_CONFIG;
    for (int i = 1; i < 5; ++i) {
      const int cs = 1 << i;
      d.cluster_ctas[i] = 0;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(cs, 1, 1);
      cfg.blockDim = dim3(rows::kClusterThreads, 1, 1);
      cfg.dynamicSmemBytes = sizeof(rows::Smem);
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nclusters = 0;
      if (cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel<float>, &cfg) == cudaSuccess)
        d.cluster_ctas[i] = nclusters * cs;
      else
        cudaGetLastError();
    }
    d.ready = true;
  }
  *out = d;
  return DSA_OK;
}

// Launch plan from host-known sizes only. A cluster per row pays off when rows
// are few and long: each rank then streams a chunk of at least kMinChunk
// elements. From 32 rows on, one CTA per row finishes sooner unless the rows
// are long (kLongRow elements and up): the merge costs more than the split
// saves. The largest cluster size whose whole grid is resident at once is
// taken (the merge waits on every rank of a cluster).
static void plan(const DeviceInfo& d, int64_t num_rows, int64_t row_stride, int* cs_out, int64_t* grid_out) {
  constexpr int64_t kMinChunk = 16384;
  constexpr int64_t kLongRow = 262144;
  int cs = 1;
  if (num_rows > 0 && num_rows < d.sms && (num_rows < 32 || row_stride >= kLongRow)) {
    for (int i = 1; i < 5; ++i) {
      const int c = 1 << i;
      if (d.cluster_ctas[i] >= num_rows * c && row_stride / c >= kMinChunk) cs = c;
    }
  }
  *cs_out = cs;
  if (cs == 1)
    *grid_out = num_rows < d.sms ? num_rows : d.sms;
  else
    *grid_out = num_rows * cs;
}

static int elem_size(int32_t dtype) {
  switch (dtype) {
    case DSA_DTYPE_F32: return 4;
    case DSA_DTYPE_BF16:
    case DSA_DTYPE_F16: return 2;
    default: return 0;
  }
}

static int check_args(const void* logits, int32_t dtype, int64_t row_stride, const void* lengths, int64_t num_rows,
                      int32_t k, uint32_t flags, const void* table, int64_t table_stride, const void* out) {
  const int es = elem_size(dtype);
  if (es == 0) return DSA_ERR_BAD_DTYPE;
  if (flags & ~static_cast<uint32_t>(DSA_FLAG_UNSORTED)) return DSA_ERR_BAD_FLAGS;
  if (k < 1 || k > kMaxK) return DSA_ERR_BAD_K;
  if (row_stride < 1) return DSA_ERR_BAD_STRIDE;
  if (num_rows < 0) return DSA_ERR_BAD_ROWS;
  if (table && table_stride < 1) return DSA_ERR_BAD_STRIDE;
  if (num_rows > 0 && row_stride > INT64_MAX / num_rows) return DSA_ERR_OVERFLOW;
  if (num_rows > 0 && num_rows > INT64_MAX / k) return DSA_ERR_OVERFLOW;
  if (table && num_rows > 0 && table_stride > INT64_MAX / num_rows) return DSA_ERR_OVERFLOW;
  if (num_rows == 0) return DSA_OK;
  if (!logits || !lengths || !out) return DSA_ERR_NULL_POINTER;
  if ((reinterpret_cast<uintptr_t>(logits) & static_cast<uintptr_t>(es - 1)) ||
      ((reinterpret_cast<uintptr_t>(lengths) | reinterpret_cast<uintptr_t>(out) |
        reinterpret_cast<uintptr_t>(table)) &
       3u))
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

template <class T>
static cudaError_t launch_as(const cudaLaunchConfig_t& cfg, const rows::Params& p, bool clustered) {
  if (clustered) return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<T>, p);
  // rows that always fit one stage take the kernel instance that copies a
  // stage with no threshold whole
  if (p.row_stride <= rows::kShortStride) return cudaLaunchKernelEx(&cfg, topk_rows_kernel<T, true>, p);
  return cudaLaunchKernelEx(&cfg, topk_rows_kernel<T, false>, p);
}

static int launch(const DeviceInfo& d, int32_t dtype, const rows::Params& p, cudaStream_t stream) {
  int cs;
  int64_t grid;
  plan(d, p.num_rows, p.row_stride, &cs, &grid);
  if (grid > 0x7fffffff) return DSA_ERR_OVERFLOW;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(cs == 1 ? rows::kThreads : rows::kClusterThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(rows::Smem);
  cfg.stream = stream;
  // programmatic dependent launch: this grid may be scheduled while the
  // previous kernel in the stream drains; its griddepcontrol.wait holds every
  // access to inputs and outputs until that kernel has completed
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cs;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cs == 1 ? 1 : 2;
  cudaError_t e;
  switch (dtype) {
    case DSA_DTYPE_F32: e = launch_as<float>(cfg, p, cs > 1); break;
    case DSA_DTYPE_BF16: e = launch_as<__nv_bfloat16>(cfg, p, cs > 1); break;
    default: e = launch_as<__half>(cfg, p, cs > 1); break;
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_LAUNCH;
  }
  return DSA_OK;
}

static int run(const void* logits, int32_t dtype, int64_t row_stride, const int32_t* lengths, int64_t num_rows,
               int32_t k, uint32_t flags, const int32_t* table, int64_t table_stride, int32_t* out,
               cudaStream_t stream) {
  int rc = check_args(logits, dtype, row_stride, lengths, num_rows, k, flags, table, table_stride, out);
  if (rc != DSA_OK || num_rows == 0) return rc;
  DeviceInfo d;
  rc = current_device(&d);
  if (rc != DSA_OK) return rc;
  const rows::Params p{logits, row_stride, lengths, num_rows, k, flags, table, table ? table_stride : 0, out};
  return launch(d, dtype, p, stream);
}

}  // namespace dsa

DSA_EXPORT int dsa_topk(const float* logits, int64_t row_stride, const int32_t* lengths, int64_t num_rows,
                        int32_t k, int32_t* out_idx, dsa_stream_t stream) {
  return dsa::run(logits, DSA_DTYPE_F32, row_stride, lengths, num_rows, k, 0u, nullptr, 0, out_idx, stream);
}

DSA_EXPORT int dsa_topk_ex(const void* logits, int32_t dtype, int64_t row_stride, const int32_t* lengths,
                           int64_t num_rows, int32_t k, uint32_t flags, const int32_t* index_table,
                           int64_t table_stride, int32_t* out, dsa_stream_t stream) {
  return dsa::run(logits, dtype, row_stride, lengths, num_rows, k, flags, index_table, table_stride, out, stream);
}

DSA_EXPORT int dsa_topk_host(const float* h_logits, int64_t row_stride, const int32_t* h_lengths, int64_t num_rows,
                             int32_t k, int32_t* h_out, float* d_logits, int32_t* d_lengths, int32_t* d_out,
                             dsa_stream_t stream) {
  int rc = dsa::check_args(h_logits, DSA_DTYPE_F32, row_stride, h_lengths, num_rows, k, 0u, nullptr, 0, h_out);
  if (rc != DSA_OK || num_rows == 0) return rc;
  rc = dsa::check_args(d_logits, DSA_DTYPE_F32, row_stride, d_lengths, num_rows, k, 0u, nullptr, 0, d_out);
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
  const dsa::rows::Params p{d_logits, row_stride, d_lengths, num_rows, k, 0u, nullptr, 0, d_out};
  rc = dsa::launch(d, DSA_DTYPE_F32, p, stream);
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

DSA_EXPORT int dsa_topk_set_test_hooks(uint64_t wait_limit_ns, int64_t skip_stage) {
  const unsigned long long lim = wait_limit_ns ? static_cast<unsigned long long>(wait_limit_ns) : dsa::kWaitLimitNs;
  const long long skip = skip_stage < 0 ? -1ll : static_cast<long long>(skip_stage);
  if (cudaMemcpyToSymbol(dsa::g_wait_limit_ns, &lim, sizeof(lim)) != cudaSuccess ||
      cudaMemcpyToSymbol(dsa::g_skip_stage, &skip, sizeof(skip)) != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_LAUNCH;
  }
  return DSA_OK;
}

DSA_EXPORT const char* dsa_topk_strerror(int code) {
  switch (code) {
    case DSA_OK: return "success";
    case DSA_ERR_NULL_POINTER: return "a required pointer is NULL";
    case DSA_ERR_BAD_K: return "k must be in [1, 2048]";
    case DSA_ERR_BAD_STRIDE: return "row_stride (and table_stride, with a table) must be >= 1";
    case DSA_ERR_BAD_ROWS: return "num_rows must be >= 0";
    case DSA_ERR_OVERFLOW: return "sizes overflow int64 / the launch grid";
    case DSA_ERR_MISALIGNED: return "a pointer is not aligned to its element size";
    case DSA_ERR_NO_DEVICE: return "no current CUDA device of compute capability 10.0 (sm_100a)";
    case DSA_ERR_LAUNCH: return "the CUDA runtime rejected a launch or copy";
    case DSA_ERR_CONFIG: return "kernel attribute set-up failed on this device";
    case DSA_ERR_BAD_DTYPE: return "dtype must be DSA_DTYPE_F32, DSA_DTYPE_BF16 or DSA_DTYPE_F16";
    case DSA_ERR_BAD_FLAGS: return "unknown flag bits";
    default: return "unknown dsa_topk error code";
  }
}

DSA_EXPORT int dsa_topk_version(void) { return 200; }
