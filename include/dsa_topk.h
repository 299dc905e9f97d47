/*
 * dsa_topk.h -- strided indexer top-k for the DeepSeek-V4 sparse-attention
 * indexer, hand-written for NVIDIA B200 (sm_100a).
 *
 * C ABI. Every pointer is plain memory; there are no framework types in any
 * signature. All functions are thread-safe. Nothing here aborts or throws:
 * failures come back as negative return codes (see dsa_topk_strerror).
 *
 * Method sources (the pages this library restates):
 *   - vLLM PR #42169 report, "实现拆解" items 1-2: a row of logits starts at
 *     row * stride(0); the valid width of a row is shorter than its stride
 *     because the DeepGEMM logits are padded to a multiple of 256 and then
 *     sliced (non-contiguous). Using size(1) as the stride was the bug.
 *   - SGLang PR #34167 code excerpt (TopKCluster::forward, phase 3): indices
 *     are row-local (chunk_start + local index); values above the threshold
 *     are taken outright and values equal to it are resolved separately.
 *   - SGLang PR #34167 "实现拆解" item 4: k up to 2048 (k in {512, 1024, 2048}).
 */
#ifndef DSA_TOPK_H_
#define DSA_TOPK_H_

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream). NULL = the legacy default
 * stream of the calling thread's current device. */
typedef struct CUstream_st* dsa_stream_t;

/* Return codes. */
#define DSA_OK 0
#define DSA_ERR_NULL_POINTER -1   /* a required pointer is NULL */
#define DSA_ERR_BAD_K -2          /* k outside [1, DSA_TOPK_MAX_K] */
#define DSA_ERR_BAD_STRIDE -3     /* row_stride < 1 */
#define DSA_ERR_BAD_ROWS -4       /* num_rows < 0 */
#define DSA_ERR_OVERFLOW -5       /* num_rows * row_stride (or * k) overflows int64 */
#define DSA_ERR_MISALIGNED -6     /* a pointer is not 4-byte aligned */
#define DSA_ERR_NO_DEVICE -7      /* no current CUDA device, or it is not compute capability 10.0 */
#define DSA_ERR_LAUNCH -8         /* the CUDA runtime rejected a launch or a copy */
#define DSA_ERR_CONFIG -9         /* kernel attribute set-up failed on this device */
#define DSA_ERR_BAD_DTYPE -10     /* dtype is not one of DSA_DTYPE_* */
#define DSA_ERR_BAD_FLAGS -11     /* flags holds bits other than DSA_FLAG_* */

#define DSA_TOPK_MAX_K 2048

/* Element types of the logits (dsa_topk_ex). */
#define DSA_DTYPE_F32 0
#define DSA_DTYPE_BF16 1
#define DSA_DTYPE_F16 2

/* Flags (dsa_topk_ex). */
#define DSA_FLAG_UNSORTED 1u /* the row's top-k index set, in unspecified order */

/* Device status bits (dsa_topk_device_status). */
#define DSA_STATUS_WAIT_TIMEOUT 1u   /* error: a pipeline wait gave up; that call's output is undefined */
#define DSA_STATUS_SELECT_BROKEN 2u  /* error: a radix select lost its invariant (never expected) */
#define DSA_STATUS_REREAD 4u         /* info: a row's speculative threshold let too few values
                                        through and the row was read again (the result is exact) */
#define DSA_STATUS_ERRORS (DSA_STATUS_WAIT_TIMEOUT | DSA_STATUS_SELECT_BROKEN)

/*
 * dsa_topk -- per-row top-k indices of fp32 logits over a valid prefix.
 *
 * For each row r in [0, num_rows):
 *   L_r = clamp(lengths[r], 0, row_stride), m_r = min(k, L_r);
 *   the m_r indices j in [0, L_r) of the largest values logits[r*row_stride+j]
 *   are written to out_idx[r*k + 0 .. m_r-1], ordered by value descending,
 *   equal values by ascending index; out_idx[r*k + m_r .. k-1] = -1.
 *   Order on values: NaN (any payload) above +inf, -0.0 equal to +0.0,
 *   -inf is an ordinary value (it can be selected).
 *
 * Arguments:
 *   logits     device, fp32. Row r starts at logits + r*row_stride. Must be
 *              4-byte aligned; any alignment beyond that and any stride are
 *              accepted. Entries past L_r are never used (their values do not
 *              affect the result). Rows are fetched in 16-byte aligned blocks:
 *              a row may be read up to 12 bytes BEFORE its first element
 *              (for row 0 that is before `logits` itself) and up to 12 bytes
 *              past its last valid element, never leaving the 16-byte aligned
 *              blocks that hold those two elements. Those bytes must be
 *              readable device memory; they are whenever the buffer comes from
 *              one cudaMalloc (or PyTorch) allocation, whose base is aligned.
 *   row_stride elements (not bytes) between consecutive rows: the tensor's
 *              stride(0). >= 1.
 *   lengths    device, int32[num_rows]. Values outside [0, row_stride] are
 *              clamped on the device (no error, no host synchronisation).
 *   num_rows   >= 0. 0 launches nothing and returns DSA_OK.
 *   k          1 .. DSA_TOPK_MAX_K.
 *   out_idx    device, int32[num_rows * k], rows of k, contiguous. Must not
 *              overlap logits.
 *   stream     the call is asynchronous on this stream.
 *
 * Ownership: the caller owns every buffer; the library allocates no memory
 * at all (its working storage is on-chip shared memory) and keeps no pointer
 * after returning. Buffers must stay
 * valid until the stream reaches the call. The call can be captured in a CUDA
 * graph once the device has seen one uncaptured call (that first call sets
 * per-device kernel attributes). Launches use programmatic dependent launch:
 * a call may be scheduled while the previous kernel in the stream drains, and
 * touches no input or output until that kernel has completed.
 *
 * Errors: argument errors return before any launch; DSA_ERR_LAUNCH carries a
 * CUDA runtime failure of the launch. A device-side wait that exceeds its
 * time limit records a flag readable with dsa_topk_device_status().
 */
int dsa_topk(const float* logits, int64_t row_stride, const int32_t* lengths,
             int64_t num_rows, int32_t k, int32_t* out_idx, dsa_stream_t stream);

/*
 * dsa_topk_ex -- dsa_topk with three options. No page fixes these options;
 * each is the plain reading of a step the pages mention:
 *
 *   dtype        DSA_DTYPE_F32, DSA_DTYPE_BF16 or DSA_DTYPE_F16: the element
 *                type of `logits` (row_stride is in elements of that type;
 *                `logits` aligned to the element size). Values are widened to
 *                fp32 exactly before they are compared, with the order of
 *                dsa_topk. Lower-precision logits halve the bytes read.
 *   flags        DSA_FLAG_UNSORTED: out[r*k .. r*k + m_r - 1] holds the same
 *                index SET as dsa_topk (ties still go to the lowest indices),
 *                in an unspecified order; the -1 padding is unchanged. The
 *                SGLang PR #34167 code excerpt (TopKCluster::forward, phase 3)
 *                emits its indices at atomic positions, i.e. as a set.
 *   index_table  NULL, or device int32: then each selected row-local index j
 *                of row r is written as index_table[r*table_stride + j]
 *                instead of j (-1 padding stays -1). Row r of the table must
 *                hold at least L_r entries; table_stride >= 1, in elements.
 *                This is the index "transform" applied at the end of the
 *                SGLang top-k kernels (SGLang PR #34167 code excerpt:
 *                problem_transform into get_output_ptr, topk_transform_512),
 *                read here as a per-row lookup table, e.g. token position ->
 *                KV-cache slot (vLLM PR #52823 perf script: block_table,
 *                slot_mapping).
 *
 * All other arguments, the ownership rules and the codes are those of
 * dsa_topk (DSA_ERR_BAD_DTYPE / DSA_ERR_BAD_FLAGS in addition).
 */
int dsa_topk_ex(const void* logits, int32_t dtype, int64_t row_stride,
                const int32_t* lengths, int64_t num_rows, int32_t k, uint32_t flags,
                const int32_t* index_table, int64_t table_stride, int32_t* out_idx,
                dsa_stream_t stream);

/*
 * dsa_topk_host -- the same operation on HOST buffers, with the copies on
 * `stream`: h_logits (num_rows*row_stride floats) and h_lengths are copied to
 * the caller's device buffers d_logits / d_lengths, dsa_topk runs on them into
 * d_out, and d_out is copied back to h_out (num_rows*k int32). Pinned host
 * memory makes the copies asynchronous; the caller synchronises the stream
 * before reading h_out. Same argument rules and codes as dsa_topk.
 */
int dsa_topk_host(const float* h_logits, int64_t row_stride, const int32_t* h_lengths,
                  int64_t num_rows, int32_t k, int32_t* h_out,
                  float* d_logits, int32_t* d_lengths, int32_t* d_out, dsa_stream_t stream);

/*
 * dsa_topk_plan -- the launch dsa_topk would choose on the current device for
 * these host-known sizes (it never looks at lengths). cluster_size = CTAs
 * that share one row (1 = one CTA per row, persistent over rows; > 1 = a
 * thread-block cluster per row, chosen only when every cluster of the launch
 * is resident at once); grid = CTAs launched. Either output pointer may be NULL. Returns DSA_OK or an error
 * code as dsa_topk would.
 */
int dsa_topk_plan(int64_t num_rows, int64_t row_stride, int32_t k,
                  int32_t* cluster_size, int32_t* grid);

/*
 * dsa_topk_device_status -- sticky device-side status bits of the current
 * device (DSA_STATUS_*; DSA_STATUS_ERRORS are the error bits). Synchronises
 * the device. With clear != 0 the bits are reset to 0 afterwards. Returns
 * DSA_OK or DSA_ERR_LAUNCH.
 *
 * Every wait inside a kernel is bounded (0.5 s by default). The first wait
 * that gives up sets DSA_STATUS_WAIT_TIMEOUT and ends every other wait of its
 * CTA at once: the CTA's roles leave their loops together, the producer waits
 * for the bulk copies it already issued, and the kernel returns. The output
 * of that call is undefined (rows split across a cluster are written as -1);
 * the device stays usable and later calls are unaffected.
 */
int dsa_topk_device_status(uint32_t* status, int clear);

/*
 * dsa_topk_set_test_hooks -- TEST USE ONLY. Sets, on the current device, the
 * time limit of every pipeline wait (wait_limit_ns; 0 restores the default
 * 0.5 s) and a stage index that each CTA's producer leaves unissued
 * (skip_stage; -1 disables). With a stage skipped, the consumers' wait for it
 * runs out after the limit and the call ends through the path described at
 * dsa_topk_device_status: no copy is aimed at bad memory and nothing faults.
 * Synchronous. Returns DSA_OK or DSA_ERR_LAUNCH.
 */
int dsa_topk_set_test_hooks(uint64_t wait_limit_ns, int64_t skip_stage);

/* Human-readable text for a return code (static storage). */
const char* dsa_topk_strerror(int code);

/* Library version as an integer: major*10000 + minor*100 + patch. */
int dsa_topk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_TOPK_H_ */
